"""CPU float64 oracle for exact tiled attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it.  The CUDA library and its
Python binding never import it, and it imports nothing from them.
"""

from .attention import (allowed_mask, ref_bwd, ref_bwd_slice, ref_fwd,
                        ref_fwd_slice)
from .dropout import (keep_mask, keep_threshold, philox4x32_10, ref_bwd_dropout_slice,
                      ref_fwd_dropout_slice)
from .fp8 import (dequantize_tiles, e4m3_decode, e4m3_encode, e4m3_round, fp8_error_bound,
                  quantize_tiles, ref_fwd_fp8_slice)
from .online_model import tiled_fwd_slice

__all__ = ["allowed_mask", "ref_fwd_slice", "ref_fwd", "ref_bwd_slice",
           "ref_bwd", "tiled_fwd_slice", "philox4x32_10", "keep_threshold", "keep_mask",
           "ref_fwd_dropout_slice", "ref_bwd_dropout_slice", "e4m3_round", "e4m3_encode",
           "e4m3_decode", "quantize_tiles", "dequantize_tiles", "ref_fwd_fp8_slice",
           "fp8_error_bound"]
