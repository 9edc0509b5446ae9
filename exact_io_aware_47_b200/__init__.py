"""Exact tiled attention for B200 (sm_100a): a CUDA library with a C ABI
(``include/fa.h``) and a thin Python binding.

    from exact_io_aware_47_b200 import forward, backward
    o, lse = forward(q, k, v, causal=True)
    dq, dk, dv = backward(q, k, v, o, lse, do, causal=True)

Packed variable-length batches ([H, T, d], sequence b in rows
cu_seqlens[b] .. cu_seqlens[b + 1] - 1): ``forward_varlen`` /
``backward_varlen``.  Block-sparse attention (a [nt, nt] mask over 128 x 128
score tiles): ``forward_blocksparse`` / ``backward_blocksparse``.  Dropout on
the probabilities (Philox4x32-10 mask from seed and offset):
``forward_dropout`` / ``backward_dropout``.  8-bit inputs with one descale
per 128-row tile: ``quantize_e4m3`` / ``forward_e4m3``.

The CUDA library is loaded on first use; a missing library raises instead of
falling back to anything else.
"""

from .attention import (backward, backward_blocksparse, backward_dropout, backward_varlen,
                        device_status, forward, forward_blocksparse, forward_dropout,
                        forward_e4m3, forward_varlen, quantize_e4m3, workspace_bytes)

__all__ = ["forward", "backward", "forward_varlen", "backward_varlen", "forward_blocksparse",
           "backward_blocksparse", "forward_dropout", "backward_dropout", "quantize_e4m3",
           "forward_e4m3", "workspace_bytes", "device_status"]
