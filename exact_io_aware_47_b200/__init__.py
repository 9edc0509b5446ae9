"""Exact tiled attention for B200 (sm_100a): a CUDA library with a C ABI
(``include/fa.h``) and a thin Python binding.

    from exact_io_aware_47_b200 import forward, backward
    o, lse = forward(q, k, v, causal=True)
    dq, dk, dv = backward(q, k, v, o, lse, do, causal=True)

The CUDA library is loaded on first use; a missing library raises instead of
falling back to anything else.
"""

from .attention import backward, device_status, forward, workspace_bytes

__all__ = ["forward", "backward", "workspace_bytes", "device_status"]
