"""ctypes binding of the C ABI in ``include/fa.h`` (marshalling only).

The functions keep the C names and arguments; every computation happens in
the CUDA library.  Loading fails loudly when the library is missing: there is
no fallback of any kind.
"""

import ctypes
import os

from .build import LIB_PATH

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_ALIGNMENT = 3
FA_ERR_ARCH = 4
FA_ERR_CUDA = 5
FA_ERR_DEVICE_TIMEOUT = 6
FA_ERR_DEVICE_SEQLEN = 7
FA_ERR_WORKSPACE = 8
FA_ERR_DEVICE_LAYOUT = 9
FA_ERR_SCRATCH_LIMIT = 10
FA_ERR_DEVICE_SCALE = 11

FA_BF16 = 0
FA_FP16 = 1

# exported symbol -> (restype, argtypes)
_VP, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _VP, _I, _VP]),
    "fa_bwd_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "fa_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ,
                    _I, _I, _I, _I, _F, _I, _VP, _I, _VP]),
    "fa_bwd_preprocess": (_I, [_VP, _VP, _VP, _SZ, _I, _I, _I, _I, _I, _VP]),
    "fa_bwd_main": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _I, _I, _I, _I, _F, _I, _VP,
                         _I, _VP]),
    "fa_bwd_postprocess": (_I, [_VP, _SZ, _VP, _I, _I, _I, _I, _F, _I, _VP]),
    "fa_bwd_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                            _I, _I, _I, _I, _F, _I, _VP, _I, _VP]),
    "fa_bwd_noalloc_max_bytes": (_SZ, []),
    "fa_fwd_dropout": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _VP, _F,
                            ctypes.c_uint64, ctypes.c_uint32, _I, _VP]),
    "fa_bwd_dropout": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ,
                            _I, _I, _I, _I, _F, _I, _VP, _F, ctypes.c_uint64, ctypes.c_uint32,
                            _I, _VP]),
    "fa_fwd_blocksparse": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _VP, _I,
                                _VP]),
    "fa_bwd_blocksparse": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP,
                                _I, _I, _I, _I, _F, _I, _VP, _I, _VP]),
    "fa_fwd_varlen": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "fa_bwd_varlen_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "fa_bwd_varlen": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP,
                           _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "fa_quantize_e4m3": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP]),
    "fa_fwd_e4m3": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _VP, _I,
                         _VP]),
    "fa_set_wait_limit_ns": (ctypes.c_ulonglong, [ctypes.c_ulonglong]),
    "fa_device_status": (_I, [_VP, ctypes.POINTER(ctypes.c_uint32)]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_version": (_I, []),
}

_lib = None


class FAError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


def load(path=None):
    """Load (once) and return the CUDA library; raises if it is not built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"CUDA library {p} is missing: run exact_io_aware_47_b200.build.build() "
                           "(there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def status_string(status):
    return load().fa_status_string(status).decode()


def check(fn_name, status):
    if status != FA_OK:
        raise FAError(fn_name, status, status_string(status))
    return status


def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, seqlens, dtype, stream):
    return load().fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, seqlens, dtype, stream)


def fa_bwd_workspace_size(B, H, N, d):
    return load().fa_bwd_workspace_size(B, H, N, d)


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N, d, scale,
           causal, seqlens, dtype, stream):
    return load().fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N,
                         d, scale, causal, seqlens, dtype, stream)


def fa_bwd_preprocess(o, dout, workspace, workspace_bytes, B, H, N, d, dtype, stream):
    return load().fa_bwd_preprocess(o, dout, workspace, workspace_bytes, B, H, N, d, dtype, stream)


def fa_bwd_main(q, k, v, dout, lse, dk, dv, workspace, workspace_bytes, B, H, N, d, scale, causal,
                seqlens, dtype, stream):
    return load().fa_bwd_main(q, k, v, dout, lse, dk, dv, workspace, workspace_bytes, B, H, N, d,
                              scale, causal, seqlens, dtype, stream)


def fa_bwd_postprocess(workspace, workspace_bytes, dq, B, H, N, d, scale, dtype, stream):
    return load().fa_bwd_postprocess(workspace, workspace_bytes, dq, B, H, N, d, scale, dtype,
                                     stream)


def fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, seqlens, dtype,
                   stream):
    return load().fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal,
                                 seqlens, dtype, stream)


def fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, scale, causal, seqlens, p_drop, seed, offset,
                   dtype, stream):
    return load().fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, scale, causal, seqlens, p_drop,
                                 seed, offset, dtype, stream)


def fa_bwd_dropout(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N, d,
                   scale, causal, seqlens, p_drop, seed, offset, dtype, stream):
    return load().fa_bwd_dropout(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes,
                                 B, H, N, d, scale, causal, seqlens, p_drop, seed, offset, dtype,
                                 stream)


def fa_fwd_blocksparse(q, k, v, o, lse, block_mask, B, H, N, d, scale, causal, seqlens, dtype,
                       stream):
    return load().fa_fwd_blocksparse(q, k, v, o, lse, block_mask, B, H, N, d, scale, causal,
                                     seqlens, dtype, stream)


def fa_bwd_blocksparse(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, block_mask,
                       B, H, N, d, scale, causal, seqlens, dtype, stream):
    return load().fa_bwd_blocksparse(q, k, v, o, dout, lse, dq, dk, dv, workspace,
                                     workspace_bytes, block_mask, B, H, N, d, scale, causal,
                                     seqlens, dtype, stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, B, H, T, max_seqlen, d, scale, causal, dtype,
                  stream):
    return load().fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, B, H, T, max_seqlen, d, scale, causal,
                                dtype, stream)


def fa_bwd_varlen_workspace_size(B, H, T, d):
    return load().fa_bwd_varlen_workspace_size(B, H, T, d)


def fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, cu_seqlens, B, H,
                  T, max_seqlen, d, scale, causal, dtype, stream):
    return load().fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes,
                                cu_seqlens, B, H, T, max_seqlen, d, scale, causal, dtype, stream)


def fa_quantize_e4m3(x, x8, descale, B, H, N, d, dtype, stream):
    return load().fa_quantize_e4m3(x, x8, descale, B, H, N, d, dtype, stream)


def fa_fwd_e4m3(q8, k8, v8, q_descale, k_descale, v_descale, o, lse, B, H, N, d, scale, causal,
                seqlens, out_dtype, stream):
    return load().fa_fwd_e4m3(q8, k8, v8, q_descale, k_descale, v_descale, o, lse, B, H, N, d,
                              scale, causal, seqlens, out_dtype, stream)


def fa_bwd_noalloc_max_bytes():
    return load().fa_bwd_noalloc_max_bytes()


def fa_set_wait_limit_ns(ns):
    """Bound of every pipeline wait of later launches (0: the 2 s default);
    returns the previous bound."""
    return load().fa_set_wait_limit_ns(ns)


def fa_device_status(stream):
    """Returns (status, raw_word)."""
    word = ctypes.c_uint32(0)
    st = load().fa_device_status(stream, ctypes.byref(word))
    return st, word.value


def fa_version():
    return load().fa_version()
