"""torch-facing calls of the CUDA library: allocate outputs, pass pointers.

``forward`` and ``backward`` ([B, H, N, d]), ``forward_dropout`` /
``backward_dropout`` (dropout on the probabilities), ``forward_blocksparse`` /
``backward_blocksparse`` (the same with a 128 x 128 tile mask) and
``forward_varlen`` / ``backward_varlen`` (packed [H, T, d] with cu_seqlens),
``quantize_e4m3`` / ``forward_e4m3`` (8-bit inputs with per-tile descales)
validate tensor
properties that ctypes cannot see (device, dtype, contiguity, shapes),
allocate the outputs and the backward workspace with torch, and call the
library on the current CUDA stream.  No arithmetic of the method happens
here.
"""

import math

import torch

from . import _lib

_DTYPES = {torch.bfloat16: _lib.FA_BF16, torch.float16: _lib.FA_FP16}


def _stream_handle(device):
    return ctypes_void(torch.cuda.current_stream(device).cuda_stream)


def ctypes_void(x):
    return x if x else None


def _check_inputs(tensors, shape, dtype, device):
    for name, t in tensors.items():
        if t is None:
            raise ValueError(f"{name} is None")
        if not t.is_cuda or t.device != device:
            raise ValueError(f"{name} must be a CUDA tensor on {device}")
        if t.dtype != dtype:
            raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, N, d]")


def _on_device(name, t, device):
    """Refuse a side tensor that lives on another accelerator: its pointer
    would be read by the kernel as if it were memory of ``device``.  Host
    tensors and lists are copied to ``device`` by the callers."""
    if torch.is_tensor(t) and t.device.type != "cpu" and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device} (or a host tensor)")


def _seqlens_arg(seqlens, B, device):
    if seqlens is None:
        return None, None
    _on_device("seqlens", seqlens, device)
    sl = seqlens
    if not (torch.is_tensor(sl) and sl.is_cuda and sl.dtype == torch.int32 and sl.is_contiguous()):
        sl = torch.as_tensor(seqlens, dtype=torch.int32).to(device).contiguous()
    if sl.shape != (B,):
        raise ValueError(f"seqlens must have shape ({B},)")
    return sl, sl.data_ptr()


def forward(q, k, v, scale=None, causal=False, seqlens=None, out=None, lse=None):
    """O, LSE = attention(q, k, v) on the GPU ([B, H, N, d] bf16/fp16)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = q.shape
    dev = q.device
    if q.dtype not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float16")
    _check_inputs({"q": q, "k": k, "v": v}, (B, H, N, d), q.dtype, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    _check_inputs({"out": out}, (B, H, N, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (B, H, N), torch.float32, dev)
    sl, sl_ptr = _seqlens_arg(seqlens, B, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                         B, H, N, d, scale, int(bool(causal)), sl_ptr, _DTYPES[q.dtype],
                         _stream_handle(dev))
    _lib.check("fa_fwd", st)
    return out, lse


def workspace_bytes(B, H, N, d):
    return _lib.fa_bwd_workspace_size(B, H, N, d)


def backward(q, k, v, o, lse, do, scale=None, causal=False, seqlens=None, workspace=None,
             dq=None, dk=None, dv=None):
    """dQ, dK, dV of the loss <dO, O> on the GPU."""
    B, H, N, d = q.shape
    dev = q.device
    _check_inputs({"q": q, "k": k, "v": v, "o": o, "do": do}, (B, H, N, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (B, H, N), torch.float32, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_inputs({"dq": dq, "dk": dk, "dv": dv}, (B, H, N, d), q.dtype, dev)
    need = workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    sl, sl_ptr = _seqlens_arg(seqlens, B, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                         lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                         workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                         B, H, N, d, scale, int(bool(causal)), sl_ptr, _DTYPES[q.dtype],
                         _stream_handle(dev))
    _lib.check("fa_bwd", st)
    return dq, dk, dv


def forward_dropout(q, k, v, p_drop, seed, offset=0, scale=None, causal=False, seqlens=None,
                    out=None, lse=None):
    """O, LSE of attention with dropout on the probabilities ([B, H, N, d];
    the keep mask is a function of seed, offset and the score's position)."""
    B, H, N, d = q.shape
    dev = q.device
    if q.dtype not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float16")
    _check_inputs({"q": q, "k": k, "v": v}, (B, H, N, d), q.dtype, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    _check_inputs({"out": out}, (B, H, N, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (B, H, N), torch.float32, dev)
    sl, sl_ptr = _seqlens_arg(seqlens, B, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), B, H, N, d, scale, int(bool(causal)), sl_ptr,
                                 float(p_drop), int(seed), int(offset), _DTYPES[q.dtype],
                                 _stream_handle(dev))
    _lib.check("fa_fwd_dropout", st)
    return out, lse


def backward_dropout(q, k, v, o, lse, do, p_drop, seed, offset=0, scale=None, causal=False,
                     seqlens=None, workspace=None, dq=None, dk=None, dv=None):
    """dQ, dK, dV for the same dropout mask as forward_dropout (same p_drop,
    seed and offset)."""
    B, H, N, d = q.shape
    dev = q.device
    _check_inputs({"q": q, "k": k, "v": v, "o": o, "do": do}, (B, H, N, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (B, H, N), torch.float32, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_inputs({"dq": dq, "dk": dk, "dv": dv}, (B, H, N, d), q.dtype, dev)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    sl, sl_ptr = _seqlens_arg(seqlens, B, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                 dv.data_ptr(), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), B, H, N, d, scale,
                                 int(bool(causal)), sl_ptr, float(p_drop), int(seed), int(offset),
                                 _DTYPES[q.dtype], _stream_handle(dev))
    _lib.check("fa_bwd_dropout", st)
    return dq, dk, dv


def _block_mask_arg(block_mask, N, device):
    nt = (N + 127) // 128
    _on_device("block_mask", block_mask, device)
    bm = block_mask
    if not (torch.is_tensor(bm) and bm.is_cuda and bm.dtype == torch.uint8 and bm.is_contiguous()):
        bm = torch.as_tensor(block_mask).to(device=device, dtype=torch.uint8).contiguous()
    if tuple(bm.shape) != (nt, nt):
        raise ValueError(f"block_mask must be [{nt}, {nt}] (128 x 128 tiles)")
    return bm


def forward_blocksparse(q, k, v, block_mask, scale=None, causal=False, seqlens=None, out=None,
                        lse=None):
    """O, LSE of block-sparse attention ([B, H, N, d]; block_mask [nt, nt] over
    128 x 128 score tiles, shared by all (batch, head) slices)."""
    B, H, N, d = q.shape
    dev = q.device
    if q.dtype not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float16")
    _check_inputs({"q": q, "k": k, "v": v}, (B, H, N, d), q.dtype, dev)
    bm = _block_mask_arg(block_mask, N, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    _check_inputs({"out": out}, (B, H, N, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (B, H, N), torch.float32, dev)
    sl, sl_ptr = _seqlens_arg(seqlens, B, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     lse.data_ptr(), bm.data_ptr(), B, H, N, d, scale,
                                     int(bool(causal)), sl_ptr, _DTYPES[q.dtype],
                                     _stream_handle(dev))
    _lib.check("fa_fwd_blocksparse", st)
    return out, lse


def backward_blocksparse(q, k, v, o, lse, do, block_mask, scale=None, causal=False, seqlens=None,
                         workspace=None, dq=None, dk=None, dv=None):
    """dQ, dK, dV of block-sparse attention for the loss <dO, O>."""
    B, H, N, d = q.shape
    dev = q.device
    _check_inputs({"q": q, "k": k, "v": v, "o": o, "do": do}, (B, H, N, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (B, H, N), torch.float32, dev)
    bm = _block_mask_arg(block_mask, N, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_inputs({"dq": dq, "dk": dk, "dv": dv}, (B, H, N, d), q.dtype, dev)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    sl, sl_ptr = _seqlens_arg(seqlens, B, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_bwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                     dv.data_ptr(), workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(), bm.data_ptr(),
                                     B, H, N, d, scale, int(bool(causal)), sl_ptr,
                                     _DTYPES[q.dtype], _stream_handle(dev))
    _lib.check("fa_bwd_blocksparse", st)
    return dq, dk, dv


def _cu_seqlens_arg(cu_seqlens, T, device):
    _on_device("cu_seqlens", cu_seqlens, device)
    cu = cu_seqlens
    if not (torch.is_tensor(cu) and cu.is_cuda and cu.dtype == torch.int32 and cu.is_contiguous()):
        cu = torch.as_tensor(cu_seqlens, dtype=torch.int32).to(device).contiguous()
    if cu.dim() != 1 or cu.numel() < 2:
        raise ValueError("cu_seqlens must be [B + 1] row offsets")
    return cu, cu.numel() - 1


def forward_varlen(q, k, v, cu_seqlens, max_seqlen, scale=None, causal=False, out=None, lse=None):
    """O, LSE of packed sequences on the GPU: q, k, v [H, T, d] bf16/fp16,
    sequence b in rows cu_seqlens[b] .. cu_seqlens[b + 1] - 1 of every head."""
    if q.dim() != 3:
        raise ValueError("q must be [H, T, d]")
    H, T, d = q.shape
    dev = q.device
    if q.dtype not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float16")
    _check_inputs({"q": q, "k": k, "v": v}, (H, T, d), q.dtype, dev)
    cu, B = _cu_seqlens_arg(cu_seqlens, T, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((H, T), dtype=torch.float32, device=dev) if lse is None else lse
    _check_inputs({"out": out}, (H, T, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (H, T), torch.float32, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), cu.data_ptr(), B, H, T, int(max_seqlen), d, scale,
                                int(bool(causal)), _DTYPES[q.dtype], _stream_handle(dev))
    _lib.check("fa_fwd_varlen", st)
    return out, lse


def backward_varlen(q, k, v, o, lse, do, cu_seqlens, max_seqlen, scale=None, causal=False,
                    workspace=None, dq=None, dk=None, dv=None):
    """dQ, dK, dV of the loss <dO, O> for packed sequences ([H, T, d])."""
    H, T, d = q.shape
    dev = q.device
    _check_inputs({"q": q, "k": k, "v": v, "o": o, "do": do}, (H, T, d), q.dtype, dev)
    _check_inputs({"lse": lse}, (H, T), torch.float32, dev)
    cu, B = _cu_seqlens_arg(cu_seqlens, T, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_inputs({"dq": dq, "dk": dk, "dv": dv}, (H, T, d), q.dtype, dev)
    if workspace is None:
        workspace = torch.empty(_lib.fa_bwd_varlen_workspace_size(B, H, T, d), dtype=torch.uint8,
                                device=dev)
    with torch.cuda.device(dev):
        st = _lib.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                dv.data_ptr(), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), cu.data_ptr(), B, H,
                                T, int(max_seqlen), d, scale, int(bool(causal)), _DTYPES[q.dtype],
                                _stream_handle(dev))
    _lib.check("fa_bwd_varlen", st)
    return dq, dk, dv


_E4M3 = (torch.float8_e4m3fn, torch.uint8)


def quantize_e4m3(x, out=None, descale=None):
    """Per-tile e4m3 quantisation of x [B, H, N, d] bf16/fp16 on the GPU.

    Returns (x8 [B, H, N, d] float8_e4m3fn, descale [B, H, ceil(N / 128)]
    float32): tile t of a slice (rows 128 t ..) stands for x8 * descale[t].
    """
    if x.dim() != 4:
        raise ValueError("x must be [B, H, N, d]")
    B, H, N, d = x.shape
    dev = x.device
    if x.dtype not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float16")
    _check_inputs({"x": x}, (B, H, N, d), x.dtype, dev)
    nt = (N + 127) // 128
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float8_e4m3fn, device=dev)
    if descale is None:
        descale = torch.empty((B, H, nt), dtype=torch.float32, device=dev)
    if out.dtype not in _E4M3:
        raise ValueError(f"out has dtype {out.dtype}, expected float8_e4m3fn or uint8")
    _check_inputs({"out": out}, (B, H, N, d), out.dtype, dev)
    _check_inputs({"descale": descale}, (B, H, nt), torch.float32, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_quantize_e4m3(x.data_ptr(), out.data_ptr(), descale.data_ptr(), B, H, N, d,
                                   _DTYPES[x.dtype], _stream_handle(dev))
    _lib.check("fa_quantize_e4m3", st)
    return out, descale


def forward_e4m3(q8, k8, v8, q_descale, k_descale, v_descale, scale=None, causal=False,
                 seqlens=None, out_dtype=torch.bfloat16, out=None, lse=None):
    """O, LSE of attention on e4m3 inputs ([B, H, N, d] float8_e4m3fn or
    uint8 codes, d in {64, 128}, descales [B, H, ceil(N / 128)] float32); O
    in out_dtype."""
    if q8.dim() != 4:
        raise ValueError("q8 must be [B, H, N, d]")
    B, H, N, d = q8.shape
    dev = q8.device
    if q8.dtype not in _E4M3:
        raise ValueError("q8 must be float8_e4m3fn or uint8 codes")
    if out_dtype not in _DTYPES:
        raise ValueError("out_dtype must be bfloat16 or float16")
    _check_inputs({"q8": q8, "k8": k8, "v8": v8}, (B, H, N, d), q8.dtype, dev)
    nt = (N + 127) // 128
    _check_inputs({"q_descale": q_descale, "k_descale": k_descale, "v_descale": v_descale},
                  (B, H, nt), torch.float32, dev)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    _check_inputs({"out": out}, (B, H, N, d), out_dtype, dev)
    _check_inputs({"lse": lse}, (B, H, N), torch.float32, dev)
    sl, sl_ptr = _seqlens_arg(seqlens, B, dev)
    with torch.cuda.device(dev):
        st = _lib.fa_fwd_e4m3(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_descale.data_ptr(),
                              k_descale.data_ptr(), v_descale.data_ptr(), out.data_ptr(),
                              lse.data_ptr(), B, H, N, d, scale, int(bool(causal)), sl_ptr,
                              _DTYPES[out_dtype], _stream_handle(dev))
    _lib.check("fa_fwd_e4m3", st)
    return out, lse


def device_status(device=None):
    """Synchronise and return (status, raw word) of the device status word."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return _lib.fa_device_status(_stream_handle(dev))
