"""The C ABI library builds, loads and exports what include/fa.h declares;
host-side argument checks answer without a GPU (no compute calls here)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_47_b200 import _lib, build
    build.build()
    return _lib.load()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(fa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for want in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_device_status",
                 "fa_status_string", "fa_version"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol():
    from exact_io_aware_47_b200 import _lib
    assert set(_declared_functions()) == set(_lib.SIGNATURES)


def test_status_strings_and_version(lib):
    for code in range(0, 12):
        s = lib.fa_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.fa_version() == 100


def test_workspace_size(lib):
    B, H, N, d = 2, 3, 1000, 128
    rows = B * H * N
    r256 = lambda x: (x + 255) // 256 * 256
    assert lib.fa_bwd_workspace_size(B, H, N, d) == r256(rows * 4) + r256(rows * d * 4)
    assert lib.fa_bwd_workspace_size(B, H, N, 96) == 0
    assert lib.fa_bwd_workspace_size(0, H, N, d) == 0


def test_rejections_before_any_cuda_call(lib):
    from exact_io_aware_47_b200 import _lib
    P = 1 << 20  # never dereferenced: every case below fails validation first
    ok = dict(B=1, H=2, N=128, d=64, scale=0.125, causal=1, seqlens=None, dtype=0)

    def fwd(q=P, o=P, **kw):
        a = {**ok, **kw}
        return lib.fa_fwd(q, P, P, o, P, a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"],
                          a["seqlens"], a["dtype"], None)
    assert fwd(q=None) == _lib.FA_ERR_INVALID_ARG
    assert fwd(B=0) == _lib.FA_ERR_INVALID_ARG
    assert fwd(N=-3) == _lib.FA_ERR_INVALID_ARG
    assert fwd(scale=0.0) == _lib.FA_ERR_INVALID_ARG
    assert fwd(scale=float("inf")) == _lib.FA_ERR_INVALID_ARG
    assert fwd(dtype=2) == _lib.FA_ERR_INVALID_ARG
    assert fwd(d=32) == _lib.FA_ERR_UNSUPPORTED
    assert fwd(B=1 << 12, H=1 << 10, N=1 << 10, d=64) == _lib.FA_ERR_UNSUPPORTED
    assert fwd(q=P + 8) == _lib.FA_ERR_ALIGNMENT
    assert fwd(seqlens=P + 2) == _lib.FA_ERR_ALIGNMENT

    ws = lib.fa_bwd_workspace_size(1, 2, 128, 64)

    def bwd(wsp=P, wsb=ws, **kw):
        a = {**ok, **kw}
        return lib.fa_bwd(P, P, P, P, P, P, P, P, P, wsp, wsb, a["B"], a["H"], a["N"], a["d"],
                          a["scale"], a["causal"], a["seqlens"], a["dtype"], None)
    assert bwd(wsp=None) == _lib.FA_ERR_WORKSPACE
    assert bwd(wsb=ws - 1) == _lib.FA_ERR_WORKSPACE
    assert bwd(wsp=P + 16) == _lib.FA_ERR_ALIGNMENT
    assert bwd(d=100) == _lib.FA_ERR_UNSUPPORTED
    assert bwd(H=0) == _lib.FA_ERR_INVALID_ARG


def test_varlen_workspace_size(lib):
    """The packed backward's workspace: the dense one for [H, T, d], then the
    longest-first table (3 B + 1 ints, 256-byte padded) for B <= 4096."""
    H, T, d = 3, 1000, 64
    base = lib.fa_bwd_workspace_size(1, H, T, d)
    assert lib.fa_bwd_varlen_workspace_size(1, H, T, d) == base + 256
    assert lib.fa_bwd_varlen_workspace_size(100, H, T, d) == base + (301 * 4 + 255) // 256 * 256
    assert lib.fa_bwd_varlen_workspace_size(5000, H, T, d) == base
    assert lib.fa_bwd_varlen_workspace_size(0, H, T, d) == 0
    assert lib.fa_bwd_varlen_workspace_size(2, H, T, 96) == 0


def test_noalloc_size_limit_checked_on_the_host(lib):
    from exact_io_aware_47_b200 import _lib
    P = 1 << 20
    assert lib.fa_bwd_noalloc_max_bytes() == 32 << 20
    st = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 4, 32, 8192, 128, 0.088, 1, None, 0, None)
    assert st == _lib.FA_ERR_SCRATCH_LIMIT
    st = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 1, 1, 128, 96, 0.088, 1, None, 0, None)
    assert st == _lib.FA_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(tmp_path):
    from exact_io_aware_47_b200 import _lib
    with pytest.raises(RuntimeError, match="missing"):
        _lib.load(str(tmp_path / "nope.so"))


def test_e4m3_rejections_before_any_cuda_call(lib):
    from exact_io_aware_47_b200 import _lib
    P = 1 << 20  # never dereferenced: every case below fails validation first
    ok = dict(B=1, H=2, N=128, d=128, scale=0.125, dtype=0)

    def fwd8(q=P, ds=P, o=P, **kw):
        a = {**ok, **kw}
        return lib.fa_fwd_e4m3(q, P, P, ds, ds, ds, o, P, a["B"], a["H"], a["N"], a["d"],
                               a["scale"], 1, None, a["dtype"], None)
    assert fwd8(q=None) == _lib.FA_ERR_INVALID_ARG
    assert fwd8(ds=None) == _lib.FA_ERR_INVALID_ARG
    assert fwd8(B=0) == _lib.FA_ERR_INVALID_ARG
    assert fwd8(scale=-1.0) == _lib.FA_ERR_INVALID_ARG
    assert fwd8(dtype=5) == _lib.FA_ERR_INVALID_ARG
    assert fwd8(d=96) == _lib.FA_ERR_UNSUPPORTED                # 8-bit path: d in {64, 128}
    assert fwd8(ds=P + 2) == _lib.FA_ERR_ALIGNMENT              # descales: 4-byte aligned
    assert fwd8(q=P + 8) == _lib.FA_ERR_ALIGNMENT               # codes: 16-byte aligned
    assert fwd8(o=P + 4) == _lib.FA_ERR_ALIGNMENT

    def quant(x=P, x8=P, ds=P, **kw):
        a = {**ok, **kw}
        return lib.fa_quantize_e4m3(x, x8, ds, a["B"], a["H"], a["N"], a["d"], a["dtype"], None)
    assert quant(x=None) == _lib.FA_ERR_INVALID_ARG
    assert quant(N=0) == _lib.FA_ERR_INVALID_ARG
    assert quant(dtype=3) == _lib.FA_ERR_INVALID_ARG
    assert quant(d=80) == _lib.FA_ERR_UNSUPPORTED
    assert quant(x8=P + 8) == _lib.FA_ERR_ALIGNMENT
    assert quant(ds=P + 1) == _lib.FA_ERR_ALIGNMENT
    assert lib.fa_status_string(_lib.FA_ERR_DEVICE_SCALE) != b"unknown status"


def test_side_tensors_on_another_device_are_refused():
    """seqlens, block_mask and cu_seqlens are passed to the kernels as raw
    pointers, so one that lives on another device must be refused on the host
    (a meta tensor stands in for "another device": no GPU needed)."""
    import torch
    from exact_io_aware_47_b200 import attention as A
    dev = torch.device("cuda", 0)
    other = torch.device("meta")
    with pytest.raises(ValueError, match="seqlens"):
        A._seqlens_arg(torch.ones(2, dtype=torch.int32, device=other), 2, dev)
    with pytest.raises(ValueError, match="block_mask"):
        A._block_mask_arg(torch.ones((1, 1), dtype=torch.uint8, device=other), 128, dev)
    with pytest.raises(ValueError, match="cu_seqlens"):
        A._cu_seqlens_arg(torch.zeros(3, dtype=torch.int32, device=other), 10, dev)


def test_wait_limit_setting_is_host_state(lib):
    """fa_set_wait_limit_ns returns the previous bound; 0 restores the 2 s
    default (no GPU needed: the bound is passed to later launches)."""
    lib.fa_set_wait_limit_ns.restype = ctypes.c_ulonglong
    lib.fa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    first = lib.fa_set_wait_limit_ns(12345)
    assert first == 2_000_000_000
    assert lib.fa_set_wait_limit_ns(0) == 12345
    assert lib.fa_set_wait_limit_ns(0) == 2_000_000_000
