"""Block-sparse attention: CUDA path (fa_fwd_blocksparse / fa_bwd_blocksparse
through the C ABI) vs the float64 oracle with the same 128 x 128 tile mask."""

import numpy as np
import pytest
import torch

from helpers import assert_fwd_close, assert_grad_close, f64, sample_rows
from oracle import ref_bwd_slice, ref_fwd_slice

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def _mask(nt, density, seed, empty_row=None, empty_col=None):
    m = np.random.default_rng(seed).random((nt, nt)) < density
    if empty_row is not None:
        m[empty_row, :] = False
    if empty_col is not None:
        m[:, empty_col] = False
    return m


def _run(fa, inp, mask, causal, scale):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    sl = inp["seqlens"]
    bm = torch.from_numpy(mask.astype(np.uint8))
    o, lse = fa.forward_blocksparse(q, k, v, bm, scale=scale, causal=causal, seqlens=sl)
    dq, dk, dv = fa.backward_blocksparse(q, k, v, o, lse, do, bm, scale=scale, causal=causal,
                                         seqlens=sl)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    return dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def _check_full(fa, inp, mask, causal, scale, what):
    r = _run(fa, inp, mask, causal, scale)
    B, H, N, d = r["q"].shape
    sl = inp["seqlens"]
    g = {n: f64(r[n]) for n in r}
    refs = {}
    for b in range(B):
        L = N if sl is None else int(sl[b])
        for h in range(H):
            ro, rl = ref_fwd_slice(g["q"][b, h], g["k"][b, h], g["v"][b, h], scale, causal, L,
                                   block_mask=mask)
            empty = np.isneginf(rl)
            assert np.array_equal(np.isneginf(g["lse"][b, h]), empty), f"{what}: empty rows"
            assert np.all(g["o"][b, h][empty] == 0.0)
            assert_fwd_close(g["o"][b, h][~empty], g["lse"][b, h][~empty], ro[~empty], rl[~empty],
                             f"{what} b{b} h{h}")
            refs[b, h] = ref_bwd_slice(g["q"][b, h], g["k"][b, h], g["v"][b, h], g["do"][b, h],
                                       scale, causal, L, block_mask=mask)
    typical = [max(np.abs(x[n]).max() for x in refs.values()) for n in range(3)]
    for (b, h), ref in refs.items():
        for n, name in enumerate(("dq", "dk", "dv")):
            assert_grad_close(g[name][b, h], ref[n], f"{what} {name} b{b} h{h}",
                              typical=typical[n], floor_frac=5e-2)
    return r


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 515])
def test_random_masks_full(fa, N, causal, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    nt = (N + 127) // 128
    inp = make_inputs_shape(2, 2, N, d, torch.bfloat16, seed=N + d)
    mask = _mask(nt, 0.55, seed=N * 7 + d + int(causal))
    mask[0, 0] = True
    _check_full(fa, inp, mask, causal, d ** -0.5, f"sparse N{N} d{d} causal{causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_empty_tile_rows_and_columns(fa, causal):
    """A query tile with no allowed key tile: O = 0, LSE = -inf, dQ = 0; a key
    tile no query tile sees: dK = dV = 0."""
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    N, d = 640, 128
    inp = make_inputs_shape(1, 2, N, d, torch.bfloat16, seed=33)
    mask = _mask(5, 0.7, seed=34)
    mask[np.arange(5), np.arange(5)] = True
    mask[2, :] = False   # query tile 2 sees nothing
    mask[:, 3] = False   # key tile 3 is seen by nobody
    r = _check_full(fa, inp, mask, causal, d ** -0.5, f"sparse empty causal{causal}")
    assert torch.all(r["o"][:, :, 256:384] == 0) and torch.all(torch.isneginf(r["lse"][:, :, 256:384]))
    assert torch.all(r["dq"][:, :, 256:384] == 0)
    assert torch.all(r["dk"][:, :, 384:512] == 0) and torch.all(r["dv"][:, :, 384:512] == 0)


def test_key_padding_and_fp16(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    N, d = 600, 64
    inp = make_inputs_shape(3, 2, N, d, torch.float16, seed=35, seqlens=[600, 200, 1])
    mask = _mask(5, 0.6, seed=36)
    mask[:, 0] = True
    _check_full(fa, inp, mask, False, 0.3, "sparse seqlens fp16")


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_equals_dense_kernels(fa, causal):
    """With every tile allowed the sparse kernels run the dense arithmetic:
    O, LSE, dK, dV bit for bit (dQ is reduced in arbitrary order)."""
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    N, d = 777, 128
    inp = make_inputs_shape(2, 2, N, d, torch.bfloat16, seed=37)
    nt = (N + 127) // 128
    r = _run(fa, inp, np.ones((nt, nt), bool), causal, d ** -0.5)
    o, lse = fa.forward(r["q"], r["k"], r["v"], causal=causal)
    dq, dk, dv = fa.backward(r["q"], r["k"], r["v"], o, lse, r["do"], causal=causal)
    assert torch.equal(o, r["o"]) and torch.equal(lse, r["lse"])
    assert torch.equal(dk, r["dk"]) and torch.equal(dv, r["dv"])
    assert (dq.float() - r["dq"].float()).abs().max().item() <= 1e-2 * dq.float().abs().max().item()


def test_sliding_window_long_sampled(fa):
    """B1 H8 N8192 d128 bf16 causal with a 4-tile sliding window plus the first
    (global) key tile: sampled rows and keys against the oracle."""
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    N, d, H = 8192, 128, 8
    nt = N // 128
    i, j = np.meshgrid(np.arange(nt), np.arange(nt), indexing="ij")
    mask = ((i - j >= 0) & (i - j < 4)) | (j == 0)
    inp = make_inputs_shape(1, H, N, d, torch.bfloat16, seed=38, device="cuda")
    r = _run(fa, inp, mask, True, d ** -0.5)
    for h in (0, H - 1):
        q, k, v, do = (f64(r[n][0, h]) for n in ("q", "k", "v", "do"))
        rows = sample_rows(N, n_random=48, seed=h)
        ro, rl = ref_fwd_slice(q, k, v, d ** -0.5, True, rows=rows, row_block=512, block_mask=mask)
        assert_fwd_close(f64(r["o"][0, h])[rows], f64(r["lse"][0, h])[rows], ro, rl, f"window h{h}")
        kr = sample_rows(N, n_random=48, seed=h + 9)
        gq, gk, gv = ref_bwd_slice(q, k, v, do, d ** -0.5, True, q_rows=rows, k_rows=kr,
                                   row_block=1024, block_mask=mask)
        assert_grad_close(f64(r["dq"][0, h])[rows], gq, f"window dQ h{h}")
        assert_grad_close(f64(r["dk"][0, h])[kr], gk, f"window dK h{h}")
        assert_grad_close(f64(r["dv"][0, h])[kr], gv, f"window dV h{h}")


def test_host_side_rejections(fa):
    from exact_io_aware_47_b200 import _lib
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 128), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    st = _lib.fa_fwd_blocksparse(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), None, 1, 1, 128, 64, 0.125, 0, None, _lib.FA_BF16, s)
    assert st == _lib.FA_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        fa.forward_blocksparse(q, q, q, torch.ones((2, 2), dtype=torch.uint8))
