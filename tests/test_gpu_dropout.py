"""Dropout on the probabilities: CUDA path (fa_fwd_dropout / fa_bwd_dropout
through the C ABI) vs the float64 oracle with the same Philox4x32-10 mask."""

import numpy as np
import pytest
import torch

from helpers import assert_fwd_close, assert_grad_close, f64, sample_rows
from oracle import keep_mask, keep_threshold, ref_bwd_dropout_slice, ref_fwd_dropout_slice

pytestmark = pytest.mark.gpu

SEED = 0x0123456789ABCDEF


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def _run(fa, inp, causal, scale, p, seed=SEED, offset=3):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    sl = inp["seqlens"]
    o, lse = fa.forward_dropout(q, k, v, p, seed, offset, scale=scale, causal=causal, seqlens=sl)
    dq, dk, dv = fa.backward_dropout(q, k, v, o, lse, do, p, seed, offset, scale=scale,
                                     causal=causal, seqlens=sl)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    return dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,p", [(300, 0.25), (515, 0.5)])
def test_against_oracle_full(fa, N, p, causal, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    B, H = 2, 2
    inp = make_inputs_shape(B, H, N, d, torch.bfloat16, seed=N + d + 5)
    scale = d ** -0.5
    r = _run(fa, inp, causal, scale, p)
    g = {n: f64(r[n]) for n in r}
    refs = {}
    for b in range(B):
        for h in range(H):
            bh = b * H + h
            args = (g["q"][b, h], g["k"][b, h], g["v"][b, h])
            ro, rl = ref_fwd_dropout_slice(*args, scale, causal, p, SEED, 3, bh)
            assert_fwd_close(g["o"][b, h], g["lse"][b, h], ro, rl, f"dropout b{b} h{h}")
            refs[b, h] = ref_bwd_dropout_slice(*args, g["do"][b, h], scale, causal, p, SEED, 3, bh)
    typical = [max(np.abs(x[n]).max() for x in refs.values()) for n in range(3)]
    for (b, h), ref in refs.items():
        for n, name in enumerate(("dq", "dk", "dv")):
            assert_grad_close(g[name][b, h], ref[n], f"dropout {name} b{b} h{h}",
                              typical=typical[n], floor_frac=5e-2)


def test_forward_mask_is_the_oracle_mask_bit_for_bit(fa):
    """Q = 0 makes P uniform (1/128 exactly) and V = I makes O = P * Z * 256/t:
    O[i, j] != 0 exactly where the oracle keeps score (i, j)."""
    B, H, N, d, p = 2, 3, 128, 128, 0.3
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    v = torch.eye(N, dtype=torch.bfloat16, device="cuda").expand(B, H, N, d).contiguous()
    for offset in (0, 9):
        o, _ = fa.forward_dropout(q, q, v, p, SEED, offset)
        t, keep = keep_threshold(p)
        for b in range(B):
            for h in range(H):
                z = keep_mask(b * H + h, np.arange(N), N, SEED, offset, p)
                got = o[b, h].float().cpu().numpy()
                assert np.array_equal(got != 0, z), (offset, b, h)
                np.testing.assert_allclose(got[z], 1 / 128 / keep, rtol=4e-3)


def test_backward_mask_is_the_oracle_mask_bit_for_bit(fa):
    """With P uniform and dO = I, dV = (P * Z)^T dO * 256/t = Z^T / 128 * 256/t:
    the backward regenerates the same mask from (seed, offset, position)."""
    B, H, N, d, p = 1, 2, 128, 128, 0.45
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    v = torch.randn((B, H, N, d), device="cuda").to(torch.bfloat16)
    do = torch.eye(N, dtype=torch.bfloat16, device="cuda").expand(B, H, N, d).contiguous()
    o, lse = fa.forward_dropout(q, q, v, p, SEED, 5)
    dq, dk, dv = fa.backward_dropout(q, q, v, o, lse, do, p, SEED, 5)
    for h in range(H):
        z = keep_mask(h, np.arange(N), N, SEED, 5, p)
        assert np.array_equal(dv[0, h].float().cpu().numpy().T != 0, z), h


def test_keep_fraction_and_seeds(fa):
    B, H, N, d, p = 1, 4, 512, 64, 0.2
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    v = torch.ones((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    t, keep = keep_threshold(p)
    o1, _ = fa.forward_dropout(q, q, v, p, 1)
    o2, _ = fa.forward_dropout(q, q, v, p, 2)
    # row means of the kept fraction scaled back: E[O] = 1 (unbiased); the
    # spread over 2048 rows of 512 Bernoulli draws each
    m = o1.float().mean().item()
    assert abs(m - 1.0) < 6 * np.sqrt((1 - keep) / keep / (H * N * N)) + 1e-2
    assert not torch.equal(o1, o2)


def test_rate_below_the_resolution_runs_the_plain_kernels(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(1, 2, 333, 128, torch.bfloat16, seed=8)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = fa.forward_dropout(q, k, v, 0.0, SEED, causal=True)
    o2, l2 = fa.forward(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_key_padding_fp16_sampled_long(fa):
    """B2 H4 N2048 d128 fp16 with key lengths, p = 0.1: sampled rows."""
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(2, 4, 2048, 128, torch.float16, seed=9, seqlens=[2048, 1500],
                            device="cuda")
    scale, p = 128 ** -0.5, 0.1
    r = _run(fa, inp, False, scale, p, offset=77)
    for b, h in ((0, 0), (1, 3)):
        L = [2048, 1500][b]
        q, k, v, do = (f64(r[n][b, h]) for n in ("q", "k", "v", "do"))
        rows = sample_rows(2048, n_random=40, seed=b + h)
        ro, rl = ref_fwd_dropout_slice(q, k, v, scale, False, p, SEED, 77, b * 4 + h, L, rows=rows)
        assert_fwd_close(f64(r["o"][b, h])[rows], f64(r["lse"][b, h])[rows], ro, rl, f"long b{b}")
        gq, gk, gv = ref_bwd_dropout_slice(q, k, v, do, scale, False, p, SEED, 77, b * 4 + h, L)
        for name, ref in (("dq", gq), ("dk", gk), ("dv", gv)):
            assert_grad_close(f64(r[name][b, h])[rows], ref[rows], f"long {name} b{b}")


def test_host_side_rejections(fa):
    from exact_io_aware_47_b200 import _lib
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 128), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for p in (-0.1, 1.0, float("nan")):
        st = _lib.fa_fwd_dropout(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(),
                                 lse.data_ptr(), 1, 1, 128, 64, 0.125, 0, None, p, 1, 0,
                                 _lib.FA_BF16, s)
        assert st == _lib.FA_ERR_INVALID_ARG, p
