"""Backward parity: CUDA kernels (through the C ABI) vs the float64 oracle."""

import numpy as np
import pytest
import torch

from helpers import assert_grad_close, f64, sample_rows, subset_slices
from oracle import ref_bwd_slice

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def _run(fa, inp, causal, scale):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    sl = inp["seqlens"]
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal, seqlens=sl)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, scale=scale, causal=causal, seqlens=sl)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    return q, k, v, do, dq, dk, dv


def _check_full(fa, inp, causal, scale, what):
    q, k, v, do, dq, dk, dv = _run(fa, inp, causal, scale)
    B, H, N, d = q.shape
    sl = inp["seqlens"]
    refs = {}
    for b in range(B):
        L = N if sl is None else int(sl[b])
        for h in range(H):
            # kept in float32 (the tolerances are 5e-2 relative): the ragged
            # workload's 128 slices would take 1.6 GB of float64
            refs[b, h] = [g.astype(np.float32) for g in ref_bwd_slice(
                f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), f64(do[b, h]), scale, causal, L)]
    typical = [max(np.abs(g[n]).max() for g in refs.values()) for n in range(3)]
    for b in range(B):
        L = N if sl is None else int(sl[b])
        for h in range(H):
            for n, (name, got) in enumerate(zip(("dQ", "dK", "dV"), (dq, dk, dv))):
                assert_grad_close(f64(got[b, h]), refs[b, h][n], f"{what} {name} b{b} h{h}",
                                  typical=typical[n])
            # padded keys: exactly zero
            assert torch.all(dk[b, h, L:] == 0) and torch.all(dv[b, h, L:] == 0)


def _check_sampled(fa, inp, causal, scale, slices, what, n_random=48):
    q, k, v, do, dq, dk, dv = _run(fa, inp, causal, scale)
    N = q.shape[2]
    sl = inp["seqlens"]
    for (b, h) in slices:
        L = N if sl is None else int(sl[b])
        qr = sample_rows(N, n_random=n_random, seed=b * 100 + h)
        kr = sample_rows(N, n_random=n_random, seed=b * 100 + h + 7)
        g = ref_bwd_slice(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), f64(do[b, h]), scale, causal,
                          L, q_rows=qr, k_rows=kr, row_block=1024)
        assert_grad_close(f64(dq[b, h])[qr], g[0], f"{what} dQ b{b} h{h}")
        assert_grad_close(f64(dk[b, h])[kr], g[1], f"{what} dK b{b} h{h}")
        assert_grad_close(f64(dv[b, h])[kr], g[2], f"{what} dV b{b} h{h}")
        assert torch.all(dk[b, h, L:] == 0) and torch.all(dv[b, h, L:] == 0)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_tiny_fp32_draws(fa, dtype):
    from exact_io_aware_47_b200.inputs import make_inputs
    _check_full(fa, make_inputs("tiny", dtype=dtype), False, 1 / 8, f"tiny {dtype}")


def test_small_training_shape_causal(fa):
    from exact_io_aware_47_b200.inputs import make_inputs
    _check_full(fa, make_inputs("small"), True, 1 / 8, "small")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 257, 515])
def test_edge_lengths(fa, N, causal, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(2, 2, N, d, torch.bfloat16, seed=N + d + 1)
    _check_full(fa, inp, causal, d ** -0.5, f"N{N} d{d} causal{causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,lens", [(300, [1, 127, 128, 129]), (256, [256, 1, 255, 130])])
def test_edge_seqlens(fa, N, lens, causal, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(len(lens), 2, N, d, torch.bfloat16, seed=3 * N + d, seqlens=lens)
    _check_full(fa, inp, causal, d ** -0.5, f"N{N} lens{lens} d{d} causal{causal}")


def test_fp16_and_scale(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(1, 2, 700, 128, torch.float16, seed=4)
    _check_full(fa, inp, True, 0.3, "fp16 scale0.3")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_mid_context_sampled(fa, dtype):
    from exact_io_aware_47_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["mid"]
    inp = make_inputs("mid", dtype=dtype, device="cuda")
    _check_sampled(fa, inp, True, w.scale, subset_slices(w.B, w.H), f"mid {dtype}")


def test_long_context_sampled(fa):
    from exact_io_aware_47_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["long"]
    inp = make_inputs("long", device="cuda")
    _check_sampled(fa, inp, True, w.scale, subset_slices(w.B, w.H), "long", n_random=24)


def test_ragged_padded_batch_every_slice(fa):
    """B8 H16 N4099 d128 with key padding: dQ, dK and dV of every (batch,
    head) slice, every row, against the oracle; padded keys exactly zero."""
    from exact_io_aware_47_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["ragged"]
    _check_full(fa, make_inputs("ragged", device="cuda"), False, w.scale, "ragged")


def test_workspace_contents_do_not_matter_and_guards_hold(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    B, H, N, d = 2, 2, 333, 128
    inp = make_inputs_shape(B, H, N, d, torch.bfloat16, seed=12)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, causal=True)
    ref = fa.backward(q, k, v, o, lse, do, causal=True)
    n = B * H * N * d
    bufs = [torch.full((n + 2048,), 5.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    ws = torch.full((fa.workspace_bytes(B, H, N, d) // 4,), float("nan"), device="cuda")
    got = fa.backward(q, k, v, o, lse, do, causal=True, workspace=ws.view(torch.uint8),
                      dq=bufs[0][:n].view(B, H, N, d), dk=bufs[1][:n].view(B, H, N, d),
                      dv=bufs[2][:n].view(B, H, N, d))
    torch.cuda.synchronize()
    for bb in bufs:
        assert torch.all(bb[n:] == 5.0)
    for a, b in zip(ref, got):
        assert torch.isfinite(b).all()
        assert (a.float() - b.float()).abs().max().item() <= 1e-2 * a.float().abs().max().item()


def test_dk_dv_deterministic(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(1, 4, 900, 64, torch.bfloat16, seed=13)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, causal=True)
    g1 = fa.backward(q, k, v, o, lse, do, causal=True)
    g2 = fa.backward(q, k, v, o, lse, do, causal=True)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])


def test_workspace_too_small_is_refused(fa):
    from exact_io_aware_47_b200 import _lib
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(1, 1, 128, 64, torch.bfloat16, seed=1)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v)
    ws = torch.empty(fa.workspace_bytes(1, 1, 128, 64) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.FAError) as e:
        fa.backward(q, k, v, o, lse, do, workspace=ws)
    assert e.value.status == _lib.FA_ERR_WORKSPACE
