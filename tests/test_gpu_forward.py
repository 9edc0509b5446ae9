"""Forward parity: CUDA kernel (through the C ABI) vs the float64 oracle."""

import numpy as np
import pytest
import torch

from helpers import assert_fwd_close, f64, sample_rows, subset_slices
from oracle import ref_fwd_slice

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def _check_full(fa, inp, causal, scale, what):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    sl = inp["seqlens"]
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal, seqlens=sl)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    B, H, N, d = q.shape
    q64, k64, v64 = f64(q), f64(k), f64(v)
    o64, l64 = f64(o), f64(lse)
    for b in range(B):
        L = N if sl is None else int(sl[b])
        for h in range(H):
            ro, rl = ref_fwd_slice(q64[b, h], k64[b, h], v64[b, h], scale, causal, L)
            assert_fwd_close(o64[b, h], l64[b, h], ro, rl, f"{what} b{b} h{h}")


def _check_sampled(fa, inp, causal, scale, slices, what, n_random=96):
    q, k, v = inp["q"], inp["k"], inp["v"]
    sl = inp["seqlens"]
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal, seqlens=sl)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    N = q.shape[2]
    for (b, h) in slices:
        L = N if sl is None else int(sl[b])
        rows = sample_rows(N, n_random=n_random, seed=b * 1000 + h)
        q64, k64, v64 = f64(q[b, h]), f64(k[b, h]), f64(v[b, h])
        ro, rl = ref_fwd_slice(q64, k64, v64, scale, causal, L, rows=rows, row_block=256)
        assert_fwd_close(f64(o[b, h])[rows], f64(lse[b, h])[rows], ro, rl, f"{what} b{b} h{h}")
    return o, lse


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_tiny_fp32_draws(fa, dtype):
    from exact_io_aware_47_b200.inputs import make_inputs
    inp = make_inputs("tiny", dtype=dtype)
    _check_full(fa, inp, False, 1 / 8, f"tiny {dtype}")


def test_small_training_shape_causal(fa):
    from exact_io_aware_47_b200.inputs import make_inputs
    inp = make_inputs("small")
    _check_full(fa, inp, True, 1 / 8, "small")


EDGE_N = [1, 2, 127, 128, 129, 255, 256, 257, 383, 515]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", EDGE_N)
def test_edge_lengths(fa, N, causal, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(2, 2, N, d, torch.bfloat16, seed=N + d)
    _check_full(fa, inp, causal, d ** -0.5, f"N{N} d{d} causal{causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,lens", [(300, [1, 127, 128, 129]), (256, [256, 1, 255, 130]),
                                    (129, [129, 128, 2, 1])])
def test_edge_seqlens(fa, N, lens, causal, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(len(lens), 2, N, d, torch.bfloat16, seed=7 * N + d, seqlens=lens)
    _check_full(fa, inp, causal, d ** -0.5, f"N{N} lens{lens} d{d} causal{causal}")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_edge_fp16_and_scale(fa, dtype):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(1, 3, 700, 128, dtype, seed=3)
    _check_full(fa, inp, True, 0.3, f"scale0.3 {dtype}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_mid_context_sampled(fa, dtype):
    from exact_io_aware_47_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["mid"]
    inp = make_inputs("mid", dtype=dtype, device="cuda", with_do=False)
    _check_sampled(fa, inp, True, w.scale, subset_slices(w.B, w.H), f"mid {dtype}")


def test_long_context_sampled_and_linear_memory(fa):
    from exact_io_aware_47_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["long"]
    inp = make_inputs("long", device="cuda", with_do=False)
    q, k, v = inp["q"], inp["k"], inp["v"]
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    fa.forward(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    extra = torch.cuda.max_memory_allocated() - base
    # one N x N fp16 score matrix of one head would be 2 GiB; the call allocates nothing
    assert extra < 64 * 2 ** 20, f"forward allocated {extra} bytes"
    inp2 = {"q": q, "k": k, "v": v, "seqlens": None}
    _check_sampled(fa, inp2, True, w.scale, subset_slices(w.B, w.H), "long", n_random=48)


def test_ragged_padded_batch_every_slice(fa):
    """B8 H16 N4099 d128, key padding, K growing along the sequence (the
    workload built to stress the rescale): every (batch, head) slice, every
    row, against the oracle."""
    from exact_io_aware_47_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["ragged"]
    inp = make_inputs("ragged", device="cuda", with_do=False)
    q, k, v, sl = inp["q"], inp["k"], inp["v"], inp["seqlens"]
    o, lse = fa.forward(q, k, v, scale=w.scale, causal=False, seqlens=sl)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    lens = sl.cpu().tolist()
    for b in range(w.B):
        for h in range(w.H):
            ro, rl = ref_fwd_slice(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), w.scale, False,
                                   lens[b])
            assert_fwd_close(f64(o[b, h]), f64(lse[b, h]), ro, rl, f"ragged b{b} h{h} L{lens[b]}")


def test_output_guard_regions_untouched(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    B, H, N, d = 2, 3, 333, 128
    inp = make_inputs_shape(B, H, N, d, torch.bfloat16, seed=11)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    n_o = B * H * N * d
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((B * H * N + 1024,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[:n_o].view(B, H, N, d)
    lse = l_buf[:B * H * N].view(B, H, N)
    fa.forward(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(o_buf[n_o:] == 7.0)
    assert torch.all(l_buf[B * H * N:] == 7.0)


def test_deterministic(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(2, 4, 1000, 128, torch.bfloat16, seed=5)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = fa.forward(q, k, v, causal=True)
    o2, l2 = fa.forward(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_seqlens_are_clamped_and_reported(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    N = 200
    inp = make_inputs_shape(2, 1, N, 64, torch.bfloat16, seed=9)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    sl = torch.tensor([0, N + 50], dtype=torch.int32, device="cuda")
    o, lse = fa.forward(q, k, v, causal=False, seqlens=sl)
    st, word = fa.device_status()
    assert st == 7 and (word & 0xff) == 7
    assert fa.device_status()[0] == 0  # cleared
    for b, L in ((0, 1), (1, N)):
        ro, rl = ref_fwd_slice(f64(q[b, 0]), f64(k[b, 0]), f64(v[b, 0]), 0.125, False, L)
        assert_fwd_close(f64(o[b, 0]), f64(lse[b, 0]), ro, rl, f"clamped b{b}")


def test_host_side_rejections(fa):
    from exact_io_aware_47_b200 import _lib
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    lse = torch.zeros(1, 1, 128, dtype=torch.float32, device="cuda")
    p = q.data_ptr()
    args = dict(B=1, H=1, N=128, d=64, scale=0.125, causal=0, seqlens=None, dtype=0, stream=None)

    def call(**kw):
        a = {**args, **kw}
        return _lib.fa_fwd(kw.get("q", p), p, p, o.data_ptr(), lse.data_ptr(), a["B"], a["H"], a["N"], a["d"],
                           a["scale"], a["causal"], a["seqlens"], a["dtype"], a["stream"])
    assert call(d=96) == _lib.FA_ERR_UNSUPPORTED
    assert call(N=0) == _lib.FA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == _lib.FA_ERR_INVALID_ARG
    assert call(q=p + 2) == _lib.FA_ERR_ALIGNMENT
    assert call(dtype=5) == _lib.FA_ERR_INVALID_ARG
    assert call() == _lib.FA_OK
    torch.cuda.synchronize()


# --- closed forms on the GPU: cases where rounding cannot hide an error ------------

def _bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (float64 array)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_single_visible_key_returns_its_value_exactly(fa, d, causal):
    # one visible key: P = 1 exactly after the max is subtracted, so O = v_0
    # with no rounding at all, and LSE = scale * q_i . k_0
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    N = 300
    inp = make_inputs_shape(2, 3, N, d, torch.bfloat16, seed=31 + d, seqlens=[1, 1])
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, causal=causal, seqlens=inp["seqlens"])
    assert torch.equal(o, v[:, :, :1, :].expand_as(o))
    s0 = (f64(q) * f64(k)[:, :, :1, :]).sum(-1) * d ** -0.5
    assert np.abs(f64(lse) - s0).max() <= 1e-4


@pytest.mark.parametrize("d", [64, 128])
def test_causal_row_zero_is_first_value_exactly(fa, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(2, 2, 777, d, torch.bfloat16, seed=41 + d)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, causal=True)
    assert torch.equal(o[:, :, 0], v[:, :, 0])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("L", [3, 128, 129, 1000])
def test_zero_query_gives_mean_within_one_ulp(fa, d, L):
    # uniform scores: every p = 1 exactly, O = fp32 mean of the valid V rows,
    # rounded once to bf16; LSE = ln L
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    N = 1000
    inp = make_inputs_shape(1, 2, N, d, torch.bfloat16, seed=L + d, seqlens=[L])
    k, v = inp["k"].cuda(), inp["v"].cuda()
    q = torch.zeros_like(k)
    o, lse = fa.forward(q, k, v, seqlens=inp["seqlens"])
    mean = f64(v)[:, :, :L].mean(axis=2, keepdims=True)
    err = np.abs(f64(o) - mean)
    assert (err <= _bf16_ulp(mean) * 0.5 + 1e-5 * np.abs(mean) + 1e-6).all(), err.max()
    assert np.abs(f64(lse) - np.log(L)).max() <= 1e-5 * max(1.0, np.log(L))
