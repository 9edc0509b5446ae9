"""8-bit (e4m3) path on the GPU (fa_quantize_e4m3, fa_fwd_e4m3 through the C
ABI) against the oracle.

* The quantiser decides its integer codes in fp32 on both sides, so codes and
  descales must be identical, bit for bit.
* The forward runs on codes the oracle produced and is compared with plain
  softmax attention (oracle.attention, the definition) of the dequantised
  inputs code x descale.  The one step of the 8-bit path that the definition
  does not have is the rounding of the probabilities to e4m3 before the
  product with V ("How Flash Attention Works", section "FlashAttention 2 and
  3": lower-precision paths); oracle.fp8.fp8_error_bound bounds what that
  rounding can change, element by element, from the format's precision alone.
  So every O element must lie within the dense tolerance (2e-2) plus that
  bound, the mean error within 2e-3 plus the mean bound, and LSE, which the
  rounding does not touch, within the dense 1e-3.  No fraction of elements is
  exempt.
"""

import numpy as np
import pytest
import torch

from helpers import LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, f64, sample_rows
from oracle import ref_fwd_slice
from oracle.fp8 import dequantize_tiles, fp8_error_bound, quantize_tiles

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def _oracle_quantize(x):
    """x [B, H, N, d] 16-bit torch -> (codes uint8 [B, H, N, d], descale [B, H, nt])."""
    B, H, N, d = x.shape
    xs = x.float().cpu().numpy()
    nt = (N + 127) // 128
    codes = np.zeros((B, H, N, d), dtype=np.uint8)
    ds = np.zeros((B, H, nt), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            codes[b, h], ds[b, h] = quantize_tiles(xs[b, h])
    return codes, ds


def _check_against_definition(o, lse, q8, k8, v8, sq, sk, sv, scale, causal, valid, rows, what):
    """o, lse: the GPU's rows ``rows`` of one slice; the rest: that slice's
    codes and descales.  Plain attention of the dequantised inputs, and the
    element-wise bound of the 8-bit rounding of P."""
    qd, kd, vd = (dequantize_tiles(c, s) for c, s in ((q8, sq), (k8, sk), (v8, sv)))
    ro, rl = ref_fwd_slice(qd, kd, vd, scale, causal, valid, rows=rows)
    bound = fp8_error_bound(q8, k8, v8, sq, sk, sv, scale, causal, valid, rows=rows)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), f"{what}: non-finite output"
    err = np.abs(o - ro)
    dl = np.abs(lse - rl).max()
    assert dl <= LSE_MAX_ABS, f"{what}: LSE max err {dl:.3e}"
    over = err > O_MAX_ABS + bound
    assert not over.any(), \
        f"{what}: {int(over.sum())} O elements beyond 2e-2 + bound (worst excess " \
        f"{(err - O_MAX_ABS - bound).max():.3e})"
    assert err.mean() <= O_MEAN_ABS + bound.mean(), \
        f"{what}: O mean err {err.mean():.3e} vs {O_MEAN_ABS + bound.mean():.3e}"
    return err.max(), err.mean(), bound.mean()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("d", [64, 128])
def test_quantizer_is_the_oracle_bit_for_bit(fa, dtype, d):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    B, H, N = 2, 3, 300                                        # ragged last tile
    x = make_inputs_shape(B, H, N, d, dtype, seed=d + 1)["q"]
    x[0, 1, 128:256] = 0                                       # a tile of zeros
    x[1, 2, :128] *= 1e-4                                      # small values: subnormal codes
    x[1, 0, 256:] *= 300                                       # large values
    x = x.to(dtype)
    x8, ds = fa.quantize_e4m3(x.cuda())
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    codes, rds = _oracle_quantize(x)
    assert np.array_equal(x8.view(torch.uint8).cpu().numpy(), codes)
    assert np.array_equal(ds.cpu().numpy(), rds)


def _fwd_case(fa, B, H, N, causal, seed, seqlens=None, out_dtype=torch.bfloat16, v_scales=None,
              d=128):
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(B, H, N, d, torch.bfloat16, seed=seed, seqlens=seqlens)
    v = inp["v"].float()
    if v_scales is not None:                                   # V tiles on different scales
        for t, f in enumerate(v_scales):
            v[:, :, t * 128:(t + 1) * 128] *= f
    qc, sq = _oracle_quantize(inp["q"])
    kc, sk = _oracle_quantize(inp["k"])
    vc, sv = _oracle_quantize(v.to(torch.bfloat16))
    dev = torch.device("cuda")
    t8 = lambda c: torch.from_numpy(c).to(dev).view(torch.float8_e4m3fn)
    td = lambda a: torch.from_numpy(a).to(dev)
    scale = d ** -0.5
    o, lse = fa.forward_e4m3(t8(qc), t8(kc), t8(vc), td(sq), td(sk), td(sv), scale=scale,
                             causal=causal, seqlens=inp["seqlens"], out_dtype=out_dtype)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    return (qc, kc, vc, sq, sk, sv), f64(o), f64(lse), scale


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 515])
def test_forward_against_oracle(fa, N, causal, d):
    """d = 64 runs the d = 128 kernel on zero-filled columns 64..127."""
    B, H = 2, 2
    (qc, kc, vc, sq, sk, sv), o, lse, scale = _fwd_case(fa, B, H, N, causal, seed=N + causal + d,
                                                        d=d)
    assert o.shape == (B, H, N, d)
    for b in range(B):
        for h in range(H):
            a = (qc[b, h], kc[b, h], vc[b, h], sq[b, h], sk[b, h], sv[b, h])
            _check_against_definition(o[b, h], lse[b, h], *a, scale, causal, N, np.arange(N),
                                      f"N{N} causal{causal} b{b} h{h}")


def test_forward_key_padding_fp16_out_and_v_tile_scales(fa):
    B, H, N = 2, 2, 450
    lens = [450, 200]
    (qc, kc, vc, sq, sk, sv), o, lse, scale = _fwd_case(
        fa, B, H, N, False, seed=4, seqlens=lens, out_dtype=torch.float16,
        v_scales=(1.0, 0.03, 6.0, 0.4))
    for b in range(B):
        for h in range(H):
            a = (qc[b, h], kc[b, h], vc[b, h], sq[b, h], sk[b, h], sv[b, h])
            _check_against_definition(o[b, h], lse[b, h], *a, scale, False, lens[b],
                                      np.arange(N), f"padded b{b} h{h}")


def test_full_size_causal_sampled(fa):
    """B2 H32 N8192 d128 causal, the product path end to end: bf16 inputs
    quantised on the GPU, then the 8-bit forward; sampled slices and rows."""
    from exact_io_aware_47_b200.inputs import make_inputs
    inp = make_inputs("mid", dtype=torch.bfloat16, seed=0, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    B, H, N, d = q.shape
    (q8, sq), (k8, sk), (v8, sv) = (fa.quantize_e4m3(t) for t in (q, k, v))
    scale = d ** -0.5
    o, lse = fa.forward_e4m3(q8, k8, v8, sq, sk, sv, scale=scale, causal=True)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    for b, h in ((0, 0), (1, H - 1)):
        oracle_in = []
        for t, c8, ds in ((q, q8, sq), (k, k8, sk), (v, v8, sv)):
            codes, rds = quantize_tiles(t[b, h].float().cpu().numpy())
            assert np.array_equal(c8[b, h].view(torch.uint8).cpu().numpy(), codes)
            assert np.array_equal(ds[b, h].cpu().numpy(), rds)
            oracle_in += [codes, rds]
        a = (oracle_in[0], oracle_in[2], oracle_in[4], oracle_in[1], oracle_in[3], oracle_in[5])
        rows = sample_rows(N, n_random=24, seed=b + h)
        _check_against_definition(f64(o[b, h])[rows], f64(lse[b, h])[rows], *a, scale, True, N,
                                  rows, f"full b{b} h{h}")


def test_rejections_and_device_scale_status(fa):
    from exact_io_aware_47_b200 import _lib
    s = torch.cuda.current_stream().cuda_stream
    q8 = torch.zeros((1, 1, 128, 128), dtype=torch.uint8, device="cuda")
    ds = torch.ones((1, 1, 1), dtype=torch.float32, device="cuda")
    o = torch.empty((1, 1, 128, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 128), dtype=torch.float32, device="cuda")
    args = lambda qp, dsp, d: (qp, qp, qp, dsp, dsp, dsp, o.data_ptr(), lse.data_ptr(), 1, 1, 128,
                               d, 0.1, 0, None, _lib.FA_BF16, s)
    q96 = torch.zeros((1, 1, 128, 96), dtype=torch.uint8, device="cuda")
    assert _lib.fa_fwd_e4m3(*args(q96.data_ptr(), ds.data_ptr(), 96)) == _lib.FA_ERR_UNSUPPORTED
    assert _lib.fa_fwd_e4m3(*args(q8.data_ptr(), ds.data_ptr() + 2, 128)) == _lib.FA_ERR_ALIGNMENT
    assert _lib.fa_fwd_e4m3(*args(q8.data_ptr(), None, 128)) == _lib.FA_ERR_INVALID_ARG
    bad = torch.full((1, 1, 1), -1.0, dtype=torch.float32, device="cuda")
    assert _lib.fa_fwd_e4m3(*args(q8.data_ptr(), bad.data_ptr(), 128)) == _lib.FA_OK
    st, _ = _lib.fa_device_status(s)
    assert st == _lib.FA_ERR_DEVICE_SCALE
    x = torch.ones((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    x[0, 0, 5, 7] = float("inf")
    fa.quantize_e4m3(x)
    st, _ = _lib.fa_device_status(s)
    assert st == _lib.FA_ERR_DEVICE_SCALE
    x[0, 0, 5, 7] = float("nan")                               # NaN is reported too
    fa.quantize_e4m3(x)
    st, _ = _lib.fa_device_status(s)
    assert st == _lib.FA_ERR_DEVICE_SCALE
    assert _lib.fa_device_status(s)[0] == _lib.FA_OK           # read and cleared
