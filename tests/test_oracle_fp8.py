"""Pins of the e4m3 oracle (oracle/fp8.py) to things other than itself.

* the format: every code decodes as torch's float8_e4m3fn does (a library
  routine), rounding matches torch's conversion inside the finite range, and
  hand-derived values from the format's definition (ties to even,
  subnormals, saturation);
* the quantiser: its extreme element lands on +-448, and dequantisation is
  within the format's relative precision;
* the attention: when every rounded probability is exactly representable it
  equals the plain softmax attention of the dequantised inputs (including a
  lazy rescale); in general it stays inside the derived element-wise bound,
  and its LSE is the exact one (l is taken before rounding).
"""

import math

import numpy as np
import pytest
import torch

from oracle import ref_fwd_slice
from oracle.fp8 import (E4M3_MAX, dequantize_tiles, e4m3_decode, e4m3_encode, e4m3_round,
                        fp8_error_bound, quantize_tiles, ref_fwd_fp8_slice)


def _torch_codes(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.tensor(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0x7E] == E4M3_MAX


def test_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(e4m3_encode(e4m3_decode(codes)), codes)


def test_rounding_matches_torch_inside_the_range():
    rng = np.random.default_rng(3)
    finite = np.sort(e4m3_decode(np.arange(0x7F, dtype=np.uint8)))   # 0 .. 448
    mids = (finite[1:] + finite[:-1]) / 2                            # exact ties
    x = np.concatenate([
        rng.standard_normal(20000) * 30,
        rng.standard_normal(5000) * 1e-2,                            # subnormal range
        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
    ]).astype(np.float32)
    x = x[np.abs(x) < 464]                                           # below the saturation tie
    assert np.array_equal(e4m3_encode(x.astype(np.float64)), _torch_codes(x))


@pytest.mark.parametrize("x,code", [
    (1.0, 0x38),                      # exponent 7 (bias 7), mantissa 0
    (448.0, 0x7E),                    # largest finite: 1.75 * 2^8
    (2.0 ** -9, 0x01),                # smallest subnormal
    (2.0 ** -6, 0x08),                # smallest normal
    (1.0625, 0x38),                   # tie between 1 and 1.125: even mantissa 0
    (1.1875, 0x3A),                   # tie between 1.125 and 1.25: even mantissa 2
    (-3.0, 0xC4),                     # 1.5 * 2^1, sign set
    (2.0 ** -10, 0x00),               # tie between 0 and 2^-9: even (zero)
    (3 * 2.0 ** -10, 0x02),           # tie between 2^-9 and 2^-8: even mantissa 2
    (460.0, 0x7E),                    # nearer to 448 than to the (absent) 480
    (500.0, 0x7E),                    # saturates
    (-1e6, 0xFE),
    (-0.0, 0x80),
])
def test_hand_derived_codes(x, code):
    assert int(e4m3_encode(np.array([x]))[0]) == code
    assert e4m3_round(np.array([x]))[0] == e4m3_decode(np.array([code], dtype=np.uint8))[0]


def test_quantize_tiles_extremes_and_precision():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((300, 64)) * 3).astype(np.float32)
    x[128:256] *= 1e-3                                   # a tile on another scale
    x[256:] = 0                                          # a ragged tile of zeros
    codes, ds = quantize_tiles(x)
    assert ds.shape == (3,) and ds.dtype == np.float32 and ds[2] == 1.0
    assert np.all(codes[256:] & 0x7F == 0)
    vals = e4m3_decode(codes)
    for t in range(2):
        blk = slice(t * 128, (t + 1) * 128)
        amax = np.abs(x[blk]).max()
        assert np.abs(vals[blk]).max() == E4M3_MAX       # the extreme maps to +-448
        assert abs(ds[t] * E4M3_MAX - amax) <= 2.0 ** -22 * amax
    deq = dequantize_tiles(codes, ds)
    tile_ds = np.repeat(ds.astype(np.float64), 128)[:300, None]
    # half a unit in the last place of e4m3, relative or subnormal, plus the
    # fp32 rounding of the scale
    err = np.abs(deq - x)
    assert np.all(err <= 2.0 ** -4 * np.abs(x) * (1 + 2 ** -20) + 2.0 ** -10 * tile_ds * 1.01)


def _exact_case(causal, sv=0.375, n=256, d=16, seed=0):
    """Codes whose scaled scores are integers in log2 units (softmax scale
    ln 2, sq * sk = 1 on tile 0 and 2 on tile 1): every probability, taken
    against any max the lazy recurrence holds, is a power of two between 2^-8
    and 2^0, so rounding it to e4m3 is exact.  Tile 0's scores lie in [0, 8],
    tile 1's are even numbers in [18, 26], so every row that sees tile 1 moves
    its max there (by at least 10 > 8)."""
    rng = np.random.default_rng(seed)
    onehot = rng.integers(0, d, size=n)
    q8 = np.zeros((n, d), dtype=np.uint8)
    q8[np.arange(n), onehot] = e4m3_encode(np.array([1.0]))[0]
    k_int = rng.integers(0, 9, size=(n, d)).astype(np.float64)
    k_int[128:] = rng.integers(9, 14, size=(n - 128, d))
    k8 = e4m3_encode(k_int)
    assert np.array_equal(e4m3_decode(k8), k_int)
    v8 = e4m3_encode(rng.standard_normal((n, d)) * 40)
    nt = (n + 127) // 128
    sq = np.full(nt, 2.0, dtype=np.float32)
    sk = np.array([0.5, 1.0], dtype=np.float32)[:nt]
    svv = np.full(nt, sv, dtype=np.float32)
    return q8, k8, v8, sq, sk, svv


@pytest.mark.parametrize("causal", [False, True])
def test_equals_plain_attention_when_rounding_is_exact(causal):
    q8, k8, v8, sq, sk, sv = _exact_case(causal)
    scale = math.log(2.0)
    o, lse = ref_fwd_fp8_slice(q8, k8, v8, sq, sk, sv, scale, causal)
    ro, rl = ref_fwd_slice(dequantize_tiles(q8, sq), dequantize_tiles(k8, sk),
                           dequantize_tiles(v8, sv), scale, causal)
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=1e-13, atol=1e-13)


def test_exact_case_does_move_the_max():
    # the construction must actually exercise the lazy rescale: in row 200,
    # tile 1's max exceeds tile 0's by more than 8 in log2 units
    q8, k8, _, sq, sk, _ = _exact_case(False)
    s = (e4m3_decode(q8)[200] * sq[1]) @ dequantize_tiles(k8, sk).T
    assert s[128:].max() - s[:128].max() > 8


def _random_case(n, d, seed, v_tile_scales=None):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    if v_tile_scales is not None:
        for t, f in enumerate(v_tile_scales):
            v[t * 128:(t + 1) * 128] *= f
    (q8, sq), (k8, sk), (v8, sv) = (quantize_tiles(a) for a in (q, k, v))
    return q8, k8, v8, sq, sk, sv


@pytest.mark.parametrize("n,causal,valid,vts", [
    (300, False, None, None),
    (300, True, None, None),
    (515, False, 400, None),
    (400, True, None, (1.0, 0.05, 7.0, 0.5)),   # V tiles on different scales
])
def test_within_the_derived_bound_of_exact_attention(n, causal, valid, vts):
    d = 64
    q8, k8, v8, sq, sk, sv = _random_case(n, d, seed=n + (7 if causal else 0), v_tile_scales=vts)
    scale = d ** -0.5
    o, lse = ref_fwd_fp8_slice(q8, k8, v8, sq, sk, sv, scale, causal, valid)
    ro, rl = ref_fwd_slice(dequantize_tiles(q8, sq), dequantize_tiles(k8, sk),
                           dequantize_tiles(v8, sv), scale, causal, valid)
    bound = fp8_error_bound(q8, k8, v8, sq, sk, sv, scale, causal, valid)
    err = np.abs(o - ro)
    assert np.all(err <= bound + 1e-12)
    assert err.max() > 0                                  # the rounding is real
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_rows_subset_matches_full():
    q8, k8, v8, sq, sk, sv = _random_case(333, 64, seed=11)
    o, lse = ref_fwd_fp8_slice(q8, k8, v8, sq, sk, sv, 0.125, True)
    rows = np.array([0, 5, 127, 128, 200, 332])
    o2, l2 = ref_fwd_fp8_slice(q8, k8, v8, sq, sk, sv, 0.125, True, rows=rows)
    np.testing.assert_allclose(o2, o[rows], rtol=1e-12, atol=1e-14)   # BLAS blocking only
    np.testing.assert_allclose(l2, lse[rows], rtol=1e-14, atol=0)


def test_planted_mistake_leaves_the_bound():
    """Dropping the V-descale ratio (rounding P instead of rho P) is the kind of
    slip the bound must catch when V tiles differ in scale."""
    n, d = 400, 64
    q8, k8, v8, sq, sk, sv = _random_case(n, d, seed=2, v_tile_scales=(1.0, 0.02, 9.0, 0.5))
    scale = d ** -0.5
    ro, _ = ref_fwd_slice(dequantize_tiles(q8, sq), dequantize_tiles(k8, sk),
                          dequantize_tiles(v8, sv), scale, False)
    bound = fp8_error_bound(q8, k8, v8, sq, sk, sv, scale, False)
    # wrong: every V tile dequantised with the largest descale
    wrong, _ = ref_fwd_fp8_slice(q8, k8, v8, sq, sk, np.full_like(sv, sv.max()), scale, False)
    assert np.any(np.abs(wrong - ro) > bound + 1e-12)
