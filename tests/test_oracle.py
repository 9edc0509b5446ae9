"""Pins for the CPU float64 oracle (no GPU).

Each test checks the oracle against something other than itself: a worked
example derived by hand, a closed form, an invariant of the definition, or
central finite differences of the forward oracle.
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import (ref_bwd, ref_bwd_slice, ref_fwd, ref_fwd_slice,
                    tiled_fwd_slice)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ev(x):
    return float(eval(str(x), {"__builtins__": {}}, {"log": math.log}))


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --- worked example derived by hand -------------------------------------------------

@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "two_key_hand.json")))["cases"],
                         ids=lambda c: c["name"])
def test_two_key_hand_example(case):
    g = json.load(open(os.path.join(GOLDEN, "two_key_hand.json")))["inputs"]
    q = np.array([[_ev(x) for x in r] for r in g["q"]])
    k = np.array([[_ev(x) for x in r] for r in g["k"]])
    v = np.array([[_ev(x) for x in r] for r in g["v"]])
    do = np.array([[_ev(x) for x in r] for r in g["do"]])
    o, lse = ref_fwd_slice(q, k, v, g["scale"], case["causal"], case["valid_len"])
    np.testing.assert_allclose(o, [[_ev(x) for x in r] for r in case["O"]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, [_ev(x) for x in case["LSE"]], rtol=0, atol=1e-14)
    dq, dk, dv = ref_bwd_slice(q, k, v, do, g["scale"], case["causal"], case["valid_len"])
    np.testing.assert_allclose(dq, [[_ev(x) for x in r] for r in case["dQ"]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk, [[_ev(x) for x in r] for r in case["dK"]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv, [[_ev(x) for x in r] for r in case["dV"]], rtol=0, atol=1e-14)


# --- closed forms ------------------------------------------------------------------

@pytest.mark.parametrize("L", [1, 5, 13])
def test_zero_query_gives_mean_of_valid_values(L):
    n, d = 13, 6
    k, v = _rand((n, d), 1), _rand((n, d), 2)
    o, lse = ref_fwd_slice(np.zeros((n, d)), k, v, 0.3, False, L)
    np.testing.assert_allclose(o, np.broadcast_to(v[:L].mean(axis=0), (n, d)), atol=1e-14)
    np.testing.assert_allclose(lse, np.full(n, math.log(L)), atol=1e-14)


def test_zero_query_causal_gives_prefix_mean():
    n, d = 11, 5
    k, v = _rand((n, d), 3), _rand((n, d), 4)
    o, lse = ref_fwd_slice(np.zeros((n, d)), k, v, 0.7, True)
    want = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
    np.testing.assert_allclose(o, want, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.arange(1, n + 1)), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_single_valid_key_returns_its_value(causal):
    n, d = 9, 4
    q, k, v = _rand((n, d), 5), _rand((n, d), 6), _rand((n, d), 7)
    o, lse = ref_fwd_slice(q, k, v, 0.5, causal, valid_len=1)
    np.testing.assert_allclose(o, np.broadcast_to(v[0], (n, d)), atol=1e-14)
    np.testing.assert_allclose(lse, 0.5 * (q @ k[0]), atol=1e-14)


def test_causal_row_zero_is_first_value():
    n, d = 10, 8
    q, k, v = _rand((n, d), 8), _rand((n, d), 9), _rand((n, d), 10)
    o, lse = ref_fwd_slice(q, k, v, 0.25, True)
    np.testing.assert_allclose(o[0], v[0], atol=1e-14)
    np.testing.assert_allclose(lse[0], 0.25 * q[0] @ k[0], atol=1e-14)


def test_causal_row_one_two_key_closed_form():
    # row 1 sees keys 0 and 1: o = sigma(s0 - s1) v0 + sigma(s1 - s0) v1
    n, d = 4, 3
    q, k, v = _rand((n, d), 11), _rand((n, d), 12), _rand((n, d), 13)
    sc = 0.9
    o, lse = ref_fwd_slice(q, k, v, sc, True)
    s0, s1 = sc * q[1] @ k[0], sc * q[1] @ k[1]
    sig = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(o[1], sig * v[0] + (1 - sig) * v[1], atol=1e-14)
    np.testing.assert_allclose(lse[1], s0 + math.log1p(math.exp(s1 - s0)), atol=1e-14)


def test_constant_values_give_constant_output():
    # rows of P sum to one, so V = c for every key gives O = c
    n, d = 12, 5
    q, k = _rand((n, d), 14), _rand((n, d), 15)
    v = np.tile(np.arange(1.0, d + 1.0), (n, 1))
    for causal in (False, True):
        o, _ = ref_fwd_slice(q, k, v, 0.4, causal, 7)
        np.testing.assert_allclose(o, v, atol=1e-13)


def test_dominant_key_limit():
    # as the scale grows, softmax tends to the argmax of each row
    n, d = 8, 4
    q, k, v = _rand((n, d), 16), _rand((n, d), 17), _rand((n, d), 18)
    o, _ = ref_fwd_slice(q, k, v, 1e4, False)
    np.testing.assert_allclose(o, v[np.argmax(q @ k.T, axis=1)], atol=1e-12)


def test_lse_bounds():
    n, d = 16, 8
    q, k, v = _rand((n, d), 19), _rand((n, d), 20), _rand((n, d), 21)
    sc = 0.35
    _, lse = ref_fwd_slice(q, k, v, sc, True)
    s = sc * q @ k.T
    for i in range(n):
        mx = s[i, :i + 1].max()
        assert mx - 1e-14 <= lse[i] <= mx + math.log(i + 1) + 1e-14


# --- invariants --------------------------------------------------------------------

def test_permutation_invariance_non_causal():
    n, d, L = 15, 6, 11
    q, k, v = _rand((n, d), 22), _rand((n, d), 23), _rand((n, d), 24)
    perm = np.concatenate([np.random.default_rng(25).permutation(L), np.arange(L, n)])
    o1, l1 = ref_fwd_slice(q, k, v, 0.6, False, L)
    o2, l2 = ref_fwd_slice(q, k[perm], v[perm], 0.6, False, L)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_query_permutation_equivariance_non_causal():
    n, d = 9, 3
    q, k, v = _rand((n, d), 26), _rand((n, d), 27), _rand((n, d), 28)
    perm = np.random.default_rng(29).permutation(n)
    o1, l1 = ref_fwd_slice(q, k, v, 0.6, False)
    o2, l2 = ref_fwd_slice(q[perm], k, v, 0.6, False)
    np.testing.assert_allclose(o1[perm], o2, atol=1e-13)
    np.testing.assert_allclose(l1[perm], l2, atol=1e-13)


def test_row_subsets_and_blocks_match_full():
    n, d = 37, 5
    q, k, v, do = (_rand((n, d), s) for s in (30, 31, 32, 33))
    o, lse = ref_fwd_slice(q, k, v, 0.5, True, 30)
    rows = np.array([0, 5, 17, 36])
    o2, lse2 = ref_fwd_slice(q, k, v, 0.5, True, 30, rows=rows, row_block=3)
    np.testing.assert_allclose(o2, o[rows], atol=1e-14)
    np.testing.assert_allclose(lse2, lse[rows], atol=1e-14)
    dq, dk, dv = ref_bwd_slice(q, k, v, do, 0.5, True, 30)
    kr = np.array([1, 29, 30, 35])
    dq2, dk2, dv2 = ref_bwd_slice(q, k, v, do, 0.5, True, 30, q_rows=rows, k_rows=kr,
                                  row_block=4)
    np.testing.assert_allclose(dq2, dq[rows], atol=1e-13)
    np.testing.assert_allclose(dk2, dk[kr], atol=1e-13)
    np.testing.assert_allclose(dv2, dv[kr], atol=1e-13)


def test_batched_matches_slices():
    B, H, n, d = 2, 3, 7, 4
    q, k, v, do = (_rand((B, H, n, d), s) for s in (34, 35, 36, 37))
    sl = np.array([3, 7])
    o, lse = ref_fwd(q, k, v, 0.5, False, sl)
    dq, dk, dv = ref_bwd(q, k, v, do, 0.5, False, sl)
    for b in range(B):
        for h in range(H):
            o1, l1 = ref_fwd_slice(q[b, h], k[b, h], v[b, h], 0.5, False, int(sl[b]))
            np.testing.assert_allclose(o[b, h], o1, atol=0)
            np.testing.assert_allclose(lse[b, h], l1, atol=0)
            g = ref_bwd_slice(q[b, h], k[b, h], v[b, h], do[b, h], 0.5, False, int(sl[b]))
            for a, c in zip((dq[b, h], dk[b, h], dv[b, h]), g):
                np.testing.assert_allclose(a, c, atol=0)


# --- backward -------------------------------------------------------------------

def _loss(q, k, v, do, sc, causal, L):
    o, _ = ref_fwd_slice(q, k, v, sc, causal, L)
    return float((o * do).sum())


@pytest.mark.parametrize("causal,L", [(False, None), (True, None), (False, 5), (True, 6)])
def test_backward_matches_central_differences(causal, L):
    B, H, n, d = 1, 2, 8, 4
    sc = 0.45
    for h in range(H):
        q, k, v, do = (_rand((n, d), 100 * h + s) for s in (1, 2, 3, 4))
        dq, dk, dv = ref_bwd_slice(q, k, v, do, sc, causal, L)
        eps = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += eps
                xm[idx] -= eps
                args = {"q": q, "k": k, "v": v}
                args[name] = xp
                lp = _loss(args["q"], args["k"], args["v"], do, sc, causal, L)
                args[name] = xm
                lm = _loss(args["q"], args["k"], args["v"], do, sc, causal, L)
                num[idx] = (lp - lm) / (2 * eps)
            err = np.abs(num - g).max() / max(np.abs(num).max(), 1e-30)
            assert err < 1e-6, (name, err)


def test_padded_keys_get_exactly_zero_gradients():
    n, d, L = 12, 5, 7
    q, k, v, do = (_rand((n, d), s) for s in (40, 41, 42, 43))
    for causal in (False, True):
        _, dk, dv = ref_bwd_slice(q, k, v, do, 0.5, causal, L)
        assert np.all(dk[L:] == 0.0) and np.all(dv[L:] == 0.0)


def test_gradient_sum_identities():
    # softmax rows sum to one: sum_j dS_ij = 0 => sum_j dK_j = 0, sum_j dV_j = sum_i dO_i
    n, d = 14, 6
    q, k, v, do = (_rand((n, d), s) for s in (44, 45, 46, 47))
    for causal, L in ((False, None), (True, None), (False, 9)):
        _, dk, dv = ref_bwd_slice(q, k, v, do, 0.5, causal, L)
        np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
        np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)


def test_dq_zero_when_values_constant():
    # V constant over keys: O does not depend on P, so dQ = dK = 0
    n, d = 10, 4
    q, k, do = _rand((n, d), 48), _rand((n, d), 49), _rand((n, d), 50)
    v = np.tile(_rand((1, d), 51), (n, 1))
    dq, dk, _ = ref_bwd_slice(q, k, v, do, 0.7, True, None)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dk, 0.0, atol=1e-13)


# --- the online-softmax tile recurrence equals the definition ------------------------

@pytest.mark.parametrize("block_n", [1, 2, 3, 7])
@pytest.mark.parametrize("block_m", [1, 4, 5])
@pytest.mark.parametrize("tau", [0.0, 8.0, math.inf])
def test_online_model_equals_definition(block_m, block_n, tau):
    n, d = 19, 5
    q, k, v = _rand((n, d), 60), _rand((n, d), 61), _rand((n, d), 62)
    for causal, L in ((False, None), (True, None), (False, 11), (True, 4)):
        o, lse = ref_fwd_slice(q, k, v, 0.8, causal, L)
        o2, lse2 = tiled_fwd_slice(q, k, v, 0.8, causal, L, block_m, block_n, tau)
        np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)


def test_online_model_growing_max_lazy_rescale():
    # keys grow along the sequence, so the running max keeps rising across tiles
    n, d = 64, 8
    rng = np.random.default_rng(63)
    q = rng.standard_normal((n, d)) * 3.0
    k = rng.standard_normal((n, d)) * (1 + 3 * np.arange(n) / n)[:, None] * 3.0
    v = rng.standard_normal((n, d))
    for tau in (0.0, 8.0):
        o, lse = ref_fwd_slice(q, k, v, 1.0, False, 50)
        o2, lse2 = tiled_fwd_slice(q, k, v, 1.0, False, 50, 16, 8, tau)
        np.testing.assert_allclose(o2, o, rtol=0, atol=1e-11)
        np.testing.assert_allclose(lse2, lse, rtol=1e-13, atol=1e-11)


# --- block-sparse masks ------------------------------------------------------------

def _blocks(n, b):
    return [slice(i, min(i + b, n)) for i in range(0, n, b)]


@pytest.mark.parametrize("causal", [False, True])
def test_block_diagonal_mask_is_independent_blocks(causal):
    """Query block i may only see key block i: every block is then an attention
    problem of its own, computed here by the dense oracle on the slices."""
    n, d, b = 10, 3, 4
    q, k, v, do = (_rand((n, d), s) for s in (60, 61, 62, 63))
    nb = -(-n // b)
    mask = np.eye(nb, dtype=bool)
    o, lse = ref_fwd_slice(q, k, v, 0.6, causal, block_mask=mask, block=b)
    dq, dk, dv = ref_bwd_slice(q, k, v, do, 0.6, causal, block_mask=mask, block=b)
    for sl in _blocks(n, b):
        ro, rl = ref_fwd_slice(q[sl], k[sl], v[sl], 0.6, causal)
        gq, gk, gv = ref_bwd_slice(q[sl], k[sl], v[sl], do[sl], 0.6, causal)
        np.testing.assert_allclose(o[sl], ro, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[sl], rl, rtol=0, atol=1e-13)
        for a, r in ((dq, gq), (dk, gk), (dv, gv)):
            np.testing.assert_allclose(a[sl], r, rtol=0, atol=1e-12)


def test_off_diagonal_mask_is_not_transposed():
    """Mask [[0, 1], [1, 0]]: query block 0 sees only key block 1 and query
    block 1 only key block 0 (a transposed mask would give the same here only
    if it were symmetric; [[0, 1], [0, 0]] below is not)."""
    n, d, b = 8, 3, 4
    q, k, v = (_rand((n, d), s) for s in (64, 65, 66))
    o, lse = ref_fwd_slice(q, k, v, 0.7, False, block_mask=np.array([[0, 1], [0, 0]], bool), block=b)
    ro, rl = ref_fwd_slice(q[:4], k[4:], v[4:], 0.7, False)
    np.testing.assert_allclose(o[:4], ro, atol=1e-13)
    np.testing.assert_allclose(lse[:4], rl, atol=1e-13)
    assert np.all(o[4:] == 0.0) and np.all(np.isneginf(lse[4:]))


def test_fully_masked_rows_are_zero_and_drop_out_of_key_gradients():
    """Query block 1 may see no key block: its rows give O = 0, LSE = -inf and
    dQ = 0, and dK, dV equal those of the other query rows alone."""
    n, d, b = 12, 4, 4
    q, k, v, do = (_rand((n, d), s) for s in (67, 68, 69, 70))
    mask = np.array([[1, 0, 1], [0, 0, 0], [1, 1, 1]], bool)
    o, lse = ref_fwd_slice(q, k, v, 0.5, False, block_mask=mask, block=b)
    dq, dk, dv = ref_bwd_slice(q, k, v, do, 0.5, False, block_mask=mask, block=b)
    assert np.all(o[4:8] == 0.0) and np.all(np.isneginf(lse[4:8])) and np.all(dq[4:8] == 0.0)
    keep = np.r_[0:4, 8:12]          # query blocks 0 and 2, in blocks of 4 rows
    gq, gk, gv = ref_bwd_slice(q[keep], k, v, do[keep], 0.5, False, valid_len=n,
                               block_mask=mask[[0, 2]], block=b, k_rows=np.arange(n))
    np.testing.assert_allclose(dk, gk, atol=1e-12)
    np.testing.assert_allclose(dv, gv, atol=1e-12)
    np.testing.assert_allclose(dq[keep], gq, atol=1e-12)


def test_key_block_permutation_invariance():
    """Non-causal: permuting whole key blocks (K, V rows) together with the
    mask's columns leaves the output unchanged."""
    n, d, b = 12, 3, 4
    q, k, v = (_rand((n, d), s) for s in (71, 72, 73))
    mask = np.array([[1, 0, 1], [0, 1, 1], [1, 1, 0]], bool)
    perm = [2, 0, 1]
    rows = np.concatenate([np.arange(p * b, p * b + b) for p in perm])
    o1, l1 = ref_fwd_slice(q, k, v, 0.8, False, block_mask=mask, block=b)
    o2, l2 = ref_fwd_slice(q, k[rows], v[rows], 0.8, False, block_mask=mask[:, perm], block=b)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_backward_matches_central_differences(causal):
    n, d, b, sc = 9, 3, 3, 0.5
    mask = np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]], bool)
    q, k, v, do = (_rand((n, d), s) for s in (74, 75, 76, 77))
    dq, dk, dv = ref_bwd_slice(q, k, v, do, sc, causal, block_mask=mask, block=b)

    def loss(qq, kk, vv):
        o, _ = ref_fwd_slice(qq, kk, vv, sc, causal, block_mask=mask, block=b)
        return float((o * do).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][idx] += eps
            lp = loss(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * eps
            lm = loss(args["q"], args["k"], args["v"])
            num[idx] = (lp - lm) / (2 * eps)
        assert np.abs(num - g).max() / max(np.abs(num).max(), 1e-30) < 1e-6, name


# --- dropout on the probabilities --------------------------------------------------

from oracle.dropout import (keep_mask, keep_threshold, philox4x32_10, ref_bwd_dropout_slice,
                            ref_fwd_dropout_slice)


@pytest.mark.parametrize("ctr,key,expect", [
    ((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff,) * 4, (0xffffffff,) * 2, (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
])
def test_philox_known_answers(ctr, key, expect):
    """Known-answer vectors of Philox4x32-10 distributed with the generator's
    reference implementation (Random123, by the authors of the SC 2011 paper)."""
    out = philox4x32_10(*ctr, *key)
    assert tuple(int(x) for x in out) == expect


def test_dropout_zero_rate_is_plain_attention():
    n, d = 9, 4
    q, k, v, do = (_rand((n, d), s) for s in (80, 81, 82, 83))
    for causal in (False, True):
        o, lse = ref_fwd_dropout_slice(q, k, v, 0.5, causal, 0.0, seed=5, offset=0, bh=0)
        ro, rl = ref_fwd_slice(q, k, v, 0.5, causal)
        np.testing.assert_allclose(o, ro, atol=1e-14)
        np.testing.assert_allclose(lse, rl, atol=1e-14)
        g = ref_bwd_dropout_slice(q, k, v, do, 0.5, causal, 0.0, 5, 0, 0)
        r = ref_bwd_slice(q, k, v, do, 0.5, causal)
        for a, b in zip(g, r):
            np.testing.assert_allclose(a, b, atol=1e-13)


def test_keep_fraction_and_threshold():
    assert keep_threshold(0.0) == (256, 1.0)
    assert keep_threshold(0.25) == (192, 0.75)
    assert keep_threshold(0.999)[0] == 1
    m = keep_mask(3, np.arange(512), 512, seed=123456789, offset=7, p_drop=0.3)
    t, keep = keep_threshold(0.3)
    frac = m.mean()
    # 262144 Bernoulli(keep) draws: 6 standard deviations
    assert abs(frac - keep) < 6 * np.sqrt(keep * (1 - keep) / m.size)
    # different seeds, offsets and slices give different masks
    m2 = keep_mask(3, np.arange(64), 64, seed=123456790, offset=7, p_drop=0.3)
    m3 = keep_mask(3, np.arange(64), 64, seed=123456789, offset=8, p_drop=0.3)
    m4 = keep_mask(4, np.arange(64), 64, seed=123456789, offset=7, p_drop=0.3)
    for other in (m2, m3, m4):
        assert (other != m[:64, :64]).mean() > 0.2


def test_mask_rows_are_independent_of_the_row_set():
    full = keep_mask(1, np.arange(40), 37, seed=99, offset=1, p_drop=0.5)
    rows = np.array([0, 3, 4, 17, 39])
    np.testing.assert_array_equal(keep_mask(1, rows, 37, seed=99, offset=1, p_drop=0.5), full[rows])


def test_dropout_is_unbiased_over_seeds():
    """E_Z[O] = plain attention: averaged over many independent masks the
    dropout output approaches the undropped one (1/sqrt(#seeds) rate)."""
    n, d = 8, 3
    q, k, v = (_rand((n, d), s) for s in (84, 85, 86))
    ro, _ = ref_fwd_slice(q, k, v, 0.7, False)
    acc = np.zeros_like(ro)
    S = 4000
    for s in range(S):
        o, _ = ref_fwd_dropout_slice(q, k, v, 0.7, False, 0.5, seed=1000 + s, offset=0, bh=0)
        acc += o
    err = np.abs(acc / S - ro).max()
    assert err < 6 * np.abs(v).max() / np.sqrt(S), err


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_backward_matches_central_differences(causal):
    n, d, sc, p = 10, 3, 0.6, 0.4
    q, k, v, do = (_rand((n, d), s) for s in (87, 88, 89, 90))
    dq, dk, dv = ref_bwd_dropout_slice(q, k, v, do, sc, causal, p, 77, 3, 2)

    def loss(qq, kk, vv):
        o, _ = ref_fwd_dropout_slice(qq, kk, vv, sc, causal, p, 77, 3, 2)
        return float((o * do).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][idx] += eps
            lp = loss(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * eps
            lm = loss(args["q"], args["k"], args["v"])
            num[idx] = (lp - lm) / (2 * eps)
        assert np.abs(num - g).max() / max(np.abs(num).max(), 1e-30) < 1e-6, name
