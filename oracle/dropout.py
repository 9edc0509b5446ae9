"""Oracle for attention with dropout on the probabilities: plain, CPU, float64.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use
it.  It shares no code with the CUDA library.

What it computes ("How Flash Attention Works", swarnava.dev):

* section "Why Standard Attention Becomes a GPU Memory I/O Bottleneck": the
  standard pipeline computes Q K^T, applies the causal mask, runs the
  softmax, applies dropout, then multiplies by V;
* section "Kernel Fusion and Incremental Output Accumulation": dropout is one
  of the steps fused into the kernel, so its mask must be reproducible
  inside both passes rather than stored.

Readings (listed with their reasons in the design notes):

* dropout acts on the normalised probabilities: O = (P * M) V with
  M_ij = Z_ij / keep, Z_ij in {0, 1}; LSE is that of the scores, unchanged;
* Z comes from the counter-based generator Philox4x32-10 (Salmon, Moraes,
  Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011),
  written here from its published definition: one call maps a 128-bit
  counter and a 64-bit key to four 32-bit words;
* one call covers a 4 x 4 block of scores of one (batch, head) slice: the
  counter is (key block j // 4, query block i // 4, slice index b * H + h,
  offset), the key the 64-bit seed; word w of the result belongs to query
  row 4 (i // 4) + w, and its byte c (bits 8c .. 8c + 7) to key 4 (j // 4) + c;
* Z_ij = 1 iff that byte is below the 8-bit threshold t = round(256 (1 - p)),
  clamped to [1, 256]; keep = t / 256 is the exact keep probability used for
  the scale (p is represented to 1/256);
* gradients of <dO, O> by the chain rule: dV = (P * M)^T dO,
  dP = M * (dO V^T), D_i = sum_j P_ij dP_ij (= <dO_i, O_i>),
  dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q.
"""

import numpy as np

from .attention import _scores_probs

__all__ = ["philox4x32_10", "keep_threshold", "keep_mask", "ref_fwd_dropout_slice",
           "ref_bwd_dropout_slice"]

_M0, _M1 = 0xD2511F53, 0xCD9E8D57      # round multipliers
_W0, _W1 = 0x9E3779B9, 0xBB67AE85      # key schedule increments
_MASK32 = 0xFFFFFFFF


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds, element-wise over uint32 arrays (or ints).

    A round: (hi0, lo0) = M0 * c0, (hi1, lo1) = M1 * c2 as 64-bit products;
    the new counter is (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0).  The key is
    bumped by (W0, W1) between rounds.
    """
    c = [np.asarray(x, dtype=np.uint64) & _MASK32 for x in (c0, c1, c2, c3)]
    k0 = np.uint64(int(k0) & _MASK32)
    k1 = np.uint64(int(k1) & _MASK32)
    for r in range(10):
        if r:
            k0 = np.uint64((int(k0) + _W0) & _MASK32)
            k1 = np.uint64((int(k1) + _W1) & _MASK32)
        p0 = c[0] * np.uint64(_M0)
        p1 = c[2] * np.uint64(_M1)
        hi0, lo0 = p0 >> np.uint64(32), p0 & np.uint64(_MASK32)
        hi1, lo1 = p1 >> np.uint64(32), p1 & np.uint64(_MASK32)
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return [x.astype(np.uint32) for x in c]


def keep_threshold(p_drop):
    """8-bit threshold t and keep probability t / 256 for drop probability p."""
    t = int(round(256.0 * (1.0 - float(p_drop))))
    t = min(max(t, 1), 256)
    return t, t / 256.0


def keep_mask(bh, rows, n_keys, seed, offset, p_drop):
    """Boolean [len(rows), n_keys]: Z_ij for query rows ``rows`` of slice bh."""
    rows = np.asarray(rows, dtype=np.int64)
    t, _ = keep_threshold(p_drop)
    j = np.arange(n_keys, dtype=np.int64)
    qb = (rows // 4)[:, None] + np.zeros_like(j)[None, :]
    kb = (j // 4)[None, :] + np.zeros_like(rows)[:, None]
    words = philox4x32_10(kb, qb, np.full(kb.shape, bh), np.full(kb.shape, offset),
                          seed & _MASK32, (seed >> 32) & _MASK32)
    w = (rows % 4)[:, None] + np.zeros_like(j)[None, :]
    word = np.choose(w, words).astype(np.uint64)
    byte = (word >> (np.uint64(8) * (j % 4).astype(np.uint64))[None, :]) & np.uint64(0xFF)
    return byte < t


def ref_fwd_dropout_slice(q, k, v, scale, causal, p_drop, seed, offset, bh, valid_len=None,
                          rows=None, row_block=1024):
    """O [R, d], LSE [R] of one (batch, head) slice with dropout on P."""
    n = q.shape[0]
    valid_len = n if valid_len is None else valid_len
    rows = np.arange(n) if rows is None else np.asarray(rows)
    _, keep = keep_threshold(p_drop)
    out = np.zeros((rows.shape[0], v.shape[1]))
    lse = np.zeros(rows.shape[0])
    for r0 in range(0, rows.shape[0], row_block):
        rb = rows[r0:r0 + row_block]
        _, p, lse_b = _scores_probs(q, k, scale, causal, valid_len, rb)
        m = keep_mask(bh, rb, k.shape[0], seed, offset, p_drop) / keep
        out[r0:r0 + rb.shape[0]] = (p * m) @ v
        lse[r0:r0 + rb.shape[0]] = lse_b
    return out, lse


def ref_bwd_dropout_slice(q, k, v, do, scale, causal, p_drop, seed, offset, bh, valid_len=None,
                          row_block=1024):
    """dQ, dK, dV [N, d] of one (batch, head) slice for the loss <dO, O>."""
    n = q.shape[0]
    valid_len = n if valid_len is None else valid_len
    _, keep = keep_threshold(p_drop)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r0 in range(0, n, row_block):
        rb = np.arange(r0, min(n, r0 + row_block))
        _, p, _ = _scores_probs(q, k, scale, causal, valid_len, rb)
        m = keep_mask(bh, rb, k.shape[0], seed, offset, p_drop) / keep
        pm = p * m
        dv += pm.T @ do[rb]
        dp = m * (do[rb] @ v.T)
        dsum = (p * dp).sum(axis=1)
        ds = p * (dp - dsum[:, None])
        dq[rb] = scale * (ds @ k)
        dk += scale * (ds.T @ q[rb])
    return dq, dk, dv
