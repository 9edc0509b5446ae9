"""Oracle for exact scaled-dot-product attention: plain, slow, CPU, float64.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code, table or helper with the CUDA
library.

What it computes is the plain definition of attention that the pages fix:

* "How Flash Attention Works" (swarnava.dev), section "How Flash Attention
  Works: The Exact-Attention Idea": the output is softmax(Q K^T / sqrt(d)) V,
  with causal masking when asked for.
* Same page, section "Tiling Q, K, and V for Fast On-Chip Memory": causal
  masking and padding are applied to the scores.
* "attn-flash-equivalence" (zenaique.com), section "Standard attention I/O is
  the bottleneck": the textbook schedule S = Q K^T / sqrt(d_k), then
  P = softmax(S) row-wise, then O = P V.  The oracle follows that schedule
  literally and materialises S and P.
* "How Flash Attention Works", section "The Backward Pass: Recomputation
  Instead of Stored Activations": gradients with respect to Q, K and V are
  taken through P; the per-row statistics that are kept are the running max
  and the normalisation sum, which this oracle reports folded into one
  log-sum-exp per row (LSE = m + ln l).

Readings of points the pages leave open (each is listed with its reason in the
design notes of the repository):

* scale is an argument (the configurations all use 1/sqrt(d));
* causal masking is top-left aligned: key j is visible to query i iff j <= i;
* padding is key padding: with a valid length L, keys j >= L are masked for
  every query row; query rows i >= L are still computed against the L valid
  keys;
* a row whose every key is masked yields O = 0 and LSE = -inf (cannot occur
  for dense inputs: L >= 1 and key 0 is always visible; it does with a block
  mask);
* block-sparse attention ("sparse-attention-flashattention" glossary page,
  definition: the original paper's block-sparse extension, a separate
  configuration of the same exact attention): a boolean block mask over
  (query block, key block) pairs of ``block`` x ``block`` scores hides every
  score of a block whose entry is false, on top of the causal and padding
  masks; the softmax runs over what remains;
* the gradients are those of O with respect to Q, K, V by the chain rule:
  dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij, dS = P * (dP - D),
  dQ = scale * dS K, dK = scale * dS^T Q.

All arrays are numpy float64.  Per-(batch, head) slices are independent, so
the oracle can evaluate one slice, or a subset of query rows of one slice,
exactly; that is how large configurations are sampled.
"""

import numpy as np

__all__ = [
    "allowed_mask",
    "ref_fwd_slice",
    "ref_fwd",
    "ref_bwd_slice",
    "ref_bwd",
]


def allowed_mask(rows, n_keys, valid_len, causal, block_mask=None, block=128):
    """Boolean [len(rows), n_keys]: True where key j is visible to query row i.

    Key padding masks keys j >= valid_len ("Tiling Q, K, and V" section:
    padding applied per tile).  Causal masking hides keys j > i ("The
    Exact-Attention Idea": causal masking for autoregressive decoding).  A
    block mask (boolean [query blocks, key blocks]) hides the scores of every
    block whose entry is false.
    """
    rows = np.asarray(rows)
    j = np.arange(n_keys)
    allowed = np.broadcast_to(j[None, :] < valid_len, (rows.shape[0], n_keys)).copy()
    if causal:
        allowed &= j[None, :] <= rows[:, None]
    if block_mask is not None:
        bm = np.asarray(block_mask, dtype=bool)
        allowed &= bm[rows[:, None] // block, j[None, :] // block]
    return allowed


def _scores_probs(q, k, scale, causal, valid_len, rows, block_mask=None, block=128):
    """S (masked with -inf) and P = softmax(S) for the given query rows.

    Follows the textbook schedule of the "Standard attention I/O is the
    bottleneck" section: S = scale * Q K^T, then row-wise softmax.
    Returns S, P, LSE (natural log) for those rows.
    """
    n_keys = k.shape[0]
    s = scale * (q[rows] @ k.T)                       # [R, N] float64
    allowed = allowed_mask(rows, n_keys, valid_len, causal, block_mask, block)
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1)                                 # row max
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.exp(s - m_safe[:, None])                   # exp(-inf) = 0 on masked keys
    l = e.sum(axis=1)                                 # normalisation sum
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(finite[:, None], e / np.where(finite, l, 1.0)[:, None], 0.0)
        lse = np.where(finite, m_safe + np.log(np.where(finite, l, 1.0)), -np.inf)
    return s, p, lse


def ref_fwd_slice(q, k, v, scale, causal, valid_len=None, rows=None, row_block=2048,
                  block_mask=None, block=128):
    """Forward attention of one (batch, head) slice.

    q, k, v: float64 [N, d].  Returns (O [R, d], LSE [R]) for the query rows
    ``rows`` (all rows when None), computed in blocks of ``row_block`` rows so
    that S and P for a block fit in host memory.  Blocking over query rows does
    not change any value: each row is computed independently.  ``block_mask``
    (boolean [ceil(N/block), ceil(N/block)] or None) restricts the scores as
    in allowed_mask.
    """
    n = q.shape[0]
    if valid_len is None:
        valid_len = n
    rows = np.arange(n) if rows is None else np.asarray(rows)
    out = np.zeros((rows.shape[0], v.shape[1]), dtype=np.float64)
    lse = np.zeros(rows.shape[0], dtype=np.float64)
    for r0 in range(0, rows.shape[0], row_block):
        rb = rows[r0:r0 + row_block]
        _, p, lse_b = _scores_probs(q, k, scale, causal, valid_len, rb, block_mask, block)
        out[r0:r0 + rb.shape[0]] = p @ v              # O = P V
        lse[r0:r0 + rb.shape[0]] = lse_b
    return out, lse


def ref_fwd(q, k, v, scale, causal, seqlens=None, row_block=2048):
    """Forward attention over [B, H, N, d] float64 arrays.

    seqlens: None or an int array [B] of valid key lengths (key padding).
    Returns (O [B, H, N, d], LSE [B, H, N]).
    """
    B, H, N, d = q.shape
    out = np.zeros((B, H, N, v.shape[3]), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    for b in range(B):
        L = N if seqlens is None else int(seqlens[b])
        for h in range(H):
            out[b, h], lse[b, h] = ref_fwd_slice(q[b, h], k[b, h], v[b, h], scale,
                                                 causal, L, None, row_block)
    return out, lse


def ref_bwd_slice(q, k, v, do, scale, causal, valid_len=None, q_rows=None,
                  k_rows=None, row_block=2048, block_mask=None, block=128):
    """Gradients of one (batch, head) slice for the loss <dO, O>.

    Returns (dQ [len(q_rows), d], dK [len(k_rows), d], dV [len(k_rows), dv]).
    dQ of a query row needs only that row of P; dK and dV of a key row need
    the whole column of P and therefore every query row, so all rows are
    visited in blocks, while only the requested key rows are accumulated.

    Chain rule through the textbook schedule:
      dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij,
      dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
    Rows without a visible key have P = 0 and contribute nothing.
    """
    n = q.shape[0]
    if valid_len is None:
        valid_len = n
    q_rows = np.arange(n) if q_rows is None else np.asarray(q_rows)
    k_rows = np.arange(n) if k_rows is None else np.asarray(k_rows)
    want_q = np.zeros(n, dtype=bool)
    want_q[q_rows] = True

    dq_all = {}
    dk = np.zeros((k_rows.shape[0], k.shape[1]), dtype=np.float64)
    dv = np.zeros((k_rows.shape[0], v.shape[1]), dtype=np.float64)
    all_rows = np.arange(n)
    for r0 in range(0, n, row_block):
        rb = all_rows[r0:r0 + row_block]
        _, p, _ = _scores_probs(q, k, scale, causal, valid_len, rb, block_mask, block)
        dp = do[rb] @ v.T                                             # [R, N]
        dsum = (p * dp).sum(axis=1)                                   # D_i
        ds = p * (dp - dsum[:, None])                                 # dS
        sel = want_q[rb]
        if sel.any():
            dq_b = scale * (ds[sel] @ k)
            for i, r in enumerate(rb[sel]):
                dq_all[int(r)] = dq_b[i]
        dv += p[:, k_rows].T @ do[rb]
        dk += scale * (ds[:, k_rows].T @ q[rb])
    dq = np.stack([dq_all[int(r)] for r in q_rows]) if q_rows.shape[0] else \
        np.zeros((0, q.shape[1]))
    return dq, dk, dv


def ref_bwd(q, k, v, do, scale, causal, seqlens=None, row_block=2048):
    """Gradients over [B, H, N, d] float64 arrays. Returns (dQ, dK, dV)."""
    B, H, N, d = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        L = N if seqlens is None else int(seqlens[b])
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = ref_bwd_slice(
                q[b, h], k[b, h], v[b, h], do[b, h], scale, causal, L,
                None, None, row_block)
    return dq, dk, dv
