"""Float64 model of the tile-by-tile online-softmax recurrence.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.attention``): it exists to
check, apart from any kernel, that the schedule the CUDA forward kernel uses
reaches the plain definition exactly.

It follows the steps the pages give, in their order:

* "FlashAttention" (whatisai.fyi), section "How it works": split Q, K, V into
  blocks; load blocks on chip; compute attention block by block while keeping
  softmax statistics; write the output blocks back.
* "How Flash Attention Works" (swarnava.dev), section "Tiling Q, K, and V":
  one block of query rows stays resident while K and V blocks stream past it;
  causal and padding masks are applied per tile.
* Same page, section "Online Softmax Without the Full Score Matrix": every K/V
  tile updates a running row max and a running normalisation sum; when the max
  grows, the partial output and the sum are rescaled by the ratio of the old
  to the new max before the new tile's contribution is added; the recurrence
  is exact.

Two implementation choices of the kernel are modelled, both exact in real
arithmetic:

* base-2 exponentials: scores are carried as c * s with c = scale * log2(e),
  so exp(scale * s - m) = 2^(c * s - m');
* lazy rescaling with threshold ``tau`` (log2 units): the running max is only
  moved when the new tile's max exceeds it by more than ``tau``.  Values up to
  2^tau then enter the sum, and the final division uses the same (stale) max,
  so the quotient is unchanged.  ``tau = 0`` is the eager schedule the page
  describes; ``tau = inf`` fixes the max at the first visited tile.

Fully masked tiles are skipped, as the kernel skips them.
"""

import math

import numpy as np

__all__ = ["tiled_fwd_slice"]

_LOG2E = 1.0 / math.log(2.0)
_LN2 = math.log(2.0)


def tiled_fwd_slice(q, k, v, scale, causal, valid_len=None, block_m=128,
                    block_n=128, tau=8.0):
    """Online-softmax forward of one (batch, head) slice in float64.

    Returns (O [N, d], LSE [N]) with LSE in natural-log units.
    """
    n = q.shape[0]
    if valid_len is None:
        valid_len = n
    c = scale * _LOG2E
    out = np.zeros((n, v.shape[1]), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    for q0 in range(0, n, block_m):
        rows = np.arange(q0, min(q0 + block_m, n))
        m = np.full(rows.shape[0], -np.inf)            # running max (log2 units)
        l = np.zeros(rows.shape[0])                    # running sum
        acc = np.zeros((rows.shape[0], v.shape[1]))    # unnormalised output
        for k0 in range(0, n, block_n):
            keys = np.arange(k0, min(k0 + block_n, n))
            allowed = keys[None, :] < valid_len
            if causal:
                allowed = allowed & (keys[None, :] <= rows[:, None])
            else:
                allowed = np.broadcast_to(allowed, (rows.shape[0], keys.shape[0]))
            if not allowed.any():
                continue                               # fully masked tile: skipped
            t = c * (q[rows] @ k[keys].T)              # tile scores, log2 units
            t = np.where(allowed, t, -np.inf)
            tile_max = t.max(axis=1)
            with np.errstate(invalid="ignore"):
                grow = tile_max > m + tau              # (-inf) + inf: False, handled by first
            first = ~np.isfinite(m)
            move = (grow | first) & np.isfinite(tile_max)
            m_new = np.where(move, tile_max, m)
            with np.errstate(invalid="ignore"):
                alpha = np.where(move & ~first, np.exp2(m - m_new), 1.0)
            alpha = np.where(first & move, 0.0, alpha)
            acc *= alpha[:, None]                      # rescale partial output
            l *= alpha                                 # rescale partial sum
            m = m_new
            m_safe = np.where(np.isfinite(m), m, 0.0)
            p = np.exp2(t - m_safe[:, None])           # masked keys give 0
            l += p.sum(axis=1)
            acc += p @ v[keys]
        with np.errstate(divide="ignore", invalid="ignore"):
            done = l > 0
            out[rows] = np.where(done[:, None], acc / np.where(done, l, 1.0)[:, None], 0.0)
            lse[rows] = np.where(done, (m + np.log2(np.where(done, l, 1.0))) * _LN2, -np.inf)
    return out, lse
