"""Oracle for attention on 8-bit floating-point (e4m3) inputs: plain, CPU.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use
it.  It shares no code with the CUDA library.

What the pages fix: "How Flash Attention Works" (swarnava.dev), section
"FlashAttention 2 and 3", says that the third version adds lower-precision
paths on hardware that supports them.  Nothing more is given, so the readings
below (listed with their reasons in the design notes) define the path:

* the format is e4m3 as in the OCP 8-bit floating-point specification: one
  sign bit, four exponent bits with bias 7, three mantissa bits, subnormals
  with spacing 2^-9, no infinities, largest finite value 448; conversions
  round to nearest (ties to even) and saturate to +-448;
* per-tile scaling: each 128-row tile t of a (batch, head) slice of Q, K or V
  carries one positive fp32 descale factor, and the tensor it stands for is
  decode(code) * descale[t];
* the quantiser (``quantize_tiles``) takes descale = amax / 448 for a tile
  whose largest magnitude is amax; it computes 448 / amax and the product
  x * (448 / amax) in fp32 and rounds that to e4m3, so the integer codes are
  decided in fp32 (a tile of zeros gets descale 1);
* the attention (``ref_fwd_fp8_slice``) is the tiled online softmax of the
  "Online Softmax Without the Full Score Matrix" section on the dequantised
  scores, with the two steps that an 8-bit P V product needs: the
  probabilities of key tile j are multiplied by rho_j = sv_j / max_j' sv_j'
  (the V descale of the tile over the largest V descale of the slice's valid
  key tiles) and rounded to e4m3 before they multiply the e4m3 codes of V;
  the row sum l uses the probabilities before that rounding, and the output is
  O = max sv * acc / l.  The running max moves lazily (threshold 8 in log2
  units), as in the online model, because the rounding grid of P depends on
  which max it is taken against.

Floating-point work runs in float64 except where fp32 is named above.
"""

import math

import numpy as np

from .attention import allowed_mask

__all__ = ["E4M3_MAX", "e4m3_round", "e4m3_encode", "e4m3_decode", "quantize_tiles",
           "dequantize_tiles", "ref_fwd_fp8_slice", "fp8_error_bound"]

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6     # smallest normal: 2^-6
_MANT_BITS = 3
_LOG2E = 1.0 / math.log(2.0)
_LN2 = math.log(2.0)


def e4m3_round(x):
    """Nearest e4m3 value (ties to even), saturating to +-448; float64 in/out.

    In the binade [2^e, 2^(e+1)) the spacing is 2^(e-3); below 2^-6 the
    subnormal spacing 2^-9 applies.  Division by a power of two is exact, so
    rint() does the round-to-nearest-even on the exact quotient.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                      # a = f 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, _MIN_NORMAL_EXP)  # floor(log2 a), clamped to the normal floor
    step = np.ldexp(1.0, e - _MANT_BITS)
    q = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    return np.copysign(q, x)


def e4m3_encode(x):
    """uint8 codes of e4m3_round(x): sign << 7 | exponent << 3 | mantissa."""
    x = np.asarray(x, dtype=np.float64)
    q = np.abs(e4m3_round(x))
    sign = np.signbit(x).astype(np.uint8) << 7
    nan = np.isnan(q)
    q = np.where(nan, 0.0, q)
    sub = q < 2.0 ** _MIN_NORMAL_EXP
    # subnormals (and zero): mantissa = q / 2^-9; q = 2^-6 would give 8, which
    # is exponent field 1, mantissa 0: the same code
    code_sub = np.rint(np.ldexp(q, 9))
    _, ex = np.frexp(np.where(sub, 1.0, q))
    e = ex - 1                                # floor(log2 q) for normals
    mant = np.ldexp(np.where(sub, 1.0, q), -e) - 1.0   # in [0, 1), multiple of 1/8
    code_norm = (e + 7) * 8 + np.rint(mant * 8)
    code = np.where(sub, code_sub, code_norm).astype(np.uint8)
    code = np.where(nan, np.uint8(0x7F), code)
    return (code | sign).astype(np.uint8)


def e4m3_decode(codes):
    """float64 values of uint8 e4m3 codes (0x7F / 0xFF are NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, np.ldexp(m.astype(np.float64), -9),
                   np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


def quantize_tiles(x, block=128):
    """Per-tile e4m3 quantisation of one slice x [N, d] (fp32-exact values).

    Returns (codes uint8 [N, d], descale float32 [ceil(N / block)]).  For tile
    t with amax = max |x| over its rows: descale = fp32(amax / 448),
    inv = fp32(448 / amax), codes = e4m3(fp32(x * inv)); a tile of zeros has
    descale 1 and codes of +-0.
    """
    x = np.asarray(x, dtype=np.float32)
    n = x.shape[0]
    nt = (n + block - 1) // block
    codes = np.zeros(x.shape, dtype=np.uint8)
    descale = np.ones(nt, dtype=np.float32)
    for t in range(nt):
        blk = x[t * block:(t + 1) * block]
        amax = np.float32(np.abs(blk).max())
        if amax == 0:
            codes[t * block:(t + 1) * block] = e4m3_encode(blk.astype(np.float64))
            continue
        inv = np.float32(E4M3_MAX) / amax               # fp32, rounded to nearest
        descale[t] = amax / np.float32(E4M3_MAX)
        y = (blk * inv).astype(np.float32)              # fp32 products
        codes[t * block:(t + 1) * block] = e4m3_encode(y.astype(np.float64))
    return codes, descale


def dequantize_tiles(codes, descale, block=128):
    """float64 [N, d]: decode(codes) * descale of the row's tile."""
    vals = e4m3_decode(codes)
    rows = np.arange(vals.shape[0]) // block
    return vals * np.asarray(descale, dtype=np.float64)[rows][:, None]


def _key_tiles(valid_len, block):
    return (valid_len + block - 1) // block


def ref_fwd_fp8_slice(q8, k8, v8, sq, sk, sv, scale, causal, valid_len=None, rows=None,
                      block=128, tau=8.0):
    """Forward attention of one (batch, head) slice on e4m3 inputs.

    q8, k8, v8: uint8 codes [N, d]; sq, sk, sv: descales per 128-row tile.
    Returns (O [R, d], LSE [R]) for query rows ``rows`` (all when None), LSE in
    natural-log units.  Each row walks its key tiles in ascending order (the
    ones the causal and key-length limits leave), with the online softmax of
    the module docstring: lazy max, P rounded to e4m3 after the V-descale
    ratio, l from the unrounded P.
    """
    n = q8.shape[0]
    valid_len = n if valid_len is None else valid_len
    rows = np.arange(n) if rows is None else np.asarray(rows)
    qv, kv, vv = e4m3_decode(q8), e4m3_decode(k8), e4m3_decode(v8)
    sq, sk, sv = (np.asarray(a, dtype=np.float64) for a in (sq, sk, sv))
    nkb = _key_tiles(valid_len, block)
    sv_max = sv[:nkb].max()
    c = scale * _LOG2E
    out = np.zeros((rows.shape[0], v8.shape[1]))
    lse = np.zeros(rows.shape[0])
    for qt in np.unique(rows // block):
        sel = np.nonzero(rows // block == qt)[0]
        r = rows[sel]
        jend = min(nkb, qt + 1) if causal else nkb
        m = np.full(r.shape[0], -np.inf)
        l = np.zeros(r.shape[0])
        acc = np.zeros((r.shape[0], v8.shape[1]))
        qd = qv[r] * sq[qt]                                   # dequantised query rows
        for j in range(jend):
            keys = np.arange(j * block, min((j + 1) * block, n))
            t = c * (qd @ (kv[keys] * sk[j]).T)               # scores of tile j, log2 units
            allowed = allowed_mask(r, n, valid_len, causal)[:, keys]
            t = np.where(allowed, t, -np.inf)
            tmax = t.max(axis=1)
            with np.errstate(invalid="ignore"):
                move = tmax > m + tau                         # first finite tile always moves
            m_new = np.where(move, tmax, m)
            with np.errstate(invalid="ignore"):
                alpha = np.where(move & np.isfinite(m), np.exp2(m - m_new), 1.0)
            alpha = np.where(move & ~np.isfinite(m), 0.0, alpha)
            acc *= alpha[:, None]
            l *= alpha
            m = m_new
            m_safe = np.where(np.isfinite(m), m, 0.0)
            p = np.exp2(t - m_safe[:, None])                  # masked keys give 0
            l += p.sum(axis=1)
            p8 = e4m3_round(p * (sv[j] / sv_max))             # the 8-bit A operand of P V
            acc += p8 @ vv[keys]
        with np.errstate(divide="ignore", invalid="ignore"):
            done = l > 0
            out[sel] = np.where(done[:, None], acc * sv_max / np.where(done, l, 1.0)[:, None], 0.0)
            lse[sel] = np.where(done, (m + np.log2(np.where(done, l, 1.0))) * _LN2, -np.inf)
    return out, lse


def fp8_error_bound(q8, k8, v8, sq, sk, sv, scale, causal, valid_len=None, rows=None,
                    block=128, tau=8.0):
    """Element-wise bound on |ref_fwd_fp8_slice - exact attention| [R, d].

    Exact attention is the plain softmax(scale Q K^T) V of the dequantised
    inputs.  The only difference is the rounding of rho_j P to e4m3 (l uses
    the unrounded P): with P taken against a stale max m' in
    [m - tau, m] (log2 units), rho_j P_ij lies in [0, 2^tau], and rounding it
    changes it by at most 2^-4 of itself when it is normal (>= 2^-6) and by at
    most 2^-10 when it is subnormal.  Divided by l' >= L_i = sum_j 2^(c s_ij -
    max c s_i) (l' sums the same terms scaled by 2^(m - m') >= 1) and
    multiplied by max sv |v8|, the row error is at most
      2^-4 sum_j p_ij |v_j| + 2^-10 max sv sum_{j subnormal-capable} |v8_j| / L_i,
    where p is the exact softmax and rho_j P'_ij >= rho_j 2^(c s_ij - max c s_i)
    can be subnormal only if that lower end is below 2^-6.
    """
    n = q8.shape[0]
    valid_len = n if valid_len is None else valid_len
    rows = np.arange(n) if rows is None else np.asarray(rows)
    qd = dequantize_tiles(q8, sq, block)
    kd = dequantize_tiles(k8, sk, block)
    vd = dequantize_tiles(v8, sv, block)
    v8v = np.abs(e4m3_decode(v8))
    sv = np.asarray(sv, dtype=np.float64)
    nkb = _key_tiles(valid_len, block)
    sv_max = sv[:nkb].max()
    rho = np.zeros(n)
    for j in range(nkb):
        rho[j * block:(j + 1) * block] = sv[j] / sv_max
    c = scale * _LOG2E
    s = c * (qd[rows] @ kd.T)
    s = np.where(allowed_mask(rows, n, valid_len, causal), s, -np.inf)
    mx = s.max(axis=1)
    e = np.exp2(s - mx[:, None])
    big_l = e.sum(axis=1)
    p = e / big_l[:, None]
    maybe_sub = (rho[None, :] * e < 2.0 ** -6) & np.isfinite(s)
    term_rel = 2.0 ** -4 * (p @ np.abs(vd))
    term_sub = 2.0 ** -10 * sv_max * (maybe_sub.astype(np.float64) @ v8v) / big_l[:, None]
    return term_rel + term_sub
