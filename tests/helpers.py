"""Shared test helpers: tolerances, sampling, conversion to float64."""

import numpy as np
import torch

# Tolerances of the parity contract (floating-point results agree with the
# float64 oracle up to rounding, not bit for bit).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_MAX = 5e-2   # max |d(grad)| <= GRAD_REL_MAX * max |ref grad|
# Where the exact gradient vanishes (a row with one visible key: dS = P (dP - D)
# = 0), fp32 evaluation of D_i = <dO_i, O_i> and of dP_i0 in different
# summation orders leaves |dS| ~ 2^-23 sum |dO O| ~ 1e-6, so dQ ~ scale |K| 1e-6.
# The relative bound then gets this absolute floor (GRAD_REL_MAX * 1e-4 = 5e-6).
GRAD_ABS_FLOOR = 1e-4


def f64(t):
    """torch tensor (any device, 16-bit or float) -> float64 numpy."""
    return t.detach().to("cpu", torch.float64).numpy()


def sample_rows(N, n_random=96, seed=0, block=128):
    """Rows of every kind: first and last rows, rows around each of the first
    few tile boundaries, the ragged tail, and a seeded random sample."""
    rows = set(range(min(N, 4))) | set(range(max(0, N - 4), N))
    for b in range(block, min(N, 6 * block), block):
        rows |= {b - 2, b - 1, b, b + 1}
    last_tile = (N - 1) // block * block
    rows |= {last_tile, min(N - 1, last_tile + 1)}
    rng = np.random.default_rng(seed)
    rows |= set(rng.integers(0, N, size=min(n_random, N)).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N))


def subset_slices(B, H):
    """The fixed (batch, head) subset the large workloads are checked on:
    (0, 0), (0, H-1), (B-1, H/2), (B-1, H-1), without repeats.  Slices are
    independent problems, so checking some of them exactly is exact for
    those slices."""
    out = []
    for s in ((0, 0), (0, H - 1), (B - 1, H // 2), (B - 1, H - 1)):
        if s not in out:
            out.append(s)
    return out


def assert_fwd_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    do = np.abs(o_gpu - o_ref)
    dl = np.abs(lse_gpu - lse_ref)
    assert np.isfinite(o_gpu).all() and np.isfinite(lse_gpu).all(), f"{what}: non-finite output"
    assert do.max() <= O_MAX_ABS, f"{what}: O max|d| {do.max():.3e}"
    assert do.mean() <= O_MEAN_ABS, f"{what}: O mean|d| {do.mean():.3e}"
    assert dl.max() <= LSE_MAX_ABS, f"{what}: LSE max|d| {dl.max():.3e}"
    return do.max(), do.mean(), dl.max()


def assert_grad_close(g_gpu, g_ref, what="", typical=None, floor_frac=1e-3):
    """max |g_gpu - g_ref| <= GRAD_REL_MAX * max|g_ref|.

    ``typical`` is the gradient magnitude of the whole tensor the slice comes
    from.  Rounding residuals scale with the magnitudes being combined, not
    with a slice's exact result, so a slice whose exact gradient vanishes (one
    visible key) is held to GRAD_REL_MAX * floor_frac * typical (and never
    less than GRAD_REL_MAX * GRAD_ABS_FLOOR).
    """
    assert np.isfinite(g_gpu).all(), f"{what}: non-finite gradient"
    err = np.abs(g_gpu - g_ref).max()
    scale = np.abs(g_ref).max()
    floor = GRAD_ABS_FLOOR if typical is None else max(GRAD_ABS_FLOOR, floor_frac * typical)
    assert err <= GRAD_REL_MAX * max(scale, floor), \
        f"{what}: max|d| {err:.3e} vs max|ref| {scale:.3e}"
    return err / max(scale, 1e-30)
