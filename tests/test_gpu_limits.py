"""The largest problem the library accepts: B*H*N*d just below 2^31.

B1 H128 N131064 d128 bf16 causal (about 43 GB on the device).  The forward
is checked on sampled rows against the float64 oracle.  The backward is too
large for the oracle's dK/dV (every query row of a head), so it is checked
through identities that hold at any size: with P's rows summing to one,
sum_j dV_j = sum_i dO_i; with dS's rows summing to zero (D_i is the row's
own sum of P dP), sum_j dK_j = 0.  Offsets past 2^32 bytes in every tensor
exercise the 64-bit address arithmetic of all four kernels.
"""

import numpy as np
import pytest
import torch

from helpers import assert_fwd_close, f64, sample_rows
from oracle import ref_fwd_slice

pytestmark = pytest.mark.gpu

B, H, N, D = 1, 128, 131064, 128


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def test_largest_supported_problem(fa):
    from exact_io_aware_47_b200 import _lib
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    assert B * H * N * D < 2 ** 31 and B * H * (N + 8) * D >= 2 ** 31
    assert _lib.fa_bwd_workspace_size(B, H, N + 8, D) == 0      # one more row block is refused
    inp = make_inputs_shape(B, H, N, D, torch.bfloat16, seed=77, device="cuda")
    q, k, v, do = inp["q"], inp["k"], inp["v"], inp["do"]
    scale = D ** -0.5
    o, lse = fa.forward(q, k, v, causal=True)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=True)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    for h in (0, H - 1):
        rows = sample_rows(N, n_random=12, seed=h)
        ro, rl = ref_fwd_slice(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), scale, True, rows=rows,
                               row_block=64)
        assert_fwd_close(f64(o[0, h])[rows], f64(lse[0, h])[rows], ro, rl, f"max size h{h}")
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    # gradient identities per head, in float64 on the device
    for h in (0, H // 2, H - 1):
        sdv = dv[0, h].double().sum(0)
        sdo = do[0, h].double().sum(0)
        err = (sdv - sdo).abs().max().item()
        assert err <= 2e-2 * max(sdo.abs().max().item(), 1.0), (h, err)
        sdk = dk[0, h].double().sum(0)
        assert sdk.abs().max().item() <= 1e-2 * dk[0, h].double().abs().sum(0).max().item(), h
