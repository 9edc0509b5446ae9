"""fa_bwd_noalloc: the backward pass on the library's static workspace.

It serves callers that cannot allocate device memory for a workspace (plugin
hosts that hand an operator only its input and output buffers, paths that
must not call cudaMalloc).  This file is named to be collected last.
"""

import numpy as np
import pytest
import torch

from helpers import GRAD_REL_MAX, assert_grad_close, f64
from oracle import ref_bwd_slice

pytestmark = pytest.mark.gpu


def _ptr(t):
    return t.data_ptr() if t is not None else None


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_noalloc_matches_fa_bwd_on_two_calls(d, causal):
    from exact_io_aware_47_b200 import _lib, build
    build.build()
    import exact_io_aware_47_b200 as fa
    from exact_io_aware_47_b200.inputs import make_inputs_shape

    B, H, N = 2, 4, 1000
    assert fa.workspace_bytes(B, H, N, d) <= _lib.fa_bwd_noalloc_max_bytes()
    inp = make_inputs_shape(B, H, N, d, torch.bfloat16, seed=77 + d, seqlens=[N, 613])
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    sl = inp["seqlens"].cuda()
    scale = d ** -0.5
    o, lse = fa.forward(q, k, v, scale=scale, causal=causal, seqlens=sl)
    ref = fa.backward(q, k, v, o, lse, do, scale=scale, causal=causal, seqlens=sl)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        st = _lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, scale, int(causal),
                                 _ptr(sl), _lib.FA_BF16, stream)
        assert st == _lib.FA_OK, _lib.status_string(st)
        dst, word = fa.device_status()
        assert dst == 0, f"device status {dst} ({word:#x}) on call {call}"
        for name, got, want in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
            g, r = f64(got), f64(want)
            assert np.isfinite(g).all()
            err = np.abs(g - r).max()
            assert err <= GRAD_REL_MAX * np.abs(r).max(), f"call {call} {name}: {err:.3e}"
        # dK and dV involve no atomics: identical to the allocating entry point
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
        # and all three against the float64 oracle, on a full-length slice and
        # on one of the batch whose keys are padded to 613
        for b, h in ((0, 0), (1, H - 1)):
            L = int(sl[b])
            g = ref_bwd_slice(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), f64(do[b, h]), scale,
                              causal, L)
            for n, (name, got) in enumerate(zip(("dQ", "dK", "dV"), (dq, dk, dv))):
                assert_grad_close(f64(got[b, h]), g[n], f"call {call} {name} b{b} h{h} (oracle)")


def test_noalloc_refuses_problems_beyond_its_array():
    from exact_io_aware_47_b200 import _lib, build
    build.build()
    B, H, N, d = 1, 64, 8192, 128  # workspace ~ 272 MB > 32 MiB
    P = 1 << 20  # never dereferenced: the size check comes first
    st = _lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, B, H, N, d, 0.088, 1, None,
                             _lib.FA_BF16, None)
    assert st == _lib.FA_ERR_SCRATCH_LIMIT
