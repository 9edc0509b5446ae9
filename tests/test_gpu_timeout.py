"""Device-side failure detection: a pipeline wait that runs out.

Every producer/consumer wait inside the kernels is bounded
(fa_set_wait_limit_ns, 2 s by default).  With a bound of 1 ns, ordinary waits
of a correct pipeline give up: the kernel must record FA_ERR_DEVICE_TIMEOUT
with the site of the wait, stop its other roles, wait for the copies and
tensor-core work already in flight, release its tensor memory and return.
The test then restores the bound and checks that the next calls on the same
context match the oracle.  No fault, trap or endless wait is involved: the
waits that run out are ordinary ones, only given less time.
"""

import numpy as np
import pytest
import torch

from helpers import assert_fwd_close, assert_grad_close, f64
from oracle import ref_bwd_slice, ref_fwd_slice

pytestmark = pytest.mark.gpu

FWD_SITES = set(range(1, 10))      # the forward kernel's waits
BWD_SITES = set(range(20, 40))     # the backward kernel's waits


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def _inputs():
    from exact_io_aware_47_b200.inputs import make_inputs_shape
    inp = make_inputs_shape(1, 4, 1000, 128, torch.bfloat16, seed=31)
    return [inp[n].cuda() for n in ("q", "k", "v", "do")]


def _with_short_waits(lib, fn):
    prev = lib.fa_set_wait_limit_ns(1)
    try:
        fn()
    finally:
        lib.fa_set_wait_limit_ns(prev)


def test_forward_wait_timeout_is_reported_and_the_context_stays_usable(fa):
    from exact_io_aware_47_b200 import _lib
    q, k, v, _ = _inputs()
    _with_short_waits(_lib, lambda: fa.forward(q, k, v, causal=True))
    st, word = fa.device_status()
    assert st == _lib.FA_ERR_DEVICE_TIMEOUT, f"status {st} word {word:#x}"
    assert (word >> 8) & 0xFF in FWD_SITES, f"site of word {word:#x}"
    assert fa.device_status()[0] == _lib.FA_OK                 # read and cleared
    o, lse = fa.forward(q, k, v, causal=True)
    st, word = fa.device_status()
    assert st == _lib.FA_OK, f"status {st} word {word:#x}"
    for h in range(q.shape[1]):
        ro, rl = ref_fwd_slice(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), 128 ** -0.5, True)
        assert_fwd_close(f64(o[0, h]), f64(lse[0, h]), ro, rl, f"after timeout h{h}")


def test_backward_wait_timeout_is_reported_and_the_context_stays_usable(fa):
    from exact_io_aware_47_b200 import _lib
    q, k, v, do = _inputs()
    o, lse = fa.forward(q, k, v, causal=True)
    assert fa.device_status()[0] == _lib.FA_OK
    _with_short_waits(_lib, lambda: fa.backward(q, k, v, o, lse, do, causal=True))
    st, word = fa.device_status()
    assert st == _lib.FA_ERR_DEVICE_TIMEOUT, f"status {st} word {word:#x}"
    assert (word >> 8) & 0xFF in BWD_SITES, f"site of word {word:#x}"
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=True)
    st, word = fa.device_status()
    assert st == _lib.FA_OK, f"status {st} word {word:#x}"
    for h in range(q.shape[1]):
        g = ref_bwd_slice(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), f64(do[0, h]),
                          128 ** -0.5, True)
        for n, got in enumerate((dq, dk, dv)):
            assert_grad_close(f64(got[0, h]), g[n], f"after timeout grad {n} h{h}")
