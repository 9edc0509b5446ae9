"""Packed variable-length batches: CUDA path (fa_fwd_varlen / fa_bwd_varlen
through the C ABI) vs the float64 oracle, one sequence at a time.

A packed sequence is an attention problem of its own (no padding), so the
oracle's per-slice functions apply unchanged to rows
cu_seqlens[b] .. cu_seqlens[b + 1] - 1 of each head.
"""

import numpy as np
import pytest
import torch

from helpers import assert_fwd_close, assert_grad_close, f64, sample_rows
from oracle import ref_bwd_slice, ref_fwd_slice

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_47_b200 import build
    build.build()
    import exact_io_aware_47_b200 as pkg
    return pkg


def _run(fa, inp, causal, scale, backward=True):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    cu, ms = inp["cu_seqlens"].cuda(), inp["max_seqlen"]
    o, lse = fa.forward_varlen(q, k, v, cu, ms, scale=scale, causal=causal)
    out = {"q": q, "k": k, "v": v, "o": o, "lse": lse}
    if backward:
        do = inp["do"].cuda()
        out["do"] = do
        out["dq"], out["dk"], out["dv"] = fa.backward_varlen(q, k, v, o, lse, do, cu, ms,
                                                             scale=scale, causal=causal)
    st, word = fa.device_status()
    assert st == 0, f"device status {st} word {word:#x}"
    return out


def _bounds(inp):
    cu = [int(x) for x in inp["cu_seqlens"].cpu()]
    return [(b, cu[b], cu[b + 1]) for b in range(len(cu) - 1)]


def _check_full(fa, inp, causal, scale, what):
    r = _run(fa, inp, causal, scale)
    H = r["q"].shape[0]
    g = {n: f64(r[n]) for n in ("q", "k", "v", "o", "lse", "do", "dq", "dk", "dv")}
    for h in range(H):
        refs = []
        for b, s0, s1 in _bounds(inp):
            if s1 == s0:
                continue
            sl = slice(s0, s1)
            ro, rl = ref_fwd_slice(g["q"][h, sl], g["k"][h, sl], g["v"][h, sl], scale, causal)
            assert_fwd_close(g["o"][h, sl], g["lse"][h, sl], ro, rl, f"{what} h{h} seq{b}")
            refs.append((b, sl, ref_bwd_slice(g["q"][h, sl], g["k"][h, sl], g["v"][h, sl],
                                              g["do"][h, sl], scale, causal)))
        # The tolerance is stated per gradient tensor (here a head's [T, d]
        # rows); each sequence is also held to it relative to its own
        # magnitude, down to 5 % of the head's.  Below that, rounding of O to
        # 16 bits before D = <dO, O> dominates: for a causal sequence of two
        # keys the float64 chain rule with D from the rounded O differs from
        # the exact one by 0.08 % of the head's largest dK (5 % of the
        # sequence's own).
        typical = [max(np.abs(x[2][n]).max() for x in refs) for n in range(3)]
        for b, sl, ref in refs:
            for n, name in enumerate(("dq", "dk", "dv")):
                assert_grad_close(g[name][h, sl], ref[n], f"{what} {name} h{h} seq{b}",
                                  typical=typical[n], floor_frac=5e-2)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_edge_lengths_full(fa, d, causal):
    from exact_io_aware_47_b200.inputs import make_inputs_varlen
    lengths = [1, 127, 128, 129, 0, 300, 255, 2]
    inp = make_inputs_varlen(len(lengths), 2, 300, d, torch.bfloat16, seed=11 + d,
                             lengths=lengths)
    _check_full(fa, inp, causal, d ** -0.5, f"packed d{d} causal{causal}")


def test_fp16_single_sequence_equals_whole_tensor(fa):
    from exact_io_aware_47_b200.inputs import make_inputs_varlen
    inp = make_inputs_varlen(1, 3, 700, 128, torch.float16, seed=3, lengths=[700])
    _check_full(fa, inp, True, 0.3, "packed fp16 one sequence")


@pytest.mark.parametrize("causal", [False, True])
def test_packed_workload_sampled(fa, causal):
    """8 sequences, lengths ~ U{1..4099}, H16 d128 bf16: sampled rows of every
    sequence of two heads, forward and backward."""
    from exact_io_aware_47_b200.inputs import PACKED_WORKLOADS, make_inputs_packed
    w = PACKED_WORKLOADS["varlen"]
    inp = make_inputs_packed("varlen", device="cuda")
    r = _run(fa, inp, causal, w.scale)
    for h in (0, w.H - 1):
        for b, s0, s1 in _bounds(inp):
            L = s1 - s0
            sl = slice(s0, s1)
            q, k, v, do = (f64(r[n][h, sl]) for n in ("q", "k", "v", "do"))
            rows = sample_rows(L, n_random=24, seed=100 * b + h)
            ro, rl = ref_fwd_slice(q, k, v, w.scale, causal, rows=rows, row_block=512)
            assert_fwd_close(f64(r["o"][h, sl])[rows], f64(r["lse"][h, sl])[rows], ro, rl,
                             f"varlen h{h} seq{b}")
            kr = sample_rows(L, n_random=24, seed=100 * b + h + 7)
            gq, gk, gv = ref_bwd_slice(q, k, v, do, w.scale, causal, q_rows=rows, k_rows=kr,
                                       row_block=1024)
            assert_grad_close(f64(r["dq"][h, sl])[rows], gq, f"varlen dQ h{h} seq{b}")
            assert_grad_close(f64(r["dk"][h, sl])[kr], gk, f"varlen dK h{h} seq{b}")
            assert_grad_close(f64(r["dv"][h, sl])[kr], gv, f"varlen dV h{h} seq{b}")


@pytest.mark.parametrize("causal", [False, True])
def test_packed_equals_padded_layout(fa, causal):
    """The same sequences laid out padded ([B, H, N, d] with key lengths) and
    packed run the same tile arithmetic: O, LSE, dK and dV of every valid row
    agree bit for bit (dO of the padded query rows is zero, so those rows
    contribute exactly zero; dQ is reduced in arbitrary order and is compared
    with a tolerance)."""
    from exact_io_aware_47_b200.inputs import make_inputs_varlen
    lengths = [300, 1, 129, 256, 77]
    H, d = 2, 128
    inp = make_inputs_varlen(len(lengths), H, 300, d, torch.bfloat16, seed=21, lengths=lengths)
    r = _run(fa, inp, causal, d ** -0.5)
    B, N = len(lengths), max(lengths)
    pad = {n: torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
           for n in ("q", "k", "v", "do")}
    for b, s0, s1 in _bounds(inp):
        for n in pad:
            pad[n][b, :, :s1 - s0] = r[n][:, s0:s1]
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    o, lse = fa.forward(pad["q"], pad["k"], pad["v"], causal=causal, seqlens=sl)
    dq, dk, dv = fa.backward(pad["q"], pad["k"], pad["v"], o, lse, pad["do"], causal=causal,
                             seqlens=sl)
    for b, s0, s1 in _bounds(inp):
        L = s1 - s0
        assert torch.equal(o[b, :, :L], r["o"][:, s0:s1])
        assert torch.equal(lse[b, :, :L], r["lse"][:, s0:s1])
        assert torch.equal(dk[b, :, :L], r["dk"][:, s0:s1])
        assert torch.equal(dv[b, :, :L], r["dv"][:, s0:s1])
        err = (dq[b, :, :L].float() - r["dq"][:, s0:s1].float()).abs().max().item()
        assert err <= 1e-2 * max(dq[b, :, :L].float().abs().max().item(), 1e-3)


def test_rows_outside_every_sequence(fa):
    """Rows after cu_seqlens[B] belong to no sequence: o, lse, dk and dv leave
    them untouched; dq is zero there."""
    from exact_io_aware_47_b200.inputs import make_inputs_varlen
    lengths = [130, 5]
    H, d, extra = 2, 64, 37
    inp = make_inputs_varlen(len(lengths), H, 130, d, torch.bfloat16, seed=5, lengths=lengths)
    T = sum(lengths)
    big = {n: torch.randn((H, T + extra, d), device="cuda").to(torch.bfloat16)
           for n in ("q", "k", "v", "do")}
    for n in big:
        big[n][:, :T] = inp[n].cuda()
    cu, ms = inp["cu_seqlens"].cuda(), inp["max_seqlen"]
    o = torch.full((H, T + extra, d), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, T + extra), 7.0, device="cuda")
    fa.forward_varlen(big["q"], big["k"], big["v"], cu, ms, causal=True, out=o, lse=lse)
    dk = torch.full_like(o, 7.0)
    dv = torch.full_like(o, 7.0)
    dq = torch.full_like(o, 7.0)
    fa.backward_varlen(big["q"], big["k"], big["v"], o, lse, big["do"], cu, ms, causal=True,
                       dq=dq, dk=dk, dv=dv)
    assert fa.device_status()[0] == 0
    for t in (o, dk, dv):
        assert torch.all(t[:, T:] == 7.0)
    assert torch.all(lse[:, T:] == 7.0)
    assert torch.all(dq[:, T:] == 0.0)
    ref = _run(fa, inp, True, d ** -0.5)
    assert torch.equal(o[:, :T], ref["o"]) and torch.equal(dk[:, :T], ref["dk"])


def test_bad_offsets_are_clamped_and_reported(fa):
    from exact_io_aware_47_b200 import _lib
    from exact_io_aware_47_b200.inputs import make_inputs_varlen
    inp = make_inputs_varlen(3, 1, 100, 64, torch.bfloat16, seed=9, lengths=[40, 50, 10])
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    fa.device_status()
    for cu in ([0, 40, 90, 200], [0, 60, 50, 100], [0, 40, 90, 100]):
        ms = 45 if cu == [0, 40, 90, 100] else 100  # last: sequence 1 longer than max_seqlen
        o, lse = fa.forward_varlen(q, k, v, torch.tensor(cu, dtype=torch.int32), ms)
        st, word = fa.device_status()
        assert st == _lib.FA_ERR_DEVICE_SEQLEN, (cu, st, hex(word))
        assert torch.isfinite(o.float()).all()


def test_host_side_rejections(fa):
    from exact_io_aware_47_b200 import _lib
    q = torch.zeros((1, 128, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.zeros((1, 128), device="cuda")
    cu = torch.tensor([0, 128], dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    ok = _lib.fa_fwd_varlen(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(),
                            cu.data_ptr(), 1, 1, 128, 128, 64, 0.125, 0, _lib.FA_BF16, s)
    assert ok == _lib.FA_OK
    bad = [dict(cu=None), dict(ms=0), dict(B=0), dict(T=0), dict(d=96)]
    for kw in bad:
        args = dict(cu=cu.data_ptr(), B=1, T=128, ms=128, d=64)
        args.update(kw)
        st = _lib.fa_fwd_varlen(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), args["cu"], args["B"], 1, args["T"], args["ms"],
                                args["d"], 0.125, 0, _lib.FA_BF16, s)
        assert st in (_lib.FA_ERR_INVALID_ARG, _lib.FA_ERR_UNSUPPORTED), (kw, st)
    ws = torch.empty(_lib.fa_bwd_varlen_workspace_size(1, 1, 128, 64) - 256, dtype=torch.uint8,
                     device="cuda")
    st = _lib.fa_bwd_varlen(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(),
                            lse.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(),
                            ws.data_ptr(), ws.numel(), cu.data_ptr(), 1, 1, 128, 128, 64, 0.125, 0,
                            _lib.FA_BF16, s)
    assert st == _lib.FA_ERR_WORKSPACE
