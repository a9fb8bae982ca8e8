"""Failure detection on the GPU, with no GPU fault: every failure is made on
the host (a bad length, a non-finite query) or is a bounded wait that nothing
ends.  Each case checks the documented status bit and output contract of
include/entmaxkv.h, and that the context stays usable afterwards.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from sparse_entmax_kv_b200 import native as nv
from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder
from sparse_entmax_kv_b200.workloads import CONFIGS, Workload, make_inputs, to_host_u16

pytestmark = pytest.mark.gpu

OUT_ABS, OUT_REL = 2e-3, 1e-3


def _host(inp):
    return dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                page_table=inp["page_table"].cpu().numpy(), seq_lens=inp["seq_lens"].cpu().numpy())


def _close(got, want, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err <= OUT_ABS and rel <= OUT_REL, f"{what}: max abs {err:.3e}, rel L2 {rel:.3e}"


def test_bounded_wait_runs_out_and_reports_timeout():
    """A wait on an mbarrier that nothing arrives at returns after its limit
    (1 ms here), sets STATUS_TIMEOUT, and leaves the stream usable."""
    nv.get_status(clear=True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    nv.entmaxkv_selftest_wait(1_000_000)
    ev1.record()
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) == nv.STATUS_TIMEOUT
    assert ev0.elapsed_time(ev1) >= 0.9  # ms: it did wait out its limit
    # the context still runs work: a small decode step after the timed-out wait
    wl = CONFIGS["tiny_h1_L4k"].shrink(L=1024)
    inp = make_inputs(wl, 3, device="cuda")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy="topk", k=wl.k)
    dec.build_meta()
    dec.step(inp["q"])
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) == 0
    assert torch.isfinite(dec.out).all()
    with pytest.raises(nv.EntmaxKVError):
        nv.entmaxkv_selftest_wait(0)
    with pytest.raises(nv.EntmaxKVError):
        nv.entmaxkv_selftest_wait(3_000_000_000)


NONFINITE = {
    "gqa_topk": Workload("nf_topk", B=2, Hq=8, Hkv=2, d=128, L=3000, P=32, alpha=1.5, policy="topk", k=16,
                         keys="offset", needles=3, ragged=True),
    "gqa_gauss": Workload("nf_gauss", B=2, Hq=8, Hkv=2, d=64, L=2500, P=16, alpha=2.0, policy="gauss",
                          delta=0.5, keys="cluster", needles=3, ragged=True),
}


@pytest.mark.parametrize("name", list(NONFINITE))
def test_nonfinite_query_gives_nan_head_and_status(name):
    """A query row holding NaN (head (0, 1)) or +Inf (head (1, 6)): that head's
    page scores, sparse and dense outputs and tau are NaN, STATUS_NONFINITE is
    set, and every other head still matches the oracle."""
    wl = NONFINITE[name]
    inp = make_inputs(wl, 17, device="cuda")
    host = _host(inp)  # the clean queries, for the oracle
    bad = [(0, 1), (1, 6)]
    q = inp["q"].clone()
    q[0, 1, 5] = float("nan")
    q[1, 6, wl.d - 1] = float("inf")
    good = np.ones((wl.B, wl.Hq), bool)
    for b, h in bad:
        good[b, h] = False
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=wl.policy, k=wl.k or 16, delta=wl.delta or 0.5)
    dec.build_meta()
    nv.get_status(clear=True)
    dec.step(q)
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) & nv.STATUS_NONFINITE
    for b, h in bad:
        npb = -(-int(host["seq_lens"][b]) // wl.P)
        assert torch.isnan(dec.bbox[b, h, :npb]).all()
        if dec.mu is not None:
            assert torch.isnan(dec.mu[b, h, :npb]).all() and torch.isnan(dec.sigma[b, h, :npb]).all()
        assert torch.isnan(dec.out[b, h]).all()
        assert math.isnan(float(dec.tau[b, h]))
    # the other heads: the oracle's selection and output
    meta = orc.build_meta(host["K"], host["page_table"], host["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    bb, mu, sg = orc.score_pages(host["q"], meta, host["page_table"], host["seq_lens"], wl.Hkv, wl.P)
    osel, ocnt, _ = orc.select(host["seq_lens"], bb, mu, sg, wl.P, wl.policy, wl.k or 16, wl.alpha,
                               wl.delta or 0.5)
    gsel, gcnt = dec.sel.cpu().numpy(), dec.cnt.cpu().numpy()
    o, otau, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                               wl.P, wl.alpha, sel=gsel, cnt=gcnt)
    gout = dec.out.cpu().numpy()
    _close(gout[good], o[good], f"{name} finite heads")
    if wl.policy == "topk":
        for b in range(wl.B):
            for h in range(wl.Hq):
                if good[b, h]:
                    assert np.array_equal(gsel[b, h, :gcnt[b, h]], osel[b, h, :ocnt[b, h]])
    # full-cache paths: NaN for the bad heads, the oracle elsewhere
    s = dec.shape
    ws = nv.alloc_workspace(s, nv.CALL_DECODE_DENSE, "cuda")
    for alpha in (wl.alpha, 1.0):
        out = torch.empty((wl.B, wl.Hq, wl.d), device="cuda")
        tau = torch.empty((wl.B, wl.Hq), device="cuda")
        nv.get_status(clear=True)
        nv.entmaxkv_decode_dense(s, q, inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                                 alpha, out, tau, None, ws)
        torch.cuda.synchronize()
        assert nv.get_status(clear=True) & nv.STATUS_NONFINITE
        od, _, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                                 wl.P, alpha)
        out, tau = out.cpu().numpy(), tau.cpu().numpy()
        for b, h in bad:
            assert np.isnan(out[b, h]).all() and math.isnan(tau[b, h]), f"dense alpha={alpha}"
        _close(out[good], od[good], f"{name} dense alpha={alpha}")


def test_sequence_longer_than_page_table_is_clamped_and_reported():
    """seq_lens[b] above max_pages * P: every kernel treats the sequence as
    max_pages * P tokens long (no read or write past a row of max_pages
    pages) and sets STATUS_BAD_LENGTH; append skips the sequence."""
    wl = Workload("overlong", B=2, Hq=4, Hkv=2, d=64, L=1024, P=16, alpha=1.5, policy="gauss", delta=0.5,
                  keys="offset", needles=2)
    inp = make_inputs(wl, 19, device="cuda")
    cap = wl.max_pages * wl.P
    long_lens = inp["seq_lens"].clone()
    long_lens[1] = cap + 100
    s = nv.Shape(wl.B, wl.Hq, wl.Hkv, wl.d, wl.P, wl.max_pages, wl.num_blocks)
    outs = {}
    for tag, lens in (("clamped", inp["seq_lens"]), ("long", long_lens)):
        # the score rows sit inside a larger buffer whose tail must stay untouched
        n = wl.B * wl.Hq * wl.max_pages
        bufs = [torch.full((n + 4096,), float("nan"), device="cuda") for _ in range(3)]
        bbox, mu, sig = (x[:n].view(wl.B, wl.Hq, wl.max_pages) for x in bufs)
        sel = torch.full((n + 4096,), -7, dtype=torch.int32, device="cuda")
        cnt = torch.zeros((wl.B, wl.Hq), dtype=torch.int32, device="cuda")
        meta = nv.alloc_meta(s, "cuda")
        nv.get_status(clear=True)
        nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], lens, 0, -1, meta)
        nv.entmaxkv_score_pages(s, inp["q"], meta, lens, bbox, mu, sig)
        nv.entmaxkv_select(s, lens, bbox, mu, sig, nv.GAUSS, 0, wl.alpha, wl.delta,
                           sel[:n].view(wl.B, wl.Hq, wl.max_pages), cnt, None)
        out = torch.empty((wl.B, wl.Hq, wl.d), device="cuda")
        ws = nv.alloc_workspace(s, nv.CALL_DECODE_SPARSE, "cuda")
        nv.entmaxkv_decode_sparse(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], lens,
                                  sel[:n].view(wl.B, wl.Hq, wl.max_pages), cnt, wl.alpha, out, None, None, ws)
        torch.cuda.synchronize()
        st = nv.get_status(clear=True)
        if tag == "long":
            assert st & nv.STATUS_BAD_LENGTH
        else:
            assert st == 0
        for x in bufs:
            assert torch.isnan(x[n:]).all()
        assert (sel[n:] == -7).all()
        outs[tag] = (bbox.clone(), cnt.clone(), out.clone())
    # treated exactly as a max_pages * P long sequence
    for a, b in zip(outs["clamped"], outs["long"]):
        assert torch.equal(a, b)
    # append: the over-long sequence is skipped, the other is written
    k_new = torch.full((wl.B, wl.Hkv, wl.d), 1.5, dtype=torch.bfloat16, device="cuda")
    v_new = torch.full((wl.B, wl.Hkv, wl.d), -2.5, dtype=torch.bfloat16, device="cuda")
    k_before = inp["k_cache"].clone()
    meta = nv.alloc_meta(s, "cuda")
    nv.get_status(clear=True)
    nv.entmaxkv_append(s, k_new, v_new, inp["page_table"], long_lens, inp["k_cache"], inp["v_cache"], meta)
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) & nv.STATUS_BAD_LENGTH
    L0 = int(long_lens[0])
    blk0 = int(inp["page_table"][0, (L0 - 1) // wl.P])
    assert (inp["k_cache"][blk0, :, (L0 - 1) % wl.P] == 1.5).all()
    changed = (inp["k_cache"] != k_before).any(dim=-1)  # [blocks][Hkv][P]
    assert int(changed.sum()) == wl.Hkv  # only sequence 0's slot, every kv head
