"""Sequence-sharded sparse decode (one context split across ranks by page ranges).

GPU: S shards of one workload run on one device, each in its own host thread
with its own library calls; the collectives are done on the host between
launches (synchronise, exchange, barrier), so no kernel ever waits on another.
The result must be what one device computes: the same selection, the same
tau to the bit, the output within fp32 summation order.

CPU (gloo, world size 2): the same ``sharded_step`` protocol over
torch.distributed, with a shard backend written from the oracle and numpy, so
the host logic (collective order, score layout, page offsets) is checked
without a GPU; the result must equal the oracle's one-device sparse decode.
"""
import datetime
import math
import os
import socket
import sys
import threading

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle as orc  # noqa: E402
from sparse_entmax_kv_b200.sharded import TorchComm, gather_scores, shard_pages, sharded_step  # noqa: E402
from sparse_entmax_kv_b200.workloads import CONFIGS, Workload, make_inputs, to_host_u16  # noqa: E402

SMALL = {
    "gauss_small": CONFIGS["gauss_gqa_L1m"].shrink(name="gauss_small", B=2, Hq=8, Hkv=2, L=32768,
                                                   ragged=True, needles=16),
    "topk_small": CONFIGS["topk_gqa_L128k"].shrink(name="topk_small", B=2, Hq=8, Hkv=2, L=8192,
                                                   ragged=True, needles=8),
    "mha_small": CONFIGS["sweep_mha_L64k"].shrink(name="mha_small", B=3, Hq=4, Hkv=4, L=2048,
                                                  ragged=True, needles=4),
    # 320 groups: each q.K CTA builds its group's union of selected pages
    "groups320": Workload("groups320", B=40, Hq=16, Hkv=8, d=128, L=1500, P=32, alpha=1.5, policy="topk",
                          k=12, keys="offset", needles=3, ragged=True),
}


class ThreadComm:
    """Collectives among S host threads driving one device."""

    def __init__(self, shared, rank):
        self.s, self.rank = shared, rank
        self.world = len(shared["slots"])

    def _exchange(self, t):
        if t.is_cuda:
            torch.cuda.synchronize()
        self.s["slots"][self.rank] = t.clone()
        self.s["barrier"].wait()
        parts = list(self.s["slots"])
        self.s["barrier"].wait()
        return parts

    def all_gather(self, t):
        return torch.stack(self._exchange(t))

    def all_reduce_max(self, t):
        return torch.stack(self._exchange(t)).amax(0)

    def all_reduce_sum(self, t):
        parts = self._exchange(t)
        acc = parts[0].clone()
        for p in parts[1:]:
            acc += p
        return acc


_BARRIERS = []


def _run_threads(fns):
    out, err = [None] * len(fns), []

    def wrap(i, f):
        try:
            out[i] = f()
        except BaseException as e:  # surfaced below
            err.append(e)
            shared_barriers = [getattr(x, "abort", None) for x in _BARRIERS]
            for ab in shared_barriers:
                if ab:
                    ab()

    th = [threading.Thread(target=wrap, args=(i, f), daemon=True) for i, f in enumerate(fns)]
    for t in th:
        t.start()
    for t in th:
        t.join(120)
    if err:
        raise err[0]
    assert not any(t.is_alive() for t in th), "a shard thread did not finish"
    return out


# ------------------------------------------------------------------- GPU

@pytest.mark.gpu
@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("S", [2, 3])
def test_sequence_sharded_matches_one_device(name, S):
    from sparse_entmax_kv_b200 import native as nv
    from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder
    from sparse_entmax_kv_b200.sharded import NativeShard, split_context
    wl = SMALL[name]
    inp = make_inputs(wl, 31, device="cuda")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=wl.policy, k=wl.k or 64, delta=wl.delta or 0.5)
    dec.build_meta()
    nv.get_status(clear=True)
    dec.step(inp["q"])
    torch.cuda.synchronize()
    ref_out, ref_tau = dec.out.clone(), dec.tau.clone()
    ref_sel, ref_cnt = dec.sel.clone(), dec.cnt.clone()
    shards = []
    for r in range(S):
        pt, sl, p0 = split_context(inp["page_table"], inp["seq_lens"], wl.P, S, r)
        sh = NativeShard(inp["k_cache"], inp["v_cache"], pt, sl, inp["seq_lens"], wl.Hq, p0, wl.max_pages,
                         alpha=wl.alpha, policy=wl.policy, k=wl.k or 64, delta=wl.delta or 0.5, cap=4096)
        sh.build_meta()
        shards.append(sh)
    # a failing thread breaks the barrier (BrokenBarrierError in the others)
    # instead of leaving them waiting
    shared = {"slots": [None] * S, "barrier": threading.Barrier(S, timeout=60)}
    _BARRIERS[:] = [shared["barrier"]]
    outs = _run_threads([lambda r=r: sharded_step(shards[r], ThreadComm(shared, r), inp["q"]) for r in range(S)])
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) == 0
    for r in range(S):
        # the same global selection on every rank as on one device
        assert torch.equal(shards[r].cnt, ref_cnt)
        for b in range(wl.B):
            for h in range(wl.Hq):
                n = int(ref_cnt[b, h])
                assert torch.equal(shards[r].sel[b, h, :n], ref_sel[b, h, :n])
        # the same tau to the bit (same candidate list, same order, same solve)
        assert torch.equal(shards[r].tau.view(torch.int32), ref_tau.view(torch.int32))
        torch.testing.assert_close(outs[r], ref_out, rtol=1e-5, atol=1e-6)
        assert torch.equal(outs[r], outs[0])
    # and against the oracle: its decode of the global selection, every head
    host = dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                page_table=inp["page_table"].cpu().numpy(), seq_lens=inp["seq_lens"].cpu().numpy())
    sel, cnt = ref_sel.cpu().numpy(), ref_cnt.cpu().numpy()
    o, otau, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                               wl.P, wl.alpha, sel=sel, cnt=cnt)
    _assert_oracle_close(outs[0].cpu().numpy(), o, shards[0].tau.cpu().numpy(), otau, f"{name} S={S}")


def _assert_oracle_close(out, o, tau, otau, what):
    """Output within max abs 2e-3 and relative L2 1e-3 of the oracle's, tau
    within 2e-5 max(1, |tau|); heads with no selected token (NaN tau, zero
    output) must be so on both sides."""
    out, o = np.asarray(out, np.float64), np.asarray(o, np.float64)
    err = np.abs(out - o).max()
    rel = np.linalg.norm(out - o) / max(np.linalg.norm(o), 1e-30)
    assert err <= 2e-3 and rel <= 1e-3, f"{what}: max abs {err:.3e}, rel L2 {rel:.3e}"
    none = np.isnan(tau)
    assert np.array_equal(none, np.isnan(otau)) or np.all(~np.isfinite(otau[none]))
    ok = ~none
    assert np.all(np.abs(tau[ok] - otau[ok]) <= 2e-5 * np.maximum(1.0, np.abs(otau[ok]))), f"{what}: tau"


@pytest.mark.gpu
def test_sequence_sharded_candidate_cap_overflow():
    """The candidates phase with a cap smaller than a head's candidate list:
    the count stays exact, the first cap candidates are written in list
    order, and STATUS_OVERFLOW is set."""
    from sparse_entmax_kv_b200 import native as nv
    from sparse_entmax_kv_b200.sharded import NativeShard, split_context
    wl = Workload("capped", B=1, Hq=2, Hkv=1, d=64, L=64 * 40, P=64, alpha=2.0, policy="topk", k=40,
                  keys="offset", needles=0)
    inp = make_inputs(wl, 33, device="cuda")
    inp["k_cache"][:] = inp["k_cache"][0, 0, 0]  # equal keys: every selected token is a candidate
    pt, sl, p0 = split_context(inp["page_table"], inp["seq_lens"], wl.P, 1, 0)
    cap = 100
    sh = NativeShard(inp["k_cache"], inp["v_cache"], pt, sl, inp["seq_lens"], wl.Hq, p0, wl.max_pages,
                     alpha=wl.alpha, policy="topk", k=wl.k, cap=cap)
    sh.build_meta()
    nv.get_status(clear=True)
    sh.select(*sh.score(inp["q"]))
    zmax = sh.begin(inp["q"]).clone()
    cz, cn = sh.candidates(inp["q"], zmax)
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) & nv.STATUS_OVERFLOW
    host = dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                page_table=inp["page_table"].cpu().numpy(), seq_lens=inp["seq_lens"].cpu().numpy())
    sel, cnt = sh.sel.cpu().numpy(), sh.cnt.cpu().numpy()
    _, _, _, zz = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv, wl.P,
                             wl.alpha, sel=sel, cnt=cnt, want_z=True)
    cn, cz = cn.cpu().numpy(), cz.cpu().numpy()
    for h in range(wl.Hq):
        z = zz[0, h]
        zl = np.concatenate([z[p * wl.P:(p + 1) * wl.P] for p in sel[0, h, :cnt[0, h]]])  # list order
        zm = float(zmax[0, h])
        assert abs(zm - zl.max()) <= 1e-5 * max(1.0, abs(zl.max()))
        want = zl[zl > zm - 1.0]
        assert int(cn[0, h]) == want.size == cnt[0, h] * wl.P > cap
        np.testing.assert_allclose(cz[0, h, :cap], want[:cap], rtol=0, atol=1e-5)


@pytest.mark.gpu
def test_sequence_sharded_full_size_1m_tokens():
    """The 1M-token Gaussian workload split across two shards (host threads
    on one device): the same selection and tau as one device, the output
    within fp32 summation order."""
    from sparse_entmax_kv_b200 import native as nv
    from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder
    from sparse_entmax_kv_b200.sharded import NativeShard, split_context
    wl = CONFIGS["gauss_gqa_L1m"]
    inp = make_inputs(wl, 32, device="cuda")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=wl.policy, delta=wl.delta)
    dec.build_meta()
    nv.get_status(clear=True)
    dec.step(inp["q"])
    torch.cuda.synchronize()
    ref_out, ref_tau, ref_cnt = dec.out.clone(), dec.tau.clone(), dec.cnt.clone()
    del dec
    S = 2
    shards = []
    for r in range(S):
        pt, sl, p0 = split_context(inp["page_table"], inp["seq_lens"], wl.P, S, r)
        sh = NativeShard(inp["k_cache"], inp["v_cache"], pt, sl, inp["seq_lens"], wl.Hq, p0, wl.max_pages,
                         alpha=wl.alpha, policy=wl.policy, delta=wl.delta, cap=8192)
        sh.build_meta()
        shards.append(sh)
    shared = {"slots": [None] * S, "barrier": threading.Barrier(S, timeout=60)}
    _BARRIERS[:] = [shared["barrier"]]
    outs = _run_threads([lambda r=r: sharded_step(shards[r], ThreadComm(shared, r), inp["q"]) for r in range(S)])
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0
    for r in range(S):
        assert torch.equal(shards[r].cnt, ref_cnt)
        assert torch.equal(shards[r].tau.view(torch.int32), ref_tau.view(torch.int32))
        torch.testing.assert_close(outs[r], ref_out, rtol=1e-5, atol=1e-6)
    # sampled (sequence, kv head) groups against the oracle's decode of the
    # selection every rank holds
    from tests.helpers import sub_problem
    G = wl.G
    sel = shards[0].sel.cpu().numpy()
    cnt = shards[0].cnt.cpu().numpy()
    for kvh in (0, wl.Hkv - 1):
        sp = sub_problem(inp, wl, 0, kvh)
        hs = slice(kvh * G, (kvh + 1) * G)
        o, otau, _, _ = orc.decode(sp["q"], sp["K"], sp["V"], sp["page_table"], sp["seq_lens"], 1, wl.P, wl.alpha,
                                   sel=sel[0:1, hs, :sp["npb"]], cnt=cnt[0:1, hs])
        _assert_oracle_close(outs[0][0, hs].cpu().numpy(), o[0], shards[0].tau[0, hs].cpu().numpy(), otau[0],
                             f"1M kvh{kvh}")


# ------------------------------------------------------------------- CPU

class OracleShard:
    """One rank's shard on the host: every phase from the oracle and numpy."""

    def __init__(self, wl, host, S, rank):
        self.wl, self.S, self.rank = wl, S, rank
        self.M, begins = shard_pages(wl.max_pages, S)
        self.p0 = begins[rank]
        self.max_pages_global = wl.max_pages
        self.cap = 4096
        B, P = wl.B, wl.P
        pt = np.full((B, self.M), -1, np.int32)
        w = max(0, min(self.M, wl.max_pages - self.p0))
        pt[:, :w] = host["page_table"][:, self.p0:self.p0 + w]
        self.pt = pt
        self.seq = np.clip(host["seq_lens"].astype(np.int64) - self.p0 * P, 0, self.M * P).astype(np.int32)
        self.seq_g = host["seq_lens"]
        self.host = host
        self.meta = orc.build_meta(host["K"], pt, self.seq, wl.Hkv, wl.d, P, wl.num_blocks)

    def score(self, q):
        bb, mu, sg = orc.score_pages(self.host["q"], self.meta, self.pt, self.seq, self.wl.Hkv, self.wl.P)
        bb, mu, sg = (np.nan_to_num(x, nan=0.0) for x in (bb, mu, sg))
        if self.wl.policy == "topk":
            return torch.from_numpy(bb), None, None
        return torch.from_numpy(bb), torch.from_numpy(mu), torch.from_numpy(sg)

    def select(self, bbox, mu, sigma):
        wl = self.wl
        self.sel, self.cnt, _ = orc.select(self.seq_g, bbox.numpy(), None if mu is None else mu.numpy(),
                                           None if sigma is None else sigma.numpy(), wl.P, wl.policy,
                                           wl.k or 64, wl.alpha, wl.delta or 0.5)

    def begin(self, q):
        # z of this shard's selected tokens (oracle, local page ids), and its max
        wl = self.wl
        B, Hq = wl.B, wl.Hq
        sel_l = np.full_like(self.sel, -1)
        cnt_l = np.zeros_like(self.cnt)
        for b in range(B):
            for h in range(Hq):
                mine = [p - self.p0 for p in self.sel[b, h, :self.cnt[b, h]] if self.p0 <= p < self.p0 + self.M]
                cnt_l[b, h] = len(mine)
                sel_l[b, h, :len(mine)] = mine
        self.sel_l, self.cnt_l = sel_l[:, :, :self.M].copy(), cnt_l
        _, _, _, zz = orc.decode(self.host["q"], self.host["K"], self.host["V"], self.pt, self.seq, wl.Hkv, wl.P,
                                 wl.alpha, sel=self.sel_l, cnt=self.cnt_l, want_z=True)
        self.z = zz  # [B][Hq][M*P], -inf off the selection
        return torch.from_numpy(zz.max(axis=2) if zz.shape[2] else np.full((B, Hq), -np.inf))

    def candidates(self, q, zmax):
        B, Hq = self.wl.B, self.wl.Hq
        cz = np.zeros((B, Hq, self.cap))
        cn = np.zeros((B, Hq), np.int64)
        for b in range(B):
            for h in range(Hq):
                # list order: ascending page, then token
                c = []
                for p in self.sel_l[b, h, :self.cnt_l[b, h]]:
                    zp = self.z[b, h, p * self.wl.P:(p + 1) * self.wl.P]
                    c.extend(float(v) for v in zp if v > float(zmax[b, h]) - 1.0)
                cn[b, h] = len(c)
                cz[b, h, :len(c)] = c
        return torch.from_numpy(cz), torch.from_numpy(cn)

    def threshold(self, cz_all, cn_all, zmax):
        B, Hq = self.wl.B, self.wl.Hq
        tau = np.full((B, Hq), np.nan)
        for b in range(B):
            for h in range(Hq):
                c = np.concatenate([cz_all[s, b, h, :int(cn_all[s, b, h])].numpy() for s in range(self.S)])
                if len(c):
                    tau[b, h] = orc.entmax_tau(c, self.wl.alpha)
        return torch.from_numpy(tau)

    def finish(self, q, zmax, tau):
        wl = self.wl
        r = 1.0 / (wl.alpha - 1.0)
        out = np.zeros((wl.B, wl.Hq, wl.d))
        V = self.host["V"]
        for b in range(wl.B):
            for h in range(wl.Hq):
                t = float(tau[b, h])
                if not math.isfinite(t):
                    continue
                for p in self.sel_l[b, h, :self.cnt_l[b, h]]:
                    blk = self.pt[b, p]
                    for i in range(wl.P):
                        z = self.z[b, h, p * wl.P + i]
                        if z > t:
                            v = (V[blk, h // wl.G, i].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                            out[b, h] += (z - t) ** r * v
        return torch.from_numpy(out)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, name, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        wl = SMALL_CPU[name]
        inp = make_inputs(wl, 41, device="cpu")
        host = dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                    page_table=inp["page_table"].numpy(), seq_lens=inp["seq_lens"].numpy())
        shard = OracleShard(wl, host, world, rank)
        o = sharded_step(shard, TorchComm(), None)
        out.put((rank, o.numpy(), shard.sel, shard.cnt))
    finally:
        dist.destroy_process_group()


SMALL_CPU = {
    "gauss_tiny": Workload("gauss_tiny", B=2, Hq=4, Hkv=2, d=64, L=1200, P=16, alpha=1.5, policy="gauss",
                           delta=0.5, keys="cluster", needles=3, ragged=True),
    "topk_tiny": Workload("topk_tiny", B=1, Hq=2, Hkv=1, d=64, L=900, P=16, alpha=1.5, policy="topk", k=12,
                          keys="offset", needles=2, ragged=True),
}


@pytest.mark.parametrize("name", list(SMALL_CPU))
def test_sequence_sharded_protocol_on_two_gloo_ranks(name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, 2, port, name, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (o, s, c)) for r, o, s, c in (q.get(timeout=300) for _ in procs))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    wl = SMALL_CPU[name]
    inp = make_inputs(wl, 41, device="cpu")
    host = dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                page_table=inp["page_table"].numpy(), seq_lens=inp["seq_lens"].numpy())
    meta = orc.build_meta(host["K"], host["page_table"], host["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    bb, mu, sg = orc.score_pages(host["q"], meta, host["page_table"], host["seq_lens"], wl.Hkv, wl.P)
    sel, cnt, _ = orc.select(host["seq_lens"], bb, mu, sg, wl.P, wl.policy, wl.k or 64, wl.alpha,
                             wl.delta or 0.5)
    o_ref, _, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                                wl.P, wl.alpha, sel=sel, cnt=cnt)
    for r in range(2):
        o, s, c = res[r]
        np.testing.assert_array_equal(c, cnt)
        for b in range(wl.B):
            for h in range(wl.Hq):
                np.testing.assert_array_equal(s[b, h, :cnt[b, h]], sel[b, h, :cnt[b, h]])
        np.testing.assert_allclose(o, o_ref, rtol=1e-9, atol=1e-12)
    np.testing.assert_array_equal(res[0][0], res[1][0])


def test_gather_scores_puts_each_rank_at_its_page_offset():
    class Stack:
        def all_gather(self, t):
            return torch.stack([t, t + 100])
    x = torch.arange(2 * 3 * 4, dtype=torch.float32).reshape(2, 3, 4)  # [B][Hq][M]
    g = gather_scores(Stack(), x, 7)
    assert g.shape == (2, 3, 7)
    assert torch.equal(g[:, :, :4], x)
    assert torch.equal(g[:, :, 4:], (x + 100)[:, :, :3])
