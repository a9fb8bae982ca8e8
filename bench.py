"""Benchmark of one EntmaxKV sparse alpha-entmax decode step on B200.

A step is the whole hot path for one batch: append each sequence's newest
token (its key/value rows written to its slot and its page's metadata rebuilt,
entmaxkv_append), score every page (entmaxkv_score_pages), select
(entmaxkv_select, top-k or Gaussian tau_hat - Delta) and decode over the
selected pages (entmaxkv_decode_sparse).
Default workload: B=1, Hq=32, Hkv=8, d=128, 1,048,576-token context, 64-token
pages, alpha=1.5, Gaussian selection with Delta=0.5 (the long-context setting of
the EntmaxKV efficiency study), synthetic clustered keys with 64 needles per
head.  Inputs live in HBM before timing; before every step, outside the
per-step CUDA events, L2 is flushed: a 256 MiB buffer is written, then a
second 256 MiB buffer is read, so the step starts with none of its data in L2
and no dirty lines of the flush left to write back while it runs.

Reported value: effective KV bandwidth = bytes the step must touch (metadata
scanned by scoring + K tiles of the selected pages + value rows with non-zero
weight) / device time per step, summed over all ranks (one independent
problem per GPU, weak scaling, no data-path collective).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse α-entmax decode µs/step & KV GB/s vs HBM roofline at 1M ctx"
PAPER_CONTEXT = {"speedup_vs_full_softmax_flashdecoding": 3.36, "speedup_vs_full_entmax": 5.43,
                 "context_tokens": 1048576, "hardware": "not stated on the pages",
                 "source": "EntmaxKV summary, section 4 (Efficiency)"}

# DRAM bytes per launch from ncu captures (dram__bytes_read.sum + dram__bytes_write.sum),
# keyed by kernel and workload, valid only while the kernel source is unchanged
# (the source hash below); the line reports null traffic once it has changed.
NCU_TRAFFIC = {
    # one full-size launch at L=1,048,576 (201.36 MB read + 5.46 MB written), ncu --metrics
    # dram__bytes_read.sum,dram__bytes_write.sum on the score-only profile run
    "score_pages/gauss_gqa_L1m": {"bytes": 201361920 + 5464064, "src": "61c13daf6d60"},
}


def max_over_ranks(vals, world, device):
    """Each value's maximum over all ranks (the slowest rank's device time)."""
    if world == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def whole_job_gbs(bytes_per_rank, world, step_ms):
    """Whole-job throughput: every rank moves bytes_per_rank per step (weak
    scaling, one independent problem per rank), timed by the slowest rank."""
    return world * bytes_per_rank / (step_ms * 1e-3) / 1e9


def _src_hash(fname):
    """Hash of a kernel source together with the shared device helpers it includes."""
    h = hashlib.sha1()
    for f in (fname, "common.cuh"):
        h.update(open(os.path.join(ROOT, "sparse_entmax_kv_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:12]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    def __init__(self, index, directory=None):
        self.proc = None
        self.path = os.path.join(directory or tempfile.gettempdir(), f"entmaxkv_clocks_rank{index}.csv")
        self.index = index

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "window": "loaded steps bracketing the timed region (>= 1 s before, >= 0.5 s after)"}


# ------------------------------------------------------------ byte model

def step_bytes(wl, dec, support_rows):
    """Algorithmic bytes of one step.  meta: records scanned by scoring;
    gather_k: K tiles of each GQA group's union of selected pages; gather_v:
    value rows with non-zero weight for some head of the group."""
    seq = dec.seq_lens.cpu().numpy()
    npb = -(-seq // wl.P)
    rec_bytes = (12 if wl.policy in ("gauss", "gauss_est") else 4) * wl.d
    meta = int(npb.sum()) * wl.Hkv * rec_bytes
    sel, cnt = dec.sel.cpu().numpy(), dec.cnt.cpu().numpy()
    union = 0
    for b in range(wl.B):
        for kvh in range(wl.Hkv):
            s = set()
            for g in range(wl.G):
                h = kvh * wl.G + g
                s.update(sel[b, h, :cnt[b, h]].tolist())
            union += len(s)
    gather_k = union * wl.P * wl.d * 2
    gather_v = support_rows * wl.d * 2
    scores = wl.B * wl.Hq * int(npb.max()) * (12 if wl.policy == "gauss" else 4)
    qo = wl.B * wl.Hq * wl.d * (2 + 4)
    return dict(meta=meta, gather_k=gather_k, gather_v=gather_v, scores=scores, qo=qo,
                kv_touched=meta + gather_k + gather_v, union_pages=union, support_rows=support_rows)


def support_rows_of(wl, p_out):
    """Distinct (sequence, kv head, token) rows with p > 0 for some head of the group."""
    pz = (p_out > 0).view(wl.B, wl.Hkv, wl.G, -1).any(dim=2)
    return int(pz.sum().item())


# ------------------------------------------------------------- GPU arm

def run_gpu(args, rank, world):
    from sparse_entmax_kv_b200 import native as nv
    from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder, last_token_rows
    from sparse_entmax_kv_b200.workloads import CONFIGS, make_inputs

    wl = CONFIGS[args.workload]
    policy = wl.policy if wl.policy != "dense" else "topk"
    k = wl.k or 64
    delta = wl.delta or 0.5
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_inputs(wl, 1000 * 4 + rank, device=dev, sequential_pages=args.page_table == "sequential")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=policy, k=k, delta=delta, fused=not args.unfused)
    dec.build_meta()
    # each sequence's newest token (position seq_len-1) is appended again every
    # step: its key/value rows are written to their slot and its page's
    # metadata is rebuilt, leaving the cache as it was
    L0 = int(inp["seq_lens"][0])
    k_new, v_new = last_token_rows(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"])
    new_kv = (k_new, v_new)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(32 << 20, dtype=torch.int64, device=dev)


    def l2_flush():
        flush_w.fill_(1)
        torch.amax(flush_r)

    q = inp["q"]
    st = torch.cuda.current_stream()

    # byte model from one untimed step with p written out
    p_out = torch.zeros((wl.B, wl.Hq, wl.max_pages * wl.P), device=dev)
    dec.step(q, p_out=p_out, new_kv=new_kv)
    torch.cuda.synchronize()
    nbytes = step_bytes(wl, dec, support_rows_of(wl, p_out))
    del p_out
    torch.cuda.empty_cache()

    nst = 4
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(args.steps)]

    # One step (the four C-ABI calls) captured as a CUDA graph: the timed
    # region replays it, so host launch latency does not enter the device time.
    dec.step(q, new_kv=new_kv)  # eager first call: per-device set-up happens outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        dec.step(q, new_kv=new_kv)
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(graph):
        dec.step(q, new_kv=new_kv)
    torch.cuda.synchronize()
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    # The timed region lasts milliseconds, far below nvidia-smi's sampling
    # period, so clocks are sampled over a loaded window that brackets it:
    # warm-up steps for >= 1 s before, untimed steps for >= 0.5 s after.
    with ClockSampler(dev.index, args.clocks_dir) as clk:
        t0 = time.perf_counter()
        i = 0
        while i < args.warmup or time.perf_counter() - t0 < 1.0:
            l2_flush()
            graph.replay()
            if i % 16 == 15:
                torch.cuda.synchronize()
            i += 1
        torch.cuda.synchronize()
        assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t_wall = time.perf_counter()
        for i in range(args.steps):
            l2_flush()  # L2 flush, outside the step's events
            gev[i][0].record(st)
            graph.replay()
            gev[i][1].record(st)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        t_wall = time.perf_counter() - t_wall

        # per-stage device times: the same step issued call by call, each call
        # bracketed by events (the 256 MiB flush before each step keeps the
        # host ahead of the GPU, so the events see kernel time, not host gaps)
        for i in range(args.steps):
            l2_flush()
            e = ev[i]
            e[0].record(st)
            nv.entmaxkv_append(dec.shape, k_new, v_new, dec.page_table, dec.seq_lens, dec.k_cache, dec.v_cache,
                               dec.meta)
            e[1].record(st)
            nv.entmaxkv_score_pages(dec.shape, q, dec.meta, dec.seq_lens, dec.bbox, dec.mu,
                                    dec.sigma)
            e[2].record(st)
            nv.entmaxkv_select(dec.shape, dec.seq_lens, dec.bbox, dec.mu, dec.sigma, dec.policy, dec.k, dec.alpha,
                               dec.delta, dec.sel, dec.cnt, dec.tau_hat)
            e[3].record(st)
            nv.entmaxkv_decode_sparse(dec.shape, q, dec.k_cache, dec.v_cache, dec.page_table, dec.seq_lens,
                                      dec.sel, dec.cnt, dec.alpha, dec.out, dec.tau, None, dec.ws)
            e[4].record(st)
        torch.cuda.synchronize()
        # the fused call of the product step (scores, selection with the
        # union, q.K, tau with p.V), eagerly, after the same flush
        fev = []
        if dec.fused:
            for i in range(args.steps):
                l2_flush()
                fev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
                fev[-1][0].record(st)
                nv.entmaxkv_decode_step(dec.shape, q, dec.meta, dec.k_cache, dec.v_cache, dec.page_table,
                                        dec.seq_lens, dec.policy, dec.k, dec.alpha, dec.delta, dec.bbox, dec.mu,
                                        dec.sigma, dec.sel, dec.cnt, dec.out, dec.tau_hat, dec.tau, None, dec.ws)
                fev[-1][1].record(st)
            torch.cuda.synchronize()
        t1 = time.perf_counter()
        while time.perf_counter() - t1 < 0.5:
            for _ in range(16):
                l2_flush()
                graph.replay()
            torch.cuda.synchronize()
    clocks = clk.summary()
    # the scan kernel's own duration: launches back to back between two events
    # on its stream (each waits for the one before it, so launch latency is
    # hidden); valid without an L2 flush only while the metadata it streams
    # is larger than L2, so each launch reads it from DRAM again
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    scan_b2b_us = None
    if nbytes["meta"] > l2_bytes:
        nb2b = 20
        for _ in range(3):
            nv.entmaxkv_score_pages(dec.shape, q, dec.meta, dec.seq_lens, dec.bbox, dec.mu, dec.sigma)
        l2_flush()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(st)
        for _ in range(nb2b):
            nv.entmaxkv_score_pages(dec.shape, q, dec.meta, dec.seq_lens, dec.bbox, dec.mu, dec.sigma)
        b1.record(st)
        torch.cuda.synchronize()
        scan_b2b_us = b0.elapsed_time(b1) * 1e3 / nb2b
    step_ms = float(np.mean([a.elapsed_time(b) for a, b in gev]))
    stage_ms = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(nst)] for i in range(args.steps)])
    eager_step_ms = float(stage_ms.sum(axis=1).mean())
    step_ms, = max_over_ranks([step_ms], world, dev)
    stage_us = dict(zip(["append", "score_pages", "select", "decode_sparse"],
                        (stage_ms.mean(axis=0) * 1e3).round(2).tolist()))
    if fev:
        stage_us["decode_step"] = round(float(np.mean([a.elapsed_time(b) for a, b in fev])) * 1e3, 2)
    scan_b2b_us, = max_over_ranks([scan_b2b_us if scan_b2b_us is not None else -1.0], world, dev)
    scan_b2b_us = None if scan_b2b_us < 0 else scan_b2b_us

    # comparison paths at the same context: full-cache entmax and softmax
    dense = {}
    if not args.skip_dense:
        out = torch.empty((wl.B, wl.Hq, wl.d), device=dev)
        ws = nv.alloc_workspace(dec.shape, nv.CALL_DECODE_DENSE, dev)
        for alpha, name in ((wl.alpha, "dense_entmax"), (1.0, "dense_softmax")):
            ts = []
            for i in range(3 + args.dense_steps):
                l2_flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(st)
                nv.entmaxkv_decode_dense(dec.shape, q, dec.k_cache, dec.v_cache, dec.page_table, dec.seq_lens,
                                         alpha, out, None, None, ws)
                b.record(st)
                torch.cuda.synchronize()
                if i >= 3:
                    ts.append(a.elapsed_time(b))
            dense[name] = statistics.median(ts) * 1e3
        del ws

    # end to end through the C ABI with host buffers: q and the appended
    # token's k/v rows come from one pinned host buffer each step (one
    # host-to-device copy), the output goes back to host
    n_q, n_kv = q.numel(), k_new.numel()
    stage_host = torch.cat([q.reshape(-1), k_new.reshape(-1), v_new.reshape(-1)]).cpu().pin_memory()
    q_dev = torch.empty_like(q)  # where append stages the queries for the later calls
    out_host = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.float32).pin_memory()

    q_host = stage_host[:n_q].view_as(q)
    k_host = stage_host[n_q:n_q + n_kv].view_as(k_new)
    v_host = stage_host[n_q + n_kv:].view_as(v_new)

    def e2e_once():
        # the append kernel reads q and the new rows from pinned host memory
        # (the host-to-device transfer of the inputs happens inside the step)
        # and the decode writes the output straight into pinned host memory
        dec.step(q_dev, new_kv=(k_host, v_host), out=out_host, q_in=q_host)

    def time_e2e(fn):
        ts = []
        for i in range(args.warmup + args.steps):
            l2_flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            torch.cuda.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(b))
        return float(np.mean(ts))

    e2e_once()
    torch.cuda.synchronize()
    g2 = torch.cuda.CUDAGraph()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        e2e_once()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(g2):
        e2e_once()
    torch.cuda.synchronize()
    e2e_step_ms = time_e2e(g2.replay)
    e2e_eager_ms = time_e2e(e2e_once)
    e2e_step_ms, e2e_eager_ms = max_over_ranks([e2e_step_ms, e2e_eager_ms], world, dev)
    dec.step(q, new_kv=new_kv)
    torch.cuda.synchronize()
    assert torch.equal(out_host, dec.out.cpu()), "end-to-end output differs from the device step's"
    assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0

    peak, peak_kind = measured_peaks()
    # dominant kernel of the step: score_pages is a single launch (the sparse
    # decode stage is three kernels and is reported beside it)
    dom = "score_pages"
    # algorithmic bytes of the scan: the metadata records and the queries; the
    # page scores it writes are reported beside them as actual bytes.  The
    # launch duration is the back-to-back average when the metadata exceeds
    # L2, else the single eager call (which also counts its launch latency).
    alg = nbytes["meta"] + wl.B * wl.Hq * wl.d * 2
    actual = alg + nbytes["scores"]
    dur_us = scan_b2b_us if scan_b2b_us is not None else stage_us[dom]
    achieved = alg / (dur_us * 1e-6) / 1e9
    tr = NCU_TRAFFIC.get(f"{dom}/{args.workload}")
    traffic = tr["bytes"] if tr and tr.get("src") == _src_hash("score.cu") else None  # null once the kernel changed
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "algorithmic_bytes": alg,
                "actual_bytes": actual, "launch_us": round(dur_us, 2),
                "launch_timing": ("average of 20 launches back to back between two CUDA events (metadata %.0f MB > "
                                  "L2 %.0f MB, so every launch streams it from DRAM)" % (nbytes["meta"] / 1e6,
                                                                                          l2_bytes / 1e6)
                                  if scan_b2b_us is not None else
                                  "one eager call between CUDA events after an L2 flush (includes launch latency)"),
                "eager_call_us": stage_us[dom],
                "peak_kind": f"{peak_kind} copy bandwidth (burst)"}
    galg = nbytes["gather_k"] + nbytes["gather_v"] + nbytes["qo"]
    gach = galg / (stage_us["decode_sparse"] * 1e-6) / 1e9
    roofline_gather = {"bound": "hbm", "kernel": "decode_sparse (union, q.K, tau with p.V)",
                       "achieved": round(gach, 1), "peak": peak, "unit": "GB/s", "frac": round(gach / peak, 4),
                       "algorithmic_bytes": galg}
    res = dict(wl=wl, step_ms=step_ms, eager_step_ms=eager_step_ms, e2e_eager_ms=e2e_eager_ms,
               stage_us=stage_us, dense=dense, nbytes=nbytes, clocks=clocks,
               roofline=roofline, roofline_gather=roofline_gather, e2e_ms=e2e_step_ms, e2e_bytes=(stage_host.numel() * 2,
                                                               out_host.numel() * 4),
               launches=dec.kernels_per_step(True) * args.steps, fused=dec.fused, t_wall=t_wall,
               host=dict(inp=inp, dec=dec) if (rank == 0 and not args.no_cpu_baseline) else None)
    return res


# --------------------------------------------------------- CPU oracle arm

def oracle_step_sample(wl, inp_host, seconds_target=10.0, max_reps=3):
    """Time the fp64 oracle on one step of the workload (score + select +
    sparse decode, metadata prepared beforehand), repeated up to max_reps or
    until seconds_target is reached.  Returns (seconds per step, bytes per
    step by the same byte model, threads)."""
    import oracle as orc

    policy = wl.policy if wl.policy != "dense" else "topk"
    h = inp_host
    meta = orc.build_meta(h["K"], h["page_table"], h["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    times = []
    t_end = time.perf_counter() + seconds_target
    for _ in range(max_reps):
        t0 = time.perf_counter()
        bbox, mu, sig = orc.score_pages(h["q"], meta, h["page_table"], h["seq_lens"], wl.Hkv, wl.P)
        sel, cnt, _ = orc.select(h["seq_lens"], bbox, mu, sig, wl.P, policy, wl.k or 64, wl.alpha,
                                 wl.delta or 0.5)
        o, tau, pw, _ = orc.decode(h["q"], h["K"], h["V"], h["page_table"], h["seq_lens"], wl.Hkv, wl.P,
                                   wl.alpha, sel=sel, cnt=cnt, want_p=True)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() > t_end:
            break
    npb = -(-h["seq_lens"] // wl.P)
    meta_b = int(npb.sum()) * wl.Hkv * (12 if policy in ("gauss", "gauss_est") else 4) * wl.d
    union = 0
    supp = 0
    for b in range(wl.B):
        for kvh in range(wl.Hkv):
            s = set()
            rows = None
            for g in range(wl.G):
                hh = kvh * wl.G + g
                s.update(sel[b, hh, :cnt[b, hh]].tolist())
                r = pw[b, hh] > 0
                rows = r if rows is None else (rows | r)
            union += len(s)
            supp += int(rows.sum())
    nbytes = meta_b + union * wl.P * wl.d * 2 + supp * wl.d * 2
    return statistics.median(times), nbytes, orc.num_threads(), len(times)


def host_copy(inp, b0=0, nb=None):
    from sparse_entmax_kv_b200.workloads import to_host_u16
    return dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                page_table=inp["page_table"].cpu().numpy(), seq_lens=inp["seq_lens"].cpu().numpy())


def sample_workload(wl):
    """The bounded oracle sample of a workload: the first sequence, all its
    heads, at the full context (one sequence of the batch)."""
    return wl.shrink(B=1)


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, timed on the host cores, on a
    bounded sample of the same workload (rank 0 only)."""
    from sparse_entmax_kv_b200.workloads import CONFIGS, make_inputs
    if rank != 0:
        return
    wl = CONFIGS[args.workload]
    swl = sample_workload(wl)
    inp = make_inputs(swl, 1000 * 4, device="cpu")
    host = host_copy(inp)
    per = []
    for i in range(args.warmup + args.steps):
        sec, nbytes, thr, reps = oracle_step_sample(swl, host, seconds_target=0.0, max_reps=1)
        if i >= args.warmup:
            per.append(sec)
    sec = statistics.median(per)
    gbs = nbytes / sec / 1e9
    sample = f"{swl.B} of {wl.B} sequence(s), all {wl.Hq} heads, full {wl.L}-token context, one step per timed step"
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": thr, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_l_sweep(args):
    """Selection scaling with context length: for each L and policy (top-k 64,
    Gaussian with the bound, Gaussian with the capped estimate), the eager
    device time of each call of one step, medians over args.steps steps with
    the L2 flushed before each.  One JSON line per (L, policy)."""
    from sparse_entmax_kv_b200 import native as nv
    from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder
    from sparse_entmax_kv_b200.workloads import CONFIGS, make_inputs
    base = CONFIGS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(32 << 20, dtype=torch.int64, device=dev)
    st = torch.cuda.current_stream()
    for L in (65536, 131072, 262144, 524288, 1048576):
        wl = base.shrink(L=L)
        inp = make_inputs(wl, 4000, device=dev)
        for policy in ("topk", "gauss", "gauss_est"):
            dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                                  alpha=wl.alpha, policy=policy, k=64, delta=wl.delta or 0.5)
            dec.build_meta()
            calls = [
                lambda: nv.entmaxkv_score_pages(dec.shape, inp["q"], dec.meta, dec.seq_lens, dec.bbox, dec.mu,
                                                dec.sigma),
                lambda: nv.entmaxkv_select(dec.shape, dec.seq_lens, dec.bbox, dec.mu, dec.sigma, dec.policy, dec.k,
                                           dec.alpha, dec.delta, dec.sel, dec.cnt, dec.tau_hat),
                lambda: nv.entmaxkv_decode_sparse(dec.shape, inp["q"], dec.k_cache, dec.v_cache, dec.page_table,
                                                  dec.seq_lens, dec.sel, dec.cnt, dec.alpha, dec.out, dec.tau, None,
                                                  dec.ws)]
            ts = []
            for i in range(args.warmup + args.steps):
                flush_w.fill_(1)
                torch.amax(flush_r)
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
                ev[0].record(st)
                for c, e in zip(calls, ev[1:]):
                    c()
                    e.record(st)
                torch.cuda.synchronize()
                if i >= args.warmup:
                    ts.append([ev[j].elapsed_time(ev[j + 1]) * 1e3 for j in range(len(calls))])
            assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0
            med = np.median(np.array(ts), axis=0)
            print(json.dumps({"sweep": "context_length", "workload": base.name, "L": L, "policy": policy,
                              "k": 64 if policy == "topk" else None, "delta": None if policy == "topk" else wl.delta,
                              "score_us": round(float(med[0]), 2), "select_us": round(float(med[1]), 2),
                              "decode_sparse_us": round(float(med[2]), 2),
                              "step_us_eager": round(float(med.sum()), 2),
                              "pages_selected_mean": round(float(dec.cnt.float().mean()), 1),
                              "pages": wl.max_pages}), flush=True)
            del dec
        del inp
        torch.cuda.empty_cache()


def run_quality(args):
    """Approximation quality of sparse decoding at one kept set, entmax vs
    softmax (synthetic data): for each selection policy, per head, against
    the full-cache result of the same attention,
      entmax:  discarded mass delta = sum of full-cache p off the kept tokens,
               support recall (full-cache support tokens that were kept),
               relative output error, and its ratio to the 2 B delta bound
               (B = the largest value-row norm);
      softmax: discarded mass 1 - exp(lse_kept - lse_full) and the relative
               output error, on the same kept pages.
    One JSON line per policy (means and extremes over heads)."""
    from sparse_entmax_kv_b200 import native as nv
    from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder
    from sparse_entmax_kv_b200.workloads import CONFIGS, make_inputs
    wl = CONFIGS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_inputs(wl, 4000, device=dev)
    B, Hq, d, P, mp = wl.B, wl.Hq, wl.d, wl.P, wl.max_pages
    shape = nv.Shape(B, Hq, wl.Hkv, d, P, mp, wl.num_blocks)
    wsd = nv.alloc_workspace(shape, nv.CALL_DECODE_DENSE, dev)
    o_full = torch.empty((B, Hq, d), device=dev)
    p_full = torch.zeros((B, Hq, mp * P), device=dev)
    nv.entmaxkv_decode_dense(shape, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                             wl.alpha, o_full, None, p_full, wsd)
    s_full = torch.empty((B, Hq, d), device=dev)
    lse_full = torch.empty((B, Hq), device=dev)
    nv.entmaxkv_decode_dense(shape, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                             1.0, s_full, lse_full, None, wsd)
    vnorm = inp["v_cache"].float().norm(dim=-1).amax().item()  # B of the 2 B delta bound
    tok = torch.arange(mp * P, device=dev)
    valid = tok[None, :] < inp["seq_lens"][:, None].long()  # [B][tokens]
    for policy in ("topk", "gauss", "gauss_est"):
        dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], Hq,
                              alpha=wl.alpha, policy=policy, k=wl.k or 64, delta=wl.delta or 0.5)
        dec.build_meta()
        dec.step(inp["q"])
        o_sm = torch.empty((B, Hq, d), device=dev)
        lse_sm = torch.empty((B, Hq), device=dev)
        nv.entmaxkv_decode_sparse(shape, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"],
                                  inp["seq_lens"], dec.sel, dec.cnt, 1.0, o_sm, lse_sm, None, dec.ws)
        torch.cuda.synchronize()
        assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0
        # kept tokens per head: the pages of its selection
        # (entries past cnt are not written by the selection: they go to a spare column)
        keep_p = torch.zeros((B, Hq, mp + 1), dtype=torch.bool, device=dev)
        cnt = dec.cnt.long()
        used = torch.arange(mp, device=dev)[None, None, :] < cnt[..., None]
        keep_p.scatter_(2, torch.where(used, dec.sel.long().clamp(0, mp - 1), mp), True)
        keep_t = keep_p[..., :mp].repeat_interleave(P, dim=2) & valid[:, None, :]
        delta = (p_full * (~keep_t)).sum(-1)
        supp = p_full > 0
        recall = (supp & keep_t).sum(-1).float() / supp.sum(-1).clamp(min=1).float()
        rel_e = (dec.out - o_full).norm(dim=-1) / o_full.norm(dim=-1).clamp(min=1e-30)
        bound = (dec.out - o_full).norm(dim=-1) / (2 * vnorm * delta).clamp(min=1e-30)
        d_sm = 1 - torch.exp(lse_sm - lse_full)
        rel_s = (o_sm - s_full).norm(dim=-1) / s_full.norm(dim=-1).clamp(min=1e-30)
        f = lambda t: [float(f"{float(x):.4e}") for x in (t.mean(), t.min(), t.max())]
        print(json.dumps({"study": "quality", "workload": wl.name, "policy": policy,
                          "k": (wl.k or 64) if policy == "topk" else None,
                          "delta_margin": None if policy == "topk" else (wl.delta or 0.5),
                          "kept_pages_mean": round(float(dec.cnt.float().mean()), 1), "pages": mp,
                          "stats": "[mean, min, max] over (sequence, head)",
                          "entmax": {"alpha": wl.alpha, "discarded_mass": f(delta), "support_recall": f(recall),
                                     "rel_err": f(rel_e),
                                     "err_over_2B_delta": f(bound[delta > 0]) if bool((delta > 0).any()) else None},
                          "softmax": {"discarded_mass": f(d_sm), "rel_err": f(rel_s)}}), flush=True)
        del dec


def run_crossover(args):
    """Where the sparse step starts to beat reading the whole cache: the
    single-head tiny shape (B=1, Hq=Hkv=1, d=64, 16-token pages, alpha 1.5,
    top-k 32 pages, 8 needles) at growing context lengths.  Per L: the sparse
    step (append, score, select, decode) as one CUDA-graph replay, and the
    full-cache entmax and softmax decodes, eager; device time per call from
    CUDA events, mean over args.steps after args.warmup, L2 flushed before
    each.  One JSON line per L."""
    from sparse_entmax_kv_b200 import native as nv
    from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder, last_token_rows
    from sparse_entmax_kv_b200.workloads import CONFIGS, make_inputs
    base = CONFIGS["tiny_h1_L4k"]
    dev = torch.device("cuda", torch.cuda.current_device())
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(32 << 20, dtype=torch.int64, device=dev)
    st = torch.cuda.current_stream()

    def timed(fn):
        ts = []
        for i in range(args.warmup + args.steps):
            flush_w.fill_(1)
            torch.amax(flush_r)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            torch.cuda.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(b) * 1e3)
        return float(np.mean(ts))

    for L in (4096, 8192, 16384, 32768, 65536, 131072):
        wl = base.shrink(L=L)
        inp = make_inputs(wl, 4000, device=dev)
        dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                              alpha=wl.alpha, policy="topk", k=wl.k)
        dec.build_meta()
        nkv = last_token_rows(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"])
        dec.step(inp["q"], new_kv=nkv)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            dec.step(inp["q"], new_kv=nkv)
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(g):
            dec.step(inp["q"], new_kv=nkv)
        torch.cuda.synchronize()
        sparse = timed(g.replay)
        out = torch.empty((wl.B, wl.Hq, wl.d), device=dev)
        ws = nv.alloc_workspace(dec.shape, nv.CALL_DECODE_DENSE, dev)
        dense = {}
        for alpha, name in ((wl.alpha, "dense_entmax_us"), (1.0, "dense_softmax_us")):
            dense[name] = round(timed(lambda: nv.entmaxkv_decode_dense(
                dec.shape, inp["q"], dec.k_cache, dec.v_cache, dec.page_table, dec.seq_lens, alpha, out, None, None,
                ws)), 2)
        assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0
        print(json.dumps({"sweep": "crossover", "workload": base.name, "L": L, "sparse_step_us": round(sparse, 2),
                          **dense, "kv_bytes_full_cache": 2 * L * wl.d * 2,
                          "sparse_over_dense_softmax": round(sparse / dense["dense_softmax_us"], 3)}), flush=True)
        del dec, g, inp, ws
        torch.cuda.empty_cache()


def config_of(wl):
    return {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d, "L": wl.L,
            "page_size": wl.P, "alpha": wl.alpha, "policy": wl.policy, "k": wl.k, "delta": wl.delta,
            "keys": wl.keys, "needles_per_head": wl.needles, "page_table": "seeded permutation of the blocks",
            "l2": "flushed before every step (256 MiB write, then 256 MiB read of a clean buffer), "
                  "outside the per-step events"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gauss_gqa_L1m")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--dense-steps", type=int, default=5)
    ap.add_argument("--skip-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-dir", default=None,
                    help="where the nvidia-smi clock samples of the timed region are kept (default: temp dir)")
    ap.add_argument("--quality", action="store_true",
                    help="instead of the benchmark line: sparse vs full-cache error, entmax vs softmax at one kept set")
    ap.add_argument("--l-sweep", action="store_true",
                    help="instead of the benchmark line: selection scaling with context length (one line per L, policy)")
    ap.add_argument("--crossover", action="store_true",
                    help="instead of the benchmark line: sparse step vs full-cache decodes at growing L, tiny shape")
    ap.add_argument("--unfused", action="store_true",
                    help="step with the three separate calls (score, select, decode_sparse) instead of the fused "
                         "entmaxkv_decode_step")
    ap.add_argument("--page-table", default="random", choices=["random", "sequential"],
                    help="physical placement of the logical pages: a seeded permutation (default) or in order")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    torch.cuda.set_device(local)
    if args.l_sweep:
        run_l_sweep(args)
        return
    if args.quality:
        run_quality(args)
        return
    if args.crossover:
        run_crossover(args)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    from sparse_entmax_kv_b200 import native as nv  # noqa: F401  (fails loudly if not built)

    res = run_gpu(args, rank, world)
    wl = res["wl"]
    nb = res["nbytes"]
    value = whole_job_gbs(nb["kv_touched"], world, res["step_ms"])
    e2e_val = whole_job_gbs(nb["kv_touched"], world, res["e2e_ms"])
    cfg = config_of(wl)
    cfg["step"] = ("append + decode_step (scores, selection with the union, q.K, tau with p.V)" if res["fused"] else
                   "append + score_pages + select + decode_sparse")
    if args.page_table == "sequential":
        cfg["page_table"] = "identity: logical pages in block order"
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(res["step_ms"], 5),
            "us_per_step": round(res["step_ms"] * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "frac_of_hbm_peak": round(value / world / res["roofline"]["peak"], 4),
            "roofline": res["roofline"], "roofline_gather": res["roofline_gather"],
            "stages_us": res["stage_us"], "bytes_per_step": nb,
            "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "us_per_step": round(res["e2e_ms"] * 1e3, 2),
                    "h2d_bytes_per_step": res["e2e_bytes"][0], "d2h_bytes_per_step": res["e2e_bytes"][1],
                    "how": "the step's C-ABI calls, captured as one CUDA graph: append reads q and the appended "
                           "token's k/v rows from pinned host memory over the bus (copying q to the device, writing "
                           "the rows and refreshing their pages' metadata); the decode writes the output straight "
                           "into pinned host memory",
                    "eager_us_per_step": round(res["e2e_eager_ms"] * 1e3, 2)},
            "timing": "step = CUDA-graph replay of %s; stages_us: entmaxkv_append, entmaxkv_score_pages, "
                      "entmaxkv_select and entmaxkv_decode_sparse issued eagerly with events around each (sum %.2f "
                      "us)%s" % ("entmaxkv_append + entmaxkv_decode_step" if res["fused"] else
                                 "entmaxkv_append + entmaxkv_score_pages + entmaxkv_select + entmaxkv_decode_sparse",
                                 res["eager_step_ms"] * 1e3,
                                 ", decode_step the fused call alone" if res["fused"] else ""),
            "gpu_launches": res["launches"], "clocks": res["clocks"], "paper_context": PAPER_CONTEXT}
    if res["dense"]:
        de, ds = res["dense"]["dense_entmax"], res["dense"]["dense_softmax"]
        sp = res["step_ms"] * 1e3
        line["dense_us"] = {"entmax_full_cache": round(de, 1), "softmax_full_cache_splitk": round(ds, 1)}
        line["speedup"] = {"vs_dense_entmax": round(de / sp, 2), "vs_dense_softmax": round(ds / sp, 2)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        swl = sample_workload(wl)
        inp = res["host"]["inp"]
        host = host_copy({k: (v[:1] if k in ("q", "page_table", "seq_lens") else v) for k, v in inp.items()})
        sec, nbytes, thr, reps = oracle_step_sample(swl, host)
        line["cpu_baseline"] = {"value": round(nbytes / sec / 1e9, 4), "unit": "GB/s", "cores": thr,
                                "kind": "oracle",
                                "sample": f"sequence 0 of {wl.B}, all {wl.Hq} heads, full context; "
                                          f"median of {reps} oracle step(s), {sec:.2f} s each"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
