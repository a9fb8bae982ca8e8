"""Run a few decode steps of a workload for profiling (ncu) with no timing logic.

  python profile_step.py --workload gauss_gqa_L1m --steps 2 [--dense]
  python profile_step.py --workload gauss_gqa_L1m --steps 3 --score-only

Launch order per step: append (each sequence's newest token again), then the fused
decode step (score, select, union from the selection's marks, q.K, tau with p.V); with
--dense, one full-cache entmax and
one full-cache softmax decode follow the steps.  The full metadata build runs
once before the steps.  With --score-only the K/V caches are released after
the metadata build and each step is one score_pages call, so a profiler that
saves and restores device memory between passes handles only the metadata.
"""
import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from sparse_entmax_kv_b200 import native as nv  # noqa: E402
from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder, last_token_rows  # noqa: E402
from sparse_entmax_kv_b200.workloads import CONFIGS, make_inputs  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gauss_gqa_L1m")
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--dense", action="store_true")
    ap.add_argument("--L", type=int, default=0, help="override the context length")
    ap.add_argument("--score-only", action="store_true")
    args = ap.parse_args()
    wl = CONFIGS[args.workload]
    if args.L:
        wl = wl.shrink(L=args.L)
    policy = wl.policy if wl.policy != "dense" else "topk"
    inp = make_inputs(wl, 4000, device="cuda")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=policy, k=wl.k or 64, delta=wl.delta or 0.5)
    dec.build_meta()
    if args.score_only:
        q, seq_lens = inp["q"], inp["seq_lens"]
        del inp, dec.k_cache, dec.v_cache
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        for _ in range(args.steps):
            nv.entmaxkv_score_pages(dec.shape, q, dec.meta, seq_lens, dec.bbox, dec.mu, dec.sigma)
        torch.cuda.synchronize()
        assert nv.get_status(clear=True) == 0
        print("ok")
        return
    new_kv = last_token_rows(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"])
    for _ in range(args.steps):
        dec.step(inp["q"], new_kv=new_kv)
    if args.dense:
        out = torch.empty((wl.B, wl.Hq, wl.d), device="cuda")
        ws = nv.alloc_workspace(dec.shape, nv.CALL_DECODE_DENSE, "cuda")
        for alpha in (wl.alpha, 1.0):
            nv.entmaxkv_decode_dense(dec.shape, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"],
                                     inp["seq_lens"], alpha, out, None, None, ws)
    torch.cuda.synchronize()
    st = nv.get_status(clear=True)
    assert st & ~nv.STATUS_OVERFLOW == 0, st
    print("ok")


if __name__ == "__main__":
    main()
