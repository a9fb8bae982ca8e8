"""Run a few decode steps of a workload for profiling (ncu) with no timing logic.

  python -m sparse_entmax_kv_b200.profile_step --workload gauss_gqa_L1m --steps 2 [--dense]

Launch order per step: build_meta (the appended page), score_pages, select,
decode_sparse (union, q.K, tau, p.V); with --dense, one full-cache entmax and
one full-cache softmax decode follow the steps.  The full metadata build runs
once before the steps.
"""
import argparse

import torch

from . import native as nv
from .decoder import EntmaxKVDecoder
from .workloads import CONFIGS, make_inputs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gauss_gqa_L1m")
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--dense", action="store_true")
    ap.add_argument("--L", type=int, default=0, help="override the context length")
    args = ap.parse_args()
    wl = CONFIGS[args.workload]
    if args.L:
        wl = wl.shrink(L=args.L)
    policy = wl.policy if wl.policy != "dense" else "topk"
    inp = make_inputs(wl, 4000, device="cuda")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=policy, k=wl.k or 64, delta=wl.delta or 0.5)
    dec.build_meta()
    append_page = (int(inp["seq_lens"][0]) - 1) // wl.P
    for _ in range(args.steps):
        dec.step(inp["q"], append_page)
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
