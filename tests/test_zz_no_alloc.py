"""The allocation-free sparse decode (entmaxkv_decode_sparse_static).

Some callers cannot allocate device memory when they decode: code running
inside a framework whose memory pool or graph builder forbids new
allocations, or a host application whose own allocator owns all of the GPU's
memory.  For them the library keeps a fixed 16 MiB scratch array on each
device and this entry point uses it instead of a caller-provided workspace.

The test calls it twice in a row through the C ABI and checks both results
against the workspace-based entmaxkv_decode_sparse on the same inputs, within
the output tolerance of the parity tests (max abs 2e-3, relative L2 1e-3).
It lives in a file of its own, collected last, and needs no state from any
other test.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from sparse_entmax_kv_b200 import native as nv
from sparse_entmax_kv_b200.workloads import CONFIGS, make_inputs, to_host_u16

pytestmark = pytest.mark.gpu

OUT_ABS, OUT_REL = 2e-3, 1e-3


def _close(got, want):
    got = got.double().cpu().numpy()
    want = want.double().cpu().numpy()
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    return err <= OUT_ABS and rel <= OUT_REL, (err, rel)


def test_static_scratch_decode_matches_workspace_decode_twice():
    wl = CONFIGS["topk_gqa_L128k"].shrink(B=2, Hq=8, Hkv=2, L=8192, ragged=True, needles=8)
    inp = make_inputs(wl, 21, device="cuda")
    shape = nv.Shape(wl.B, wl.Hq, wl.Hkv, wl.d, wl.P, wl.max_pages, wl.num_blocks)
    assert nv.workspace_size(shape, nv.CALL_DECODE_SPARSE) <= nv.STATIC_SCRATCH_BYTES

    # selection from the oracle, so the test depends on no other kernel's output
    h = dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), page_table=inp["page_table"].cpu().numpy(),
             seq_lens=inp["seq_lens"].cpu().numpy())
    meta = orc.build_meta(h["K"], h["page_table"], h["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    bbox, mu, sig = orc.score_pages(h["q"], meta, h["page_table"], h["seq_lens"], wl.Hkv, wl.P)
    sel_h, cnt_h, _ = orc.select(h["seq_lens"], np.nan_to_num(bbox), np.nan_to_num(mu), np.nan_to_num(sig),
                                 wl.P, "topk", wl.k, wl.alpha, 0.0)
    sel, cnt = torch.from_numpy(sel_h).cuda(), torch.from_numpy(cnt_h).cuda()

    args = (shape, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], sel, cnt,
            wl.alpha)
    ref = torch.empty((wl.B, wl.Hq, wl.d), device="cuda")
    ref_tau = torch.empty((wl.B, wl.Hq), device="cuda")
    ws = nv.alloc_workspace(shape, nv.CALL_DECODE_SPARSE, "cuda")
    nv.entmaxkv_decode_sparse(*args, ref, ref_tau, None, ws)

    for call in range(2):
        out = torch.full((wl.B, wl.Hq, wl.d), float("nan"), device="cuda")
        tau = torch.full((wl.B, wl.Hq), float("nan"), device="cuda")
        nv.entmaxkv_decode_sparse_static(*args, out, tau)
        torch.cuda.synchronize()
        ok, (err, rel) = _close(out, ref)
        assert ok, f"call {call}: max abs {err:.3e}, rel L2 {rel:.3e}"
        assert torch.allclose(tau, ref_tau, atol=1e-6, rtol=0)
    assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0
