"""CUDA path vs the fp64 CPU oracle on identical seeded inputs.

Tolerances (EntmaxKV hot-path contract):
  * page metadata, bbox scores, top-k indices: bit-exact;
  * Gaussian page statistics mu, sigma (fp32 chains on the GPU, fp64 in the
    oracle): within the forward error bound of a d-term fp32 dot product,
    |err| <= 2 d u sum_j |term_j| with u = 2^-24 (doubled for slack);
  * Gaussian selection: exact except pages whose bound lies within 1e-5
    (relative) of the cutoff tau_hat - Delta; tau_hat within 1e-5 max(1,|tau_hat|);
  * outputs: max abs error <= 2e-3 and relative L2 <= 1e-3 (fp32 accumulation);
  * support sets: exact except tokens with |z - tau| < 1e-5.
Small cases run every stage on the whole batch; full-size workloads are
checked on sampled (sequence, kv head) sub-problems the oracle can finish.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from sparse_entmax_kv_b200 import native as nv
from sparse_entmax_kv_b200.decoder import EntmaxKVDecoder, last_token_rows
from sparse_entmax_kv_b200.workloads import CONFIGS, Workload, make_inputs, sweep_points, to_host_u16

pytestmark = pytest.mark.gpu

OUT_ABS, OUT_REL = 2e-3, 1e-3
BAND = 1e-5

# ------------------------------------------------------------- workloads

SMALL = {
    "tiny_full": CONFIGS["tiny_h1_L4k"],
    "tiny_ragged": CONFIGS["tiny_h1_L4k"].shrink(name="tiny_ragged", B=3, L=3000, ragged=True),
    "dense_small": CONFIGS["dense_gqa_L32k"].shrink(name="dense_small", B=2, Hq=8, Hkv=2, L=4096 + 32,
                                                    ragged=True, needles=8),
    "topk_small": CONFIGS["topk_gqa_L128k"].shrink(name="topk_small", B=2, Hq=8, Hkv=2, L=8192,
                                                   ragged=True, needles=8),
    "gauss_small": CONFIGS["gauss_gqa_L1m"].shrink(name="gauss_small", B=2, Hq=8, Hkv=2, L=32768,
                                                   ragged=True, needles=16),
    "mha_small": CONFIGS["sweep_mha_L64k"].shrink(name="mha_small", B=3, Hq=4, Hkv=4, L=2048,
                                                  ragged=True, needles=4),
    "gqa2_d64": Workload("gqa2_d64", B=2, Hq=4, Hkv=2, d=64, L=1500, P=16, alpha=1.25, policy="topk",
                         k=20, keys="offset", needles=3, ragged=True),
    "gqa8_d128": Workload("gqa8_d128", B=1, Hq=8, Hkv=1, d=128, L=2000, P=64, alpha=2.0, policy="gauss",
                          delta=0.25, keys="cluster", needles=2, ragged=True),
    # 400 (sequence, kv head) groups: the q.K grid (five CTAs per SM, 148
    # SMs) has one CTA per group, and each q.K CTA builds its group's union
    # of selected pages itself
    "groups400_gqa": Workload("groups400_gqa", B=50, Hq=16, Hkv=8, d=128, L=1500, P=32, alpha=1.5,
                              policy="topk", k=12, keys="offset", needles=3, ragged=True),
    # 320 groups: two q.K CTAs per group, each building the union and writing
    # the entries of every other step
    "groups320_gqa": Workload("groups320_gqa", B=40, Hq=16, Hkv=8, d=128, L=1500, P=32, alpha=1.5,
                              policy="topk", k=12, keys="offset", needles=3, ragged=True),
    "groups320_mha": Workload("groups320_mha", B=80, Hq=4, Hkv=4, d=64, L=700, P=16, alpha=1.5,
                              policy="gauss", delta=0.5, keys="cluster", needles=2, ragged=True),
    # 200 groups: three q.K CTAs per group, the union built once per group by
    # its own kernel
    "groups200_gqa": Workload("groups200_gqa", B=25, Hq=32, Hkv=8, d=64, L=1200, P=16, alpha=2.0,
                              policy="topk", k=16, keys="offset", needles=3, ragged=True),
}


def gpu_inputs(wl, seed):
    inp = make_inputs(wl, seed, device="cuda")
    host = dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                page_table=inp["page_table"].cpu().numpy(), seq_lens=inp["seq_lens"].cpu().numpy())
    return inp, host


def shape_of(wl):
    return nv.Shape(wl.B, wl.Hq, wl.Hkv, wl.d, wl.P, wl.max_pages, wl.num_blocks)


def unpack_meta(meta: torch.Tensor, wl, page_table, seq_lens):
    """Decode the library's metadata (32-page tiles in logical page order,
    16-coordinate chunks, swizzled 16-byte pieces: include/entmaxkv.h) into
    kmin, kmax, mean, var arrays indexed like the oracle's, [block*Hkv + kv
    head][d].  Rows of blocks no valid page maps to stay zero."""
    d, Hkv, B = wl.d, wl.Hkv, wl.B
    nt = -(-wl.max_pages // 32)
    NT, nch = B * Hkv * nt, d // 16
    m = meta.cpu().numpy()
    assert m.size == NT * 384 * d
    slot = np.arange(32)[:, None]
    bnd = m[:NT * 128 * d].view(np.uint16).reshape(NT, nch, 2, 32, 2, 8)
    bnd = bnd[:, :, :, slot, np.arange(2)[None, :] ^ ((slot >> 2) & 1), :]
    mom = m[NT * 128 * d:].view(np.float32).reshape(NT, nch, 2, 32, 4, 4)
    mom = mom[:, :, :, slot, np.arange(4)[None, :] ^ ((slot >> 1) & 3), :]
    logical = [x[:, :, part].transpose(0, 2, 1, 3, 4).reshape(B, Hkv, nt * 32, d)
               for x in (bnd, mom) for part in (0, 1)]
    pt = np.asarray(page_table)
    seq = np.asarray(seq_lens)
    out = [np.zeros((wl.num_blocks * Hkv, d), x.dtype) for x in logical]
    for b in range(B):
        npb = -(-int(seq[b]) // wl.P)
        rows = (pt[b, :npb].astype(np.int64)[None, :] * Hkv + np.arange(Hkv)[:, None])  # [Hkv][npb]
        for o, x in zip(out, logical):
            o[rows.reshape(-1)] = x[b, :, :npb].reshape(-1, d)
    return tuple(out)


def referenced_records(host, wl):
    recs = []
    for b in range(wl.B):
        np_b = -(-int(host["seq_lens"][b]) // wl.P)
        for p in range(np_b):
            blk = int(host["page_table"][b, p])
            recs.extend(blk * wl.Hkv + h for h in range(wl.Hkv))
    return np.array(sorted(recs))


def n_pages(host, wl, b):
    return -(-int(host["seq_lens"][b]) // wl.P)


def check_mu_sigma(gmu, gsig, omu, osig, q_u16, mean, var, recs, what=""):
    """gmu/gsig/omu/osig: [heads, pages]; q_u16: [heads, d]; recs: [heads, pages]
    record index of each (head, page).  Bound of a d-term fp32 chain: 2 d u sum|terms|."""
    from tests.helpers import bf16_bits_to_f64
    qd = bf16_bits_to_f64(q_u16)
    d = qd.shape[-1]
    u = 2.0 ** -24
    s_mu = np.einsum("hd,hpd->hp", np.abs(qd), np.abs(mean[recs].astype(np.float64))) / math.sqrt(d)
    s_v = np.einsum("hd,hpd->hp", qd * qd, var[recs].astype(np.float64)) / d
    tol_mu = 2 * 2 * d * u * s_mu + 2 * u * np.abs(omu)
    assert np.all(np.abs(gmu.astype(np.float64) - omu) <= tol_mu + 1e-30), f"{what}: mu"
    # sigma^2 has only non-negative terms: relative error <= 2 d u; sigma halves it
    tol_s = (2 * d * u + 4 * u) * np.sqrt(s_v) + 1e-30
    assert np.all(np.abs(gsig.astype(np.float64) - osig) <= tol_s), f"{what}: sigma"


def assert_outputs_close(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err <= OUT_ABS, f"{what}: max abs err {err:.3e}"
    assert rel <= OUT_REL, f"{what}: rel L2 err {rel:.3e}"


def check_support(p_gpu, z_orc, tau_orc, what=""):
    """Support of the GPU weights vs the oracle's {z > tau}, exempting |z-tau| < BAND."""
    sup_g = p_gpu > 0
    sup_o = z_orc > tau_orc
    diff = sup_g != sup_o
    if diff.any():
        near = np.abs(z_orc - tau_orc) < BAND
        assert np.all(near[diff]), f"{what}: {int((diff & ~near).sum())} support tokens differ"


def check_selection(sel_g, sel_o, cutoff_scores, cutoff, what=""):
    a, b = set(sel_g.tolist()), set(sel_o.tolist())
    if a == b:
        return
    for p in a ^ b:
        s = float(cutoff_scores[p])
        assert abs(s - cutoff) <= BAND * max(1.0, abs(cutoff)), f"{what}: page {p} differs (score {s}, cutoff {cutoff})"


@pytest.fixture(autouse=True)
def _clear_status():
    nv.get_status(clear=True)
    yield
    st = nv.get_status(clear=True)
    assert st & ~nv.STATUS_OVERFLOW == 0, f"device status {st}"


# ------------------------------------------------------------ per stage

@pytest.mark.parametrize("name", list(SMALL))
def test_meta_and_scores_bit_exact(name):
    wl = SMALL[name]
    inp, host = gpu_inputs(wl, 1)
    s = shape_of(wl)
    meta = nv.alloc_meta(s, "cuda")
    nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], inp["seq_lens"], 0, -1, meta)
    g = unpack_meta(meta, wl, host["page_table"], host["seq_lens"])
    o = orc.build_meta(host["K"], host["page_table"], host["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    recs = referenced_records(host, wl)
    for gi, oi, nm in zip(g, o, ("kmin", "kmax", "mean", "var")):
        np.testing.assert_array_equal(gi[recs].view(np.uint32 if gi.dtype == np.float32 else np.uint16),
                                      oi[recs].view(np.uint32 if oi.dtype == np.float32 else np.uint16),
                                      err_msg=nm)
    B, Hq, mp = wl.B, wl.Hq, wl.max_pages
    out = [torch.full((B, Hq, mp), float("nan"), device="cuda") for _ in range(3)]
    nv.entmaxkv_score_pages(s, inp["q"], meta, inp["seq_lens"], *out)
    ob = orc.score_pages(host["q"], o, host["page_table"], host["seq_lens"], wl.Hkv, wl.P)
    gb, gm, gs = (t.cpu().numpy() for t in out)
    for b in range(B):
        npb = n_pages(host, wl, b)
        np.testing.assert_array_equal(gb[b, :, :npb].view(np.uint32), ob[0][b, :, :npb].view(np.uint32),
                                      err_msg="bbox")
        recs = (host["page_table"][b, :npb][None, :] * wl.Hkv + (np.arange(Hq) // wl.G)[:, None])
        check_mu_sigma(gm[b, :, :npb], gs[b, :, :npb], ob[1][b, :, :npb], ob[2][b, :, :npb], host["q"][b],
                       o[2], o[3], recs, f"b{b}")
    # bound-only scoring gives the same bound
    bb2 = torch.full((B, Hq, mp), float("nan"), device="cuda")
    nv.entmaxkv_score_pages(s, inp["q"], meta, inp["seq_lens"], bb2)
    for b in range(B):
        npb = n_pages(host, wl, b)
        assert torch.equal(bb2[b, :, :npb], out[0][b, :, :npb])


@pytest.mark.parametrize("policy", ["topk", "gauss"])
def test_scores_bit_exact_with_several_tiles_per_warp(policy):
    """128 (sequence, kv head) groups of 32 metadata tiles: more tiles than
    resident warps, so every scoring warp streams two tiles back to back
    (ragged lengths leave some tiles partial or empty)."""
    wl = Workload("tiles2", B=16, Hq=32, Hkv=8, d=64, L=16384, P=16, alpha=1.5, policy=policy, k=16, delta=0.5,
                  keys="offset", needles=2, ragged=True)
    inp, host = gpu_inputs(wl, 29)
    inp["seq_lens"][3] = 16 * 100 + 5  # a short sequence: most of its tiles are empty
    host["seq_lens"] = inp["seq_lens"].cpu().numpy()
    s = shape_of(wl)
    meta = nv.alloc_meta(s, "cuda")
    nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], inp["seq_lens"], 0, -1, meta)
    o = orc.build_meta(host["K"], host["page_table"], host["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    B, Hq, mp = wl.B, wl.Hq, wl.max_pages
    out = [torch.full((B, Hq, mp), float("nan"), device="cuda") for _ in range(3)]
    gauss = policy == "gauss"
    nv.entmaxkv_score_pages(s, inp["q"], meta, inp["seq_lens"], out[0], out[1] if gauss else None,
                            out[2] if gauss else None)
    ob = orc.score_pages(host["q"], o, host["page_table"], host["seq_lens"], wl.Hkv, wl.P)
    gb, gm, gs = (t.cpu().numpy() for t in out)
    for b in range(B):
        npb = n_pages(host, wl, b)
        np.testing.assert_array_equal(gb[b, :, :npb].view(np.uint32), ob[0][b, :, :npb].view(np.uint32))
        assert np.isnan(gb[b, :, npb:]).all()  # nothing written past the sequence
        if gauss:
            recs = (host["page_table"][b, :npb][None, :] * wl.Hkv + (np.arange(Hq) // wl.G)[:, None])
            check_mu_sigma(gm[b, :, :npb], gs[b, :, :npb], ob[1][b, :, :npb], ob[2][b, :, :npb], host["q"][b],
                           o[2], o[3], recs, f"b{b}")


def _oracle_scores(host, wl):
    meta = orc.build_meta(host["K"], host["page_table"], host["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    return orc.score_pages(host["q"], meta, host["page_table"], host["seq_lens"], wl.Hkv, wl.P)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("policy", ["topk", "gauss", "gauss_est"])
def test_select_parity(name, policy):
    wl = SMALL[name]
    if policy != "topk" and abs(1.0 / (wl.alpha - 1) - round(1.0 / (wl.alpha - 1))) > 1e-9:
        pytest.skip("Gaussian policy needs integer 1/(alpha-1)")
    inp, host = gpu_inputs(wl, 2)
    bbox, mu, sig = _oracle_scores(host, wl)   # oracle scores as the shared input
    s = shape_of(wl)
    B, Hq, mp = wl.B, wl.Hq, wl.max_pages
    tb, tm, ts = (torch.from_numpy(np.nan_to_num(x, nan=0.0)).cuda() for x in (bbox, mu, sig))
    sel = torch.full((B, Hq, mp), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((B, Hq), dtype=torch.int32, device="cuda")
    th = torch.zeros((B, Hq), device="cuda")
    k = wl.k if wl.k else 16
    delta = wl.delta if wl.delta else 0.5
    pol = {"topk": nv.TOPK, "gauss": nv.GAUSS, "gauss_est": nv.GAUSS_EST}[policy]
    nv.entmaxkv_select(s, inp["seq_lens"], tb, tm, ts, pol, k, wl.alpha, delta, sel, cnt, th)
    osel, ocnt, oth = orc.select(host["seq_lens"], np.nan_to_num(bbox, nan=0.0), np.nan_to_num(mu, nan=0.0),
                                 np.nan_to_num(sig, nan=0.0), wl.P, policy, k, wl.alpha, delta)
    sel, cnt, th = sel.cpu().numpy(), cnt.cpu().numpy(), th.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            gs = sel[b, h, :cnt[b, h]]
            assert np.all(np.diff(gs) > 0), "ascending, no repeats"
            os_ = osel[b, h, :ocnt[b, h]]
            if policy == "topk":
                np.testing.assert_array_equal(gs, os_)
            else:
                assert th[b, h] == pytest.approx(oth[b, h], abs=1e-5 * max(1.0, abs(oth[b, h])))
                est = bbox[b, h].astype(np.float64)
                if policy == "gauss_est":
                    npb = n_pages(host, wl, b)
                    ntok = [min(wl.P, int(host["seq_lens"][b]) - p * wl.P) for p in range(npb)]
                    z = np.array([orc.zmax_of(t) for t in ntok] + [0.0] * (mp - npb))
                    est = np.minimum(est, mu[b, h].astype(np.float64) + z * sig[b, h].astype(np.float64))
                check_selection(gs, os_, (wl.alpha - 1) * est, oth[b, h] - delta, f"b{b}h{h}")


def _oracle_selection(host, wl, policy, k, delta):
    bbox, mu, sig = _oracle_scores(host, wl)
    return orc.select(host["seq_lens"], np.nan_to_num(bbox, nan=0.0), np.nan_to_num(mu, nan=0.0),
                      np.nan_to_num(sig, nan=0.0), wl.P, policy, k, wl.alpha, delta)


@pytest.mark.parametrize("name", list(SMALL))
def test_decode_sparse_parity(name):
    wl = SMALL[name]
    inp, host = gpu_inputs(wl, 3)
    policy = wl.policy if wl.policy != "dense" else "topk"
    k = wl.k if wl.k else 32
    osel, ocnt, _ = _oracle_selection(host, wl, policy, k, wl.delta or 0.5)
    s = shape_of(wl)
    B, Hq, d = wl.B, wl.Hq, wl.d
    sel = torch.from_numpy(osel).cuda()
    cnt = torch.from_numpy(ocnt).cuda()
    out = torch.empty((B, Hq, d), device="cuda")
    tau = torch.empty((B, Hq), device="cuda")
    pw = torch.zeros((B, Hq, wl.max_pages * wl.P), device="cuda")
    ws = nv.alloc_workspace(s, nv.CALL_DECODE_SPARSE, "cuda")
    nv.entmaxkv_decode_sparse(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                              sel, cnt, wl.alpha, out, tau, pw, ws)
    o, otau, op, oz = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                                 wl.P, wl.alpha, sel=osel, cnt=ocnt, want_p=True, want_z=True)
    assert_outputs_close(out.cpu().numpy(), o, name)
    np.testing.assert_allclose(tau.cpu().numpy(), otau, atol=2e-5 * max(1.0, np.abs(otau).max()))
    pw = pw.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            kept = np.isfinite(oz[b, h])
            check_support(pw[b, h][kept], oz[b, h][kept], otau[b, h], f"b{b}h{h}")
            np.testing.assert_allclose(pw[b, h][kept], op[b, h][kept], atol=2e-4)
    # a second call on the same workspace gives identical bits
    out2 = torch.empty_like(out)
    nv.entmaxkv_decode_sparse(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                              sel, cnt, wl.alpha, out2, None, None, ws)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("name", list(SMALL))
def test_decode_sparse_softmax_parity(name):
    """alpha = 1 on the sparse call: softmax over the tokens of the selected
    pages, and the log-sum-exp of their scores."""
    wl = SMALL[name]
    inp, host = gpu_inputs(wl, 8)
    k = wl.k if wl.k else 32
    osel, ocnt, _ = _oracle_selection(host, wl, "topk", k, 0.5)
    s = shape_of(wl)
    sel, cnt = torch.from_numpy(osel).cuda(), torch.from_numpy(ocnt).cuda()
    out = torch.empty((wl.B, wl.Hq, wl.d), device="cuda")
    lse = torch.empty((wl.B, wl.Hq), device="cuda")
    ws = nv.alloc_workspace(s, nv.CALL_DECODE_SPARSE, "cuda")
    nv.entmaxkv_decode_sparse(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                              sel, cnt, 1.0, out, lse, None, ws)
    o, olse, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                               wl.P, 1.0, sel=osel, cnt=ocnt)
    assert_outputs_close(out.cpu().numpy(), o, f"{name} softmax")
    np.testing.assert_allclose(lse.cpu().numpy(), olse, atol=2e-5 * max(1.0, np.abs(olse).max()))
    out2 = torch.empty_like(out)
    nv.entmaxkv_decode_sparse(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                              sel, cnt, 1.0, out2, None, None, ws)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("name", ["tiny_ragged", "dense_small", "mha_small", "gqa2_d64", "gqa8_d128"])
@pytest.mark.parametrize("alpha", [1.0, 1.5, 2.0, 1.25])
def test_decode_dense_parity(name, alpha):
    wl = SMALL[name]
    inp, host = gpu_inputs(wl, 4)
    s = shape_of(wl)
    B, Hq, d = wl.B, wl.Hq, wl.d
    out = torch.empty((B, Hq, d), device="cuda")
    tau = torch.empty((B, Hq), device="cuda")
    pw = torch.zeros((B, Hq, wl.max_pages * wl.P), device="cuda") if alpha > 1 else None
    ws = nv.alloc_workspace(s, nv.CALL_DECODE_DENSE, "cuda")
    nv.entmaxkv_decode_dense(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                             alpha, out, tau, pw, ws)
    o, otau, op, oz = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                                 wl.P, alpha, want_p=alpha > 1, want_z=True)
    assert_outputs_close(out.cpu().numpy(), o, f"{name} alpha={alpha}")
    np.testing.assert_allclose(tau.cpu().numpy(), otau, atol=2e-5 * max(1.0, np.abs(otau).max()))
    if alpha > 1:
        pw = pw.cpu().numpy()
        for b in range(B):
            for h in range(Hq):
                kept = np.isfinite(oz[b, h])
                check_support(pw[b, h][kept], oz[b, h][kept], otau[b, h], f"b{b}h{h}")


# ------------------------------------------------------- edge cases

def test_empty_selection_and_single_token_sequences():
    wl = Workload("edge", B=3, Hq=4, Hkv=2, d=128, L=64, P=32, alpha=1.5, policy="topk", k=4)
    inp, host = gpu_inputs(wl, 5)
    inp["seq_lens"] = torch.tensor([1, 33, 64], dtype=torch.int32, device="cuda")
    host["seq_lens"] = inp["seq_lens"].cpu().numpy()
    s = shape_of(wl)
    osel, ocnt, _ = orc.select(host["seq_lens"], np.zeros((3, 4, 2), np.float32), None, None, wl.P, "topk", 4,
                               1.5, 0.0)
    ocnt[2, 1] = 0  # one head selects nothing
    sel, cnt = torch.from_numpy(osel).cuda(), torch.from_numpy(ocnt).cuda()
    out = torch.full((3, 4, 128), 7.0, device="cuda")
    tau = torch.empty((3, 4), device="cuda")
    ws = nv.alloc_workspace(s, nv.CALL_DECODE_SPARSE, "cuda")
    nv.entmaxkv_decode_sparse(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                              sel, cnt, 1.5, out, tau, None, ws)
    o, otau, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], 2, 32, 1.5,
                               sel=osel, cnt=ocnt)
    out, tau = out.cpu().numpy(), tau.cpu().numpy()
    assert np.all(out[2, 1] == 0.0) and math.isnan(tau[2, 1])
    mask = np.ones((3, 4), bool)
    mask[2, 1] = False
    assert_outputs_close(out[mask], o[mask], "edge")
    # single-token sequence: p = 1 on that token, so out = its value row
    np.testing.assert_allclose(out[0], o[0], atol=1e-6)


def _sparse_vs_oracle(wl, inp, host, policy, k, label):
    """Oracle selection, then the library's sparse decode against the oracle's."""
    osel, ocnt, _ = _oracle_selection(host, wl, policy, k, wl.delta or 0.5)
    s = shape_of(wl)
    sel, cnt = torch.from_numpy(osel).cuda(), torch.from_numpy(ocnt).cuda()
    out = torch.empty((wl.B, wl.Hq, wl.d), device="cuda")
    tau = torch.empty((wl.B, wl.Hq), device="cuda")
    ws = nv.alloc_workspace(s, nv.CALL_DECODE_SPARSE, "cuda")
    nv.entmaxkv_decode_sparse(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                              sel, cnt, wl.alpha, out, tau, None, ws)
    o, otau, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                               wl.P, wl.alpha, sel=osel, cnt=ocnt)
    assert_outputs_close(out.cpu().numpy(), o, label)
    np.testing.assert_allclose(tau.cpu().numpy(), otau, atol=2e-5 * max(1.0, np.abs(otau).max()))


def test_decode_sparse_long_sequence_small_pages():
    """32771 pages of 16 tokens in one sequence (half a million tokens): page
    lists and z rows far longer than any on-chip buffer."""
    wl = Workload("long_p16", B=1, Hq=2, Hkv=1, d=64, L=32768 * 16 + 40, P=16, alpha=1.5, policy="topk",
                  k=48, keys="offset", needles=6, needle_scale=4.0)
    assert wl.max_pages > 32768
    inp, host = gpu_inputs(wl, 12)
    _sparse_vs_oracle(wl, inp, host, "topk", wl.k, "long_p16")


def test_decode_sparse_union_over_several_chunks():
    """A group of eight query heads (d = 64) over 61,443 pages: the union of
    the heads' selections is built 16,384 pages at a time, so the list
    positions run on across four chunks."""
    wl = Workload("union_chunks", B=1, Hq=8, Hkv=1, d=64, L=61443 * 16 - 8, P=16, alpha=1.5, policy="topk",
                  k=48, keys="offset", needles=6, needle_scale=4.0)
    assert wl.max_pages > 2 * 24576
    inp, host = gpu_inputs(wl, 14)
    _sparse_vs_oracle(wl, inp, host, "topk", wl.k, "union_chunks")


def test_decode_sparse_kernel_count():
    """The library's own count of a sparse decode's launches: a separate union
    kernel when the q.K grid splits each group over more than two CTAs, none
    when every group has one or two (those q.K CTAs build the union), two for
    softmax."""
    wide = shape_of(CONFIGS["gauss_gqa_L1m"])                      # 8 groups
    narrow = shape_of(SMALL["groups400_gqa"])                      # 400 groups: one CTA each
    two = shape_of(SMALL["groups320_gqa"])                          # 320 groups: two CTAs each
    three = shape_of(SMALL["groups200_gqa"])                        # 200 groups: three CTAs each
    assert nv.entmaxkv_decode_sparse_kernels(wide, 1.5) == 3
    assert nv.entmaxkv_decode_sparse_kernels(narrow, 1.5) == 2
    assert nv.entmaxkv_decode_sparse_kernels(two, 1.5) == 2
    assert nv.entmaxkv_decode_sparse_kernels(three, 1.5) == 3
    assert nv.entmaxkv_decode_sparse_kernels(wide, 1.0) == 2


def test_decode_sparse_all_tokens_candidates():
    """Equal keys put every selected token within 1 of the max z, more
    candidates than a head holds on chip: the exact path that rescans the z
    row (status OVERFLOW, nothing else) gives the oracle's result."""
    wl = Workload("flat", B=1, Hq=2, Hkv=1, d=64, L=64 * 600, P=64, alpha=2.0, policy="topk", k=512,
                  keys="offset", needles=0)
    inp, host = gpu_inputs(wl, 13)
    inp["k_cache"][:] = inp["k_cache"][0, 0, 0]
    host["K"] = to_host_u16(inp["k_cache"])
    nv.get_status(clear=True)
    _sparse_vs_oracle(wl, inp, host, "topk", wl.k, "flat")
    assert nv.get_status(clear=True) & nv.STATUS_OVERFLOW


def test_bad_page_table_entry_sets_status_and_skips():
    wl = SMALL["topk_small"]
    inp, _ = gpu_inputs(wl, 6)
    s = shape_of(wl)
    pt = inp["page_table"].clone()
    pt[0, 3] = wl.num_blocks + 5          # out of range: must be skipped, not read
    meta = nv.alloc_meta(s, "cuda")
    nv.get_status(clear=True)
    nv.entmaxkv_build_meta(s, inp["k_cache"], pt, inp["seq_lens"], 0, -1, meta)
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) & nv.STATUS_BAD_PAGE


def test_append_rebuild_matches_full_build():
    """Section 2.A 'maintained on append': rewriting the newest token and
    rebuilding only its page gives the same metadata as a full rebuild."""
    wl = SMALL["gauss_small"]
    inp, _ = gpu_inputs(wl, 7)
    s = shape_of(wl)
    meta = nv.alloc_meta(s, "cuda")
    nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], inp["seq_lens"], 0, -1, meta)
    b = 1
    L = int(inp["seq_lens"][b])
    p_last = (L - 1) // wl.P
    blk = int(inp["page_table"][b, p_last])
    inp["k_cache"][blk, :, (L - 1) % wl.P] = torch.randn(wl.Hkv, wl.d, device="cuda").to(torch.bfloat16) * 3
    nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], inp["seq_lens"], p_last, 1, meta)
    full = nv.alloc_meta(s, "cuda")
    nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], inp["seq_lens"], 0, -1, full)
    pt, sl = inp["page_table"].cpu().numpy(), inp["seq_lens"].cpu().numpy()
    a, c = unpack_meta(meta, wl, pt, sl), unpack_meta(full, wl, pt, sl)
    for b2 in range(wl.B):
        for p in range(-(-int(inp["seq_lens"][b2]) // wl.P)):
            bl = int(inp["page_table"][b2, p])
            for x, y in zip(a, c):
                assert np.array_equal(x[bl * wl.Hkv:(bl + 1) * wl.Hkv].view(np.uint8),
                                      y[bl * wl.Hkv:(bl + 1) * wl.Hkv].view(np.uint8))


@pytest.mark.parametrize("name", list(SMALL))
def test_append_writes_rows_and_rebuilds_page(name):
    """entmaxkv_append: each sequence's new key/value rows land in slot
    seq_len-1 (nothing else in the caches changes) and every metadata record
    equals the oracle's build over the updated cache, to the bit."""
    wl = SMALL[name]
    inp, _ = gpu_inputs(wl, 11)
    s = shape_of(wl)
    meta = nv.alloc_meta(s, "cuda")
    nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], inp["seq_lens"], 0, -1, meta)
    g = torch.Generator(device="cuda").manual_seed(5)
    k_new = (torch.randn(wl.B, wl.Hkv, wl.d, device="cuda", generator=g) * 2).to(torch.bfloat16)
    v_new = torch.randn(wl.B, wl.Hkv, wl.d, device="cuda", generator=g).to(torch.bfloat16)
    k_new[:, :, ::7] = 0.0  # exact zeros and ties with the page's other keys
    k_ref, v_ref = inp["k_cache"].clone(), inp["v_cache"].clone()
    for b in range(wl.B):
        L = int(inp["seq_lens"][b])
        if L > 0:
            blk = int(inp["page_table"][b, (L - 1) // wl.P])
            k_ref[blk, :, (L - 1) % wl.P] = k_new[b]
            v_ref[blk, :, (L - 1) % wl.P] = v_new[b]
    nv.get_status(clear=True)
    nv.entmaxkv_append(s, k_new, v_new, inp["page_table"], inp["seq_lens"], inp["k_cache"], inp["v_cache"], meta)
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) == 0
    assert torch.equal(inp["k_cache"].view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(inp["v_cache"].view(torch.int16), v_ref.view(torch.int16))
    host = dict(K=to_host_u16(k_ref), page_table=inp["page_table"].cpu().numpy(),
                seq_lens=inp["seq_lens"].cpu().numpy())
    got = unpack_meta(meta, wl, host["page_table"], host["seq_lens"])
    want = orc.build_meta(host["K"], host["page_table"], host["seq_lens"], wl.Hkv, wl.d, wl.P, wl.num_blocks)
    recs = referenced_records(host, wl)
    for gi, oi, nm in zip(got, want, ("kmin", "kmax", "mean", "var")):
        np.testing.assert_array_equal(gi[recs].view(np.uint32 if gi.dtype == np.float32 else np.uint16),
                                      oi[recs].view(np.uint32 if oi.dtype == np.float32 else np.uint16),
                                      err_msg=nm)


def test_decode_output_to_pinned_host_memory():
    """out may be pinned host memory: the kernels write the result there
    directly, equal to the device-buffer result bit for bit."""
    wl = SMALL["gauss_small"]
    inp, _ = gpu_inputs(wl, 13)
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=wl.policy, delta=wl.delta)
    dec.build_meta()
    dev_out = dec.step(inp["q"]).clone()
    host_out = torch.full((wl.B, wl.Hq, wl.d), float("nan")).pin_memory()
    dec.step(inp["q"], out=host_out)
    torch.cuda.synchronize()
    assert torch.equal(host_out, dev_out.cpu())


def test_append_reads_pinned_host_inputs_and_stages_q():
    """k_new, v_new and q_in in pinned host memory: the kernel reads them over
    the bus; the cache, the records and the staged q equal the device-input
    call's bit for bit."""
    wl = SMALL["topk_small"]
    s = shape_of(wl)
    outs = []
    for pinned in (False, True):
        inp, _ = gpu_inputs(wl, 14)
        meta = nv.alloc_meta(s, "cuda")
        nv.entmaxkv_build_meta(s, inp["k_cache"], inp["page_table"], inp["seq_lens"], 0, -1, meta)
        g = torch.Generator().manual_seed(3)
        k_new = torch.randn(wl.B, wl.Hkv, wl.d, generator=g).to(torch.bfloat16)
        v_new = torch.randn(wl.B, wl.Hkv, wl.d, generator=g).to(torch.bfloat16)
        q_in = torch.randn(wl.B, wl.Hq, wl.d, generator=g).to(torch.bfloat16)
        if pinned:
            k_new, v_new, q_in = k_new.pin_memory(), v_new.pin_memory(), q_in.pin_memory()
        else:
            k_new, v_new, q_in = k_new.cuda(), v_new.cuda(), q_in.cuda()
        q_out = torch.zeros(wl.B, wl.Hq, wl.d, dtype=torch.bfloat16, device="cuda")
        nv.get_status(clear=True)
        nv.entmaxkv_append(s, k_new, v_new, inp["page_table"], inp["seq_lens"], inp["k_cache"], inp["v_cache"], meta,
                           q_in, q_out)
        torch.cuda.synchronize()
        assert nv.get_status(clear=True) == 0
        assert torch.equal(q_out.cpu().view(torch.int16), q_in.cpu().view(torch.int16))
        outs.append((inp["k_cache"].view(torch.int16), inp["v_cache"].view(torch.int16), meta))
    for x, y in zip(*outs):
        assert torch.equal(x, y)


def test_append_bad_page_sets_status_and_skips():
    """A page-table entry outside [0, num_blocks) flags the status and that
    sequence writes nothing; the other sequences append as usual."""
    wl = SMALL["gqa2_d64"]
    inp, _ = gpu_inputs(wl, 12)
    s = shape_of(wl)
    meta = nv.alloc_meta(s, "cuda")
    pt = inp["page_table"].clone()
    L = [int(x) for x in inp["seq_lens"]]
    pt[0, (L[0] - 1) // wl.P] = wl.num_blocks  # out of range
    k_new = torch.full((wl.B, wl.Hkv, wl.d), 2.0, device="cuda", dtype=torch.bfloat16)
    v_new = torch.full((wl.B, wl.Hkv, wl.d), -3.0, device="cuda", dtype=torch.bfloat16)
    k_ref, v_ref = inp["k_cache"].clone(), inp["v_cache"].clone()
    for b in range(1, wl.B):
        if L[b] > 0:
            blk = int(pt[b, (L[b] - 1) // wl.P])
            k_ref[blk, :, (L[b] - 1) % wl.P] = k_new[b]
            v_ref[blk, :, (L[b] - 1) % wl.P] = v_new[b]
    nv.get_status(clear=True)
    nv.entmaxkv_append(s, k_new, v_new, pt, inp["seq_lens"], inp["k_cache"], inp["v_cache"], meta)
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) & nv.STATUS_BAD_PAGE
    assert torch.equal(inp["k_cache"].view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(inp["v_cache"].view(torch.int16), v_ref.view(torch.int16))


@pytest.mark.parametrize("name", ["gauss_small", "topk_small", "mha_small"])
@pytest.mark.parametrize("splits", [2, 4])
def test_kv_head_ranges_match_one_call(name, splits):
    """A step issued per kv-head range (entmaxkv_shape.kv_begin / kv_count, one
    stream each, shared buffers) writes exactly what one whole-shape step
    writes, and nothing for heads outside a range."""
    wl = SMALL[name]
    inp, _ = gpu_inputs(wl, 21)
    new_kv = last_token_rows(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"])
    outs = []
    for ks in (1, splits):
        dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                              alpha=wl.alpha, policy=wl.policy, k=wl.k or 64, delta=wl.delta or 0.5, kv_splits=ks)
        dec.build_meta()
        dec.out.fill_(float("nan"))
        dec.step(inp["q"], new_kv=new_kv)
        torch.cuda.synchronize()
        outs.append((dec.out.clone(), dec.sel.clone(), dec.cnt.clone(), dec.bbox.clone()))
    (o1, s1, c1, b1), (o2, s2, c2, b2) = outs
    assert torch.equal(o1.view(torch.int32), o2.view(torch.int32))
    assert torch.equal(c1, c2)
    for b in range(wl.B):
        for h in range(wl.Hq):
            n = int(c1[b, h])
            assert torch.equal(s1[b, h, :n], s2[b, h, :n])
    # a single range leaves the other heads' outputs alone
    s = shape_of(wl).kv_range(0, 1)
    out = torch.full((wl.B, wl.Hq, wl.max_pages), float("nan"), device="cuda")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=wl.policy, k=wl.k or 64, delta=wl.delta or 0.5)
    dec.build_meta()
    nv.entmaxkv_score_pages(s, inp["q"], dec.meta, inp["seq_lens"], out)
    torch.cuda.synchronize()
    G = wl.Hq // wl.Hkv
    assert torch.isnan(out[:, G:]).all()
    for b in range(wl.B):
        npb = -(-int(inp["seq_lens"][b]) // wl.P)
        assert torch.equal(out[b, :G, :npb], b1[b, :G, :npb])


# ------------------------------------------------------ the fused step

def _step_outputs(wl, inp, policy, fused, queries, lens=None):
    """Runs EntmaxKVDecoder.step once per query in `queries` (the last one
    counts) and returns every output of the last step."""
    seq_lens = inp["seq_lens"] if lens is None else lens
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], seq_lens, wl.Hq, alpha=wl.alpha,
                          policy=policy, k=wl.k or 16, delta=wl.delta or 0.5, fused=fused)
    assert dec.fused == fused
    dec.build_meta()
    p = torch.full((wl.B, wl.Hq, wl.max_pages * wl.P), float("nan"), device="cuda")
    for q in queries:
        for t in (dec.out, dec.tau, dec.tau_hat, dec.bbox, p):  # (p is written on the selected pages only)
            t.fill_(float("nan"))
        dec.step(q, p_out=p)
    torch.cuda.synchronize()
    return dict(out=dec.out.clone(), tau=dec.tau.clone(), tau_hat=dec.tau_hat.clone(), bbox=dec.bbox.clone(),
                mu=None if dec.mu is None else dec.mu.clone(), sigma=None if dec.sigma is None else dec.sigma.clone(),
                sel=dec.sel.clone(), cnt=dec.cnt.clone(), p=p, launches=dec.kernels_per_step(False))


def _assert_same_step(a, b, wl, lens, policy):
    def same(x, y, what):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32)), what
    same(a["out"], b["out"], "out")
    same(a["tau"], b["tau"], "tau")
    same(a["p"], b["p"], "p")
    assert torch.equal(a["cnt"], b["cnt"])
    for bb in range(wl.B):
        npb = -(-int(lens[bb]) // wl.P)
        same(a["bbox"][bb, :, :npb], b["bbox"][bb, :, :npb], "bbox")
        if a["mu"] is not None:
            same(a["mu"][bb, :, :npb], b["mu"][bb, :, :npb], "mu")
            same(a["sigma"][bb, :, :npb], b["sigma"][bb, :, :npb], "sigma")
        for h in range(wl.Hq):
            n = int(a["cnt"][bb, h])
            assert torch.equal(a["sel"][bb, h, :n], b["sel"][bb, h, :n])
            if policy != "topk":
                same(a["tau_hat"][bb, h], b["tau_hat"][bb, h], "tau_hat")


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("policy", ["topk", "gauss", "gauss_est"])
def test_decode_step_matches_separate_calls(name, policy):
    """entmaxkv_decode_step, whose selection kernel prepares each group's
    union of pages (marks in the workspace that a small kernel compacts; with
    one query head per group, the list itself), writes to the bit what
    score_pages, select and decode_sparse write, in five launches (four with
    G = 1).  The fused decoder first steps another query, so the marks of one
    call must not leak into the next."""
    wl = SMALL[name]
    inp, _ = gpu_inputs(wl, 31)
    q2 = (-inp["q"]).contiguous()
    sep = _step_outputs(wl, inp, policy, False, [inp["q"]])
    fus = _step_outputs(wl, inp, policy, True, [q2, inp["q"]])
    _assert_same_step(sep, fus, wl, inp["seq_lens"].cpu().numpy(), policy)
    assert fus["launches"] == (5 if wl.Hq > wl.Hkv else 4)


@pytest.mark.parametrize("policy", ["topk", "gauss"])
def test_decode_step_with_an_empty_sequence(policy):
    """A sequence of no tokens in the batch: its group's union is empty, its
    heads get out = 0 and tau = NaN, and the other sequences match the
    separate calls."""
    wl = SMALL["gauss_small"] if policy == "gauss" else SMALL["topk_small"]
    inp, _ = gpu_inputs(wl, 32)
    lens = inp["seq_lens"].clone()
    lens[1] = 0
    sep = _step_outputs(wl, inp, policy, False, [inp["q"]], lens)
    fus = _step_outputs(wl, inp, policy, True, [inp["q"], inp["q"]], lens)
    _assert_same_step(sep, fus, wl, lens.cpu().numpy(), policy)
    assert (fus["out"][1] == 0).all() and torch.isnan(fus["tau"][1]).all()


@pytest.mark.parametrize("policy", ["topk", "gauss", "gauss_est"])
def test_decode_step_beyond_16384_pages(policy):
    """Rows of more than 16384 pages (several top-k tiles; the single-CTA
    Gaussian solver): the selection does not build the union, the step falls
    back to the separate union pass and still matches the separate calls."""
    wl = Workload("long_rows", B=1, Hq=4, Hkv=2, d=64, L=20000 * 16 + 5, P=16, alpha=1.5, policy="gauss",
                  k=24, delta=0.5, keys="cluster", needles=8)
    assert wl.max_pages > 16384
    inp, _ = gpu_inputs(wl, 33)
    sep = _step_outputs(wl, inp, policy, False, [inp["q"]])
    fus = _step_outputs(wl, inp, policy, True, [inp["q"]])
    _assert_same_step(sep, fus, wl, inp["seq_lens"].cpu().numpy(), policy)
    assert fus["launches"] == 2 + nv.entmaxkv_decode_sparse_kernels(shape_of(wl), wl.alpha)


@pytest.mark.parametrize("policy", ["topk", "gauss"])
def test_decode_step_on_a_kv_range_clears_only_its_rows(policy):
    """A decode step on a kv-head range clears only its own groups' rows of the
    union marks in the workspace (calls on disjoint ranges may share one and
    overlap in time), and writes for its heads what the whole-shape step
    writes."""
    wl = SMALL["gauss_small"]  # B=2, Hq=8, Hkv=2
    inp, _ = gpu_inputs(wl, 41)
    s = shape_of(wl)
    whole = _step_outputs(wl, inp, policy, True, [inp["q"]])
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=policy, k=wl.k or 16, delta=wl.delta or 0.5)
    dec.build_meta()
    # the marks are the step workspace's last region: one row of ceil(max_pages/4)
    # words (rounded up to a multiple of 4) per (sequence, kv head)
    off = nv.workspace_size(s, nv.CALL_DECODE_SPARSE)
    uwords = (-(-wl.max_pages // 4) + 3) // 4 * 4
    rows = dec.ws[off:off + wl.B * wl.Hkv * uwords * 4].view(torch.int32).view(wl.B, wl.Hkv, uwords)
    rows.fill_(0x5A5A5A5A)
    r = s.kv_range(1, 1)
    G = wl.Hq // wl.Hkv
    nv.entmaxkv_decode_step(r, inp["q"], dec.meta, inp["k_cache"], inp["v_cache"], inp["page_table"],
                            inp["seq_lens"], dec.policy, dec.k, dec.alpha, dec.delta, dec.bbox, dec.mu, dec.sigma,
                            dec.sel, dec.cnt, dec.out, dec.tau_hat, dec.tau, None, dec.ws)
    torch.cuda.synchronize()
    assert nv.get_status(clear=True) & ~nv.STATUS_OVERFLOW == 0
    if G > 1:
        assert (rows[:, 0] == 0x5A5A5A5A).all()          # kv head 0: not this call's
        assert not (rows[:, 1] == 0x5A5A5A5A).any()      # kv head 1: cleared, then marked
    hs = slice(G, 2 * G)
    assert torch.equal(dec.out[:, hs].view(torch.int32), whole["out"][:, hs].view(torch.int32))
    assert torch.equal(dec.tau[:, hs].view(torch.int32), whole["tau"][:, hs].view(torch.int32))
    assert torch.equal(dec.cnt[:, hs], whole["cnt"][:, hs])


def test_decode_step_kernel_count():
    for name, n in (("gauss_gqa_L1m", 5), ("topk_gqa_L128k", 5), ("sweep_mha_L64k", 4)):
        s = shape_of(CONFIGS[name])
        for pol in (nv.TOPK, nv.GAUSS, nv.GAUSS_EST):
            assert nv.entmaxkv_decode_step_kernels(s, pol, 1.5) == n


# ---------------------------------------------------- full-size workloads

def _sub_problem(inp, wl, b, kvh):
    from tests.helpers import sub_problem
    return sub_problem(inp, wl, b, kvh)


FULL = ["tiny_h1_L4k", "dense_gqa_L32k", "topk_gqa_L128k", "gauss_gqa_L1m", "sweep_mha_L64k"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_step_sampled(name):
    """The decode step exactly as the benchmark launches it (EntmaxKVDecoder
    over the whole batch), checked on sampled (sequence, kv head) groups."""
    wl = CONFIGS[name]
    policy = wl.policy if wl.policy != "dense" else "topk"
    k = wl.k if wl.k else 64
    delta = wl.delta if wl.delta else 0.5
    inp = make_inputs(wl, 11, device="cuda")
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=policy, k=k, delta=delta)
    dec.build_meta()
    dec.step(inp["q"])
    torch.cuda.synchronize()
    gmeta = unpack_meta(dec.meta, wl, inp["page_table"].cpu().numpy(), inp["seq_lens"].cpu().numpy())
    rng = np.random.default_rng(0)
    groups = [(0, 0), (wl.B - 1, wl.Hkv - 1), (int(rng.integers(wl.B)), int(rng.integers(wl.Hkv)))]
    G = wl.G
    for b, kvh in groups:
        sp = _sub_problem(inp, wl, b, kvh)
        om = orc.build_meta(sp["K"], sp["page_table"], sp["seq_lens"], 1, wl.d, wl.P, sp["npb"])
        recs = sp["blocks"] * wl.Hkv + kvh
        for gi, oi in zip(gmeta, om):
            assert np.array_equal(gi[recs].view(np.uint8), oi.view(np.uint8))
        ob, omu, osg = orc.score_pages(sp["q"], om, sp["page_table"], sp["seq_lens"], 1, wl.P)
        hs = slice(kvh * G, (kvh + 1) * G)
        gb = dec.bbox[b, hs, :sp["npb"]].cpu().numpy()
        assert np.array_equal(gb.view(np.uint32), ob[0].view(np.uint32))
        if policy == "gauss":
            recs = np.tile(np.arange(sp["npb"])[None, :], (G, 1))
            check_mu_sigma(dec.mu[b, hs, :sp["npb"]].cpu().numpy(), dec.sigma[b, hs, :sp["npb"]].cpu().numpy(),
                           omu[0], osg[0], sp["q"][0], om[2], om[3], recs, f"{name} b{b} kvh{kvh}")
        osel, ocnt, oth = orc.select(sp["seq_lens"], ob, omu, osg, wl.P, policy, k, wl.alpha, delta)
        o, otau, _, _ = orc.decode(sp["q"], sp["K"], sp["V"], sp["page_table"], sp["seq_lens"], 1, wl.P,
                                   wl.alpha, sel=osel, cnt=ocnt)
        gsel = dec.sel[b, hs].cpu().numpy()
        gcnt = dec.cnt[b, hs].cpu().numpy()
        gout = dec.out[b, hs].cpu().numpy()
        gtau = dec.tau[b, hs].cpu().numpy()
        # the decode of the GPU's own selection, by the oracle: the output check
        # holds for every head, also where a page inside the cutoff band made
        # the two selections differ
        og, otg, _, _ = orc.decode(sp["q"], sp["K"], sp["V"], sp["page_table"], sp["seq_lens"], 1, wl.P,
                                   wl.alpha, sel=gsel[None, :, :sp["npb"]], cnt=gcnt[None])
        for g in range(G):
            gs, os_ = gsel[g, :gcnt[g]], osel[0, g, :ocnt[0, g]]
            if policy == "topk":
                np.testing.assert_array_equal(gs, os_)
            else:
                gth = float(dec.tau_hat[b, kvh * G + g])
                assert gth == pytest.approx(oth[0, g], abs=1e-5 * max(1.0, abs(oth[0, g])))
                check_selection(gs, os_, (wl.alpha - 1) * ob[0, g].astype(np.float64), oth[0, g] - delta)
            assert_outputs_close(gout[g], og[0, g], f"{name} b{b} h{kvh * G + g} (GPU selection)")
            assert float(gtau[g]) == pytest.approx(otg[0, g], abs=2e-5 * max(1, abs(otg[0, g])))
            if np.array_equal(gs, os_):
                assert_outputs_close(gout[g], o[0, g], f"{name} b{b} h{kvh * G + g}")
                assert float(gtau[g]) == pytest.approx(otau[0, g], abs=2e-5 * max(1, abs(otau[0, g])))


@pytest.mark.parametrize("name,alpha", [("dense_gqa_L32k", 1.5), ("dense_gqa_L32k", 1.0),
                                        ("gauss_gqa_L1m", 1.5), ("gauss_gqa_L1m", 1.0)])
def test_full_size_dense_sampled(name, alpha):
    wl = CONFIGS[name]
    inp = make_inputs(wl, 12, device="cuda")
    s = shape_of(wl)
    out = torch.empty((wl.B, wl.Hq, wl.d), device="cuda")
    tau = torch.empty((wl.B, wl.Hq), device="cuda")
    ws = nv.alloc_workspace(s, nv.CALL_DECODE_DENSE, "cuda")
    nv.entmaxkv_decode_dense(s, inp["q"], inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                             alpha, out, tau, None, ws)
    torch.cuda.synchronize()
    G = wl.G
    for b, kvh in [(0, 0), (wl.B - 1, wl.Hkv - 1)]:
        sp = _sub_problem(inp, wl, b, kvh)
        o, otau, _, _ = orc.decode(sp["q"], sp["K"], sp["V"], sp["page_table"], sp["seq_lens"], 1, wl.P, alpha)
        assert_outputs_close(out[b, kvh * G:(kvh + 1) * G].cpu().numpy(), o[0], f"{name} b{b} kvh{kvh}")
        np.testing.assert_allclose(tau[b, kvh * G:(kvh + 1) * G].cpu().numpy(), otau[0],
                                   atol=2e-5 * max(1.0, np.abs(otau).max()))


def _sweep_id(pt):
    pol = f"topk{pt['k']}" if pt["policy"] == "topk" else f"gauss{pt['delta']}"
    return f"a{pt['alpha']}-P{pt['P']}-{pol}-n{pt['needles']}"


@pytest.mark.parametrize("pt", sweep_points(), ids=_sweep_id)
def test_sweep_points_reduced_batch(pt):
    """Every point of the MHA sweep (alpha x page size x policy x needles, 108
    in all) at its full 65,536-token context with two sequences of two heads:
    the whole step as the benchmark launches it, against the oracle."""
    wl = CONFIGS["sweep_mha_L64k"].shrink(B=2, Hq=2, Hkv=2, **pt)
    inp = make_inputs(wl, 13, device="cuda")
    k = wl.k or 32
    delta = wl.delta or 0.5
    dec = EntmaxKVDecoder(inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], wl.Hq,
                          alpha=wl.alpha, policy=wl.policy, k=k, delta=delta)
    dec.build_meta()
    dec.step(inp["q"])
    torch.cuda.synchronize()
    host = dict(q=to_host_u16(inp["q"]), K=to_host_u16(inp["k_cache"]), V=to_host_u16(inp["v_cache"]),
                page_table=inp["page_table"].cpu().numpy(), seq_lens=inp["seq_lens"].cpu().numpy())
    ob, omu, osg = _oracle_scores(host, wl)
    assert np.array_equal(dec.bbox.cpu().numpy().view(np.uint32), ob.view(np.uint32))
    osel, ocnt, oth = orc.select(host["seq_lens"], ob, omu, osg, wl.P, wl.policy, k, wl.alpha, delta)
    gsel, gcnt, gout = dec.sel.cpu().numpy(), dec.cnt.cpu().numpy(), dec.out.cpu().numpy()
    gtau = dec.tau.cpu().numpy()
    # the oracle's decode of the GPU's own selection: checked for every head
    og, otg, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv,
                               wl.P, wl.alpha, sel=gsel, cnt=gcnt)
    o, _, _, _ = orc.decode(host["q"], host["K"], host["V"], host["page_table"], host["seq_lens"], wl.Hkv, wl.P,
                            wl.alpha, sel=osel, cnt=ocnt)
    th = dec.tau_hat.cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.Hq):
            gs, os_ = gsel[b, h, :gcnt[b, h]], osel[b, h, :ocnt[b, h]]
            assert np.all(np.diff(gs) > 0)
            if wl.policy == "gauss":
                assert th[b, h] == pytest.approx(oth[b, h], abs=1e-5 * max(1.0, abs(oth[b, h])))
                check_selection(gs, os_, (wl.alpha - 1) * ob[b, h].astype(np.float64), oth[b, h] - delta)
            else:
                np.testing.assert_array_equal(gs, os_)
            assert_outputs_close(gout[b, h], og[b, h], f"b{b}h{h} (GPU selection)")
            assert float(gtau[b, h]) == pytest.approx(otg[b, h], abs=2e-5 * max(1, abs(otg[b, h])))
            if np.array_equal(gs, os_):
                assert_outputs_close(gout[b, h], o[b, h], f"b{b}h{h}")


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
@pytest.mark.parametrize("policy", ["gauss", "gauss_est"])
def test_select_gauss_beyond_cluster_capacity(alpha, policy):
    """Sequences of more than 16,384 pages take the single-CTA Gaussian
    selection kernel (the four-CTA cluster form holds at most 16,384 pages):
    tau_hat and the kept pages against the oracle's, on 25,000 and 24,990
    pages of 16 tokens (d = 64, one kv head of four query heads)."""
    wl = Workload("gauss_long", B=2, Hq=4, Hkv=1, d=64, L=25000 * 16, P=16, alpha=alpha, policy="gauss",
                  delta=0.5, keys="cluster", needles=8, ragged=True)
    assert wl.max_pages > 16384
    inp, host = gpu_inputs(wl, 23)
    bbox, mu, sig = _oracle_scores(host, wl)
    s = shape_of(wl)
    B, Hq, mp = wl.B, wl.Hq, wl.max_pages
    tb, tm, ts = (torch.from_numpy(np.nan_to_num(x, nan=0.0)).cuda() for x in (bbox, mu, sig))
    sel = torch.full((B, Hq, mp), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((B, Hq), dtype=torch.int32, device="cuda")
    th = torch.zeros((B, Hq), device="cuda")
    pol = {"gauss": nv.GAUSS, "gauss_est": nv.GAUSS_EST}[policy]
    nv.entmaxkv_select(s, inp["seq_lens"], tb, tm, ts, pol, 1, alpha, wl.delta, sel, cnt, th)
    osel, ocnt, oth = orc.select(host["seq_lens"], np.nan_to_num(bbox, nan=0.0), np.nan_to_num(mu, nan=0.0),
                                 np.nan_to_num(sig, nan=0.0), wl.P, policy, 1, alpha, wl.delta)
    sel, cnt, th = sel.cpu().numpy(), cnt.cpu().numpy(), th.cpu().numpy()
    for b in range(B):
        npb = n_pages(host, wl, b)
        assert npb > 16384
        for h in range(Hq):
            gs, os_ = sel[b, h, :cnt[b, h]], osel[b, h, :ocnt[b, h]]
            assert np.all(np.diff(gs) > 0) and (gs.size == 0 or (gs[0] >= 0 and gs[-1] < npb))
            assert th[b, h] == pytest.approx(oth[b, h], abs=1e-5 * max(1.0, abs(oth[b, h])))
            est = bbox[b, h].astype(np.float64)
            if policy == "gauss_est":
                ntok = [min(wl.P, int(host["seq_lens"][b]) - p * wl.P) for p in range(npb)]
                z = np.array([orc.zmax_of(t) for t in ntok] + [0.0] * (mp - npb))
                est = np.minimum(est, mu[b, h].astype(np.float64) + z * sig[b, h].astype(np.float64))
            check_selection(gs, os_, (alpha - 1) * est, oth[b, h] - wl.delta, f"b{b}h{h}")
