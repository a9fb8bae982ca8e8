"""The C-ABI library on the host: it loads, exports every declared symbol, and
rejects bad arguments with the documented codes before touching the GPU
(every call below returns from its host-side checks; none reaches CUDA)."""
import ctypes as C
import os
import re

import pytest

from sparse_entmax_kv_b200 import native as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "include", "entmaxkv.h")

FAKE = C.c_void_p(0x10000)       # aligned, never dereferenced
FAKE_ODD = C.c_void_p(0x10008)   # 8-byte aligned only


def _declared():
    txt = open(HDR).read()
    return sorted(set(re.findall(r"ENTMAXKV_API\s+[\w\s\*]+?\b(entmaxkv_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = nv.lib()
    names = _declared()
    assert len(names) == 20
    assert set(names) == set(nv.EXPORTED)
    for n in names:
        assert hasattr(L, n)


def test_status_bits_match_the_header():
    txt = open(HDR).read()
    bits = dict((m.group(1), int(m.group(2))) for m in re.finditer(r"ENTMAXKV_STATUS_(\w+)\s*=\s*(\d+)", txt))
    assert bits == {"BAD_PAGE": nv.STATUS_BAD_PAGE, "BAD_SELECTION": nv.STATUS_BAD_SELECTION,
                    "TIMEOUT": nv.STATUS_TIMEOUT, "OVERFLOW": nv.STATUS_OVERFLOW,
                    "BAD_LENGTH": nv.STATUS_BAD_LENGTH, "NONFINITE": nv.STATUS_NONFINITE}
    assert len(set(bits.values())) == len(bits) and all(v & (v - 1) == 0 for v in bits.values())


def test_selftest_wait_rejects_limits_out_of_range():
    L = nv.lib()
    assert L.entmaxkv_selftest_wait(0, None) == -2
    assert L.entmaxkv_selftest_wait(2_000_000_001, None) == -2


def test_strerror_and_version():
    L = nv.lib()
    assert L.entmaxkv_version() == 100
    for code in list(nv.ERR) + [-99]:
        assert L.entmaxkv_strerror(code)


def shp(**kw):
    d = dict(B=2, Hq=8, Hkv=2, d=128, page_size=32, max_pages=64, num_blocks=128, kv_begin=0, kv_count=0)
    d.update(kw)
    return nv.Shape(*[d[f] for f, _ in nv.Shape._fields_])


def test_decode_sparse_kernels_checks_its_arguments():
    L = nv.lib()
    assert L.entmaxkv_decode_sparse_kernels(C.byref(shp(Hq=6, Hkv=4)), C.c_float(1.5)) == -2  # ERR_SHAPE
    assert L.entmaxkv_decode_sparse_kernels(C.byref(shp()), C.c_float(0.5)) == -3              # ERR_ALPHA
    with pytest.raises(nv.EntmaxKVError, match="ERR_ALPHA"):  # through the binding
        nv.entmaxkv_decode_sparse_kernels(shp(), 0.5)


def test_sizes():
    s = shp()
    assert nv.meta_bytes(s) == 2 * 2 * 2 * 32 * 12 * 128    # B * Hkv * ceil(64/32) tiles * 32 pages * 12d
    assert nv.meta_bytes(shp(max_pages=65)) == 2 * 2 * 3 * 32 * 12 * 128
    assert nv.workspace_size(s, nv.CALL_SELECT) == 0
    ws = nv.workspace_size(s, nv.CALL_DECODE_SPARSE)
    assert ws >= 2 * 8 * 64 * 32 * 4            # z of every token of the page list
    part = 64 * 2 * 8 * (128 + 2) * 4           # split-K softmax partials (both paths)
    assert ws >= 2 * 8 * 64 * 32 * 4 + part
    assert nv.workspace_size(s, nv.CALL_DECODE_DENSE) >= 2 * 8 * 64 * 32 * 4 + part
    assert nv.workspace_size(s, 99) == (1 << 64) - 1
    assert nv.meta_bytes(shp(d=96)) == 0


@pytest.mark.parametrize("bad", [dict(d=96), dict(page_size=8), dict(Hq=6, Hkv=4), dict(Hq=24, Hkv=2),
                                 dict(B=0), dict(max_pages=0), dict(num_blocks=0),
                                 dict(max_pages=1 << 26, page_size=64), dict(kv_begin=2), dict(kv_begin=-1),
                                 dict(kv_count=3), dict(kv_begin=1, kv_count=2), dict(kv_count=-1)])
def test_bad_shapes_rejected_everywhere(bad):
    L = nv.lib()
    s = C.byref(shp(**bad))
    E = -2
    assert L.entmaxkv_build_meta(s, FAKE, FAKE, FAKE, 0, -1, FAKE, None) == E
    assert L.entmaxkv_append(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None) == E
    assert L.entmaxkv_score_pages(s, FAKE, FAKE, FAKE, FAKE, None, None, None) == E
    assert L.entmaxkv_select(s, FAKE, FAKE, None, None, 0, 4, 1.5, 0.0, FAKE, FAKE, None, None, 0, None) == E
    assert L.entmaxkv_decode_sparse(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1.5, FAKE, None, None,
                                    FAKE, 1 << 40, None) == E
    assert L.entmaxkv_decode_dense(s, FAKE, FAKE, FAKE, FAKE, FAKE, 1.5, FAKE, None, None, FAKE, 1 << 40,
                                   None) == E


def test_null_alignment_and_argument_codes():
    L = nv.lib()
    s = C.byref(shp())
    assert L.entmaxkv_build_meta(None, FAKE, FAKE, FAKE, 0, -1, FAKE, None) == -1
    assert L.entmaxkv_build_meta(s, None, FAKE, FAKE, 0, -1, FAKE, None) == -1
    assert L.entmaxkv_build_meta(s, FAKE_ODD, FAKE, FAKE, 0, -1, FAKE, None) == -8
    assert L.entmaxkv_build_meta(s, FAKE, FAKE, FAKE, -1, -1, FAKE, None) == -2
    assert L.entmaxkv_build_meta(s, FAKE, FAKE, FAKE, 0, -2, FAKE, None) == -2
    # append: every pointer is required; the caches and metadata 16-byte aligned
    for i in range(7):
        args = [FAKE] * 7
        args[i] = None
        assert L.entmaxkv_append(s, *args, None, None, None) == -1
    assert L.entmaxkv_append(s, FAKE, FAKE, FAKE, FAKE, FAKE_ODD, FAKE, FAKE, None, None, None) == -8
    assert L.entmaxkv_append(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE_ODD, FAKE, None, None, None) == -8
    assert L.entmaxkv_append(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE_ODD, None, None, None) == -8
    # q_in and q_out come together
    assert L.entmaxkv_append(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == -1
    assert L.entmaxkv_append(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == -1
    assert L.entmaxkv_score_pages(s, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == -1  # mu w/o sigma
    assert L.entmaxkv_score_pages(s, FAKE, FAKE, None, FAKE, None, None, None) == -1  # no seq_lens
    assert L.entmaxkv_score_pages(s, FAKE_ODD, FAKE, FAKE, FAKE, None, None, None) == -8
    # select
    sel = lambda pol, k, a, dl, mu=FAKE: L.entmaxkv_select(s, FAKE, FAKE, mu, mu, pol, k, a, dl, FAKE, FAKE,
                                                           None, None, 0, None)
    assert sel(0, 0, 1.5, 0.0) == -4
    assert sel(7, 4, 1.5, 0.0) == -4
    assert sel(1, 0, 1.5, float("inf")) == -4
    assert sel(1, 0, 1.0, 0.5) == -3
    assert sel(1, 0, float("nan"), 0.5) == -3
    assert sel(1, 0, 1.3, 0.5) == -7            # r = 1/0.3 not an integer
    assert sel(1, 0, 1.5, 0.5, mu=None) == -1
    assert L.entmaxkv_select(shp(max_pages=200000), FAKE, FAKE, None, None, 0, 4, 1.5, 0.0, FAKE, FAKE,
                             None, None, 0, None) == -2
    # decode
    need = nv.workspace_size(shp(), nv.CALL_DECODE_SPARSE)
    dec = lambda a, ws, wsb, q=FAKE, sl=FAKE, p=None: L.entmaxkv_decode_sparse(
        s, q, FAKE, FAKE, FAKE, FAKE, sl, FAKE, a, FAKE, None, p, ws, wsb, None)
    assert dec(0.5, FAKE, need) == -3
    assert dec(float("nan"), FAKE, need) == -3
    assert dec(1.0, FAKE, need, p=FAKE) == -1    # softmax over the kept pages: no p_out
    assert dec(1.5, FAKE, need, sl=None) == -1
    assert dec(1.5, FAKE, need - 1) == -5
    assert dec(1.5, None, need) == -5
    assert dec(1.5, C.c_void_p(0x10010), need) == -8   # workspace must be 256-byte aligned
    assert dec(1.5, FAKE, need, q=FAKE_ODD) == -8
    dd = lambda a, p=None: L.entmaxkv_decode_dense(s, FAKE, FAKE, FAKE, FAKE, FAKE, a, FAKE, None, p,
                                                   FAKE, need, None)
    assert dd(0.9) == -3
    assert dd(float("inf")) == -3
    assert dd(1.0, FAKE) == -1                   # no p_out for softmax


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        nv._ptr(q, torch.bfloat16, "q")


def test_decode_step_checks_its_arguments():
    """The fused step's host-side checks, each returning before any GPU work."""
    L = nv.lib()
    s = C.byref(shp())
    need = nv.workspace_size(shp(), nv.CALL_DECODE_STEP)
    assert need > nv.workspace_size(shp(), nv.CALL_DECODE_SPARSE)   # plus the union marks and counters

    def step(pol=0, k=4, a=1.5, dl=0.5, mu=None, sg=None, meta=FAKE, ws=FAKE, wsb=need, sh=s, sel=FAKE):
        return L.entmaxkv_decode_step(sh, FAKE, meta, FAKE, FAKE, FAKE, FAKE, pol, k, a, dl, FAKE, mu, sg, sel,
                                      FAKE, None, FAKE, None, None, ws, wsb, None)
    # the decode step's extra region: one byte of head bits per page and kv head (rows of
    # ceil(max_pages / 4) words rounded up to a multiple of 4), 256-byte aligned, last
    uwords = (-(-64 // 4) + 3) // 4 * 4
    assert need - nv.workspace_size(shp(), nv.CALL_DECODE_SPARSE) == -(-(2 * 2 * uwords * 4) // 256) * 256
    odd = shp(max_pages=70)
    uw = (-(-70 // 4) + 3) // 4 * 4
    assert (nv.workspace_size(odd, nv.CALL_DECODE_STEP) - nv.workspace_size(odd, nv.CALL_DECODE_SPARSE)
            == -(-(2 * 2 * uw * 4) // 256) * 256)
    assert step(a=1.0) == -3                       # entmax only
    assert step(a=float("nan")) == -3
    assert step(pol=7) == -4
    assert step(k=0) == -4
    assert step(pol=1, mu=FAKE, sg=FAKE, dl=float("inf")) == -4
    assert step(pol=1) == -1                       # Gaussian without mu / sigma
    assert step(mu=FAKE) == -1                     # mu without sigma
    assert step(pol=1, a=1.3, mu=FAKE, sg=FAKE) == -7
    assert step(sel=None) == -1
    assert step(meta=FAKE_ODD) == -8
    assert step(wsb=need - 1) == -5
    assert step(ws=None) == -5
    assert step(ws=C.c_void_p(0x10010)) == -8      # 256-byte alignment
    assert step(sh=C.byref(shp(d=96))) == -2
    assert step(sh=C.byref(shp(max_pages=200000))) == -2
    assert L.entmaxkv_decode_step_kernels(s, 7, C.c_float(1.5)) == -4
    assert L.entmaxkv_decode_step_kernels(s, 0, C.c_float(1.0)) == -3
    assert L.entmaxkv_decode_step_kernels(C.byref(shp(Hq=6, Hkv=4)), 0, C.c_float(1.5)) == -2


def test_static_decode_rejects_problems_beyond_its_scratch():
    """The allocation-free decode checks its fixed scratch size on the host."""
    L = nv.lib()
    big = shp(B=4, Hq=32, Hkv=8, max_pages=16384, page_size=64, num_blocks=65536)
    assert nv.workspace_size(big, nv.CALL_DECODE_SPARSE) > nv.STATIC_SCRATCH_BYTES
    rc = L.entmaxkv_decode_sparse_static(C.byref(big), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1.5, FAKE,
                                         None, None, None)
    assert rc == -9
    assert b"fixed" in L.entmaxkv_strerror(-9)
    assert L.entmaxkv_decode_sparse_static(C.byref(shp(d=96)), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1.5,
                                           FAKE, None, None, None) == -2
