"""ctypes front end of the fp64 CPU oracle (oracle/entmaxkv_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product path.  It takes numpy
arrays (bf16 inputs as uint16 bit patterns) and returns numpy arrays.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        i = C.c_int
        dbl = C.c_double
        L.orc_num_threads.restype = i
        L.orc_build_meta.argtypes = [i, i, i, i, i, P, P, P, P, P, P, P]
        L.orc_score_pages.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P]
        L.orc_gauss_J.argtypes = [i, dbl]
        L.orc_gauss_J.restype = dbl
        L.orc_tau_hat.argtypes = [i, P, P, P, dbl]
        L.orc_tau_hat.restype = dbl
        L.orc_select_topk.argtypes = [i, P, i, P]
        L.orc_select_topk.restype = i
        L.orc_select_gauss.argtypes = [i, P, dbl, dbl, dbl, P]
        L.orc_select_gauss.restype = i
        L.orc_select_gauss_est.argtypes = [i, P, P, P, P, dbl, dbl, dbl, P]
        L.orc_select_gauss_est.restype = i
        L.orc_zmax_of.argtypes = [i]
        L.orc_zmax_of.restype = dbl
        for fn in ("orc_sparsemax_tau", "orc_entmax15_tau"):
            getattr(L, fn).argtypes = [P, i]
            getattr(L, fn).restype = dbl
        L.orc_entmax_tau.argtypes = [P, i, dbl]
        L.orc_entmax_tau.restype = dbl
        L.orc_decode.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, i, dbl,
                                 P, P, P, P]
        L.orc_select.argtypes = [i, i, i, i, P, P, P, P, i, i, dbl, dbl, P, P, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().orc_num_threads()


def build_meta(K, page_table, seq_lens, Hkv, d, P, num_blocks):
    """Per-record kmin/kmax (uint16 bf16 bits), mean/var (float32), [rec][d]."""
    page_table = _c(page_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    K = _c(K, np.uint16)
    B, max_pages = page_table.shape
    nrec = num_blocks * Hkv
    kmin = np.zeros((nrec, d), np.uint16)
    kmax = np.zeros((nrec, d), np.uint16)
    mean = np.zeros((nrec, d), np.float32)
    var = np.zeros((nrec, d), np.float32)
    lib().orc_build_meta(B, Hkv, d, P, max_pages, _p(K), _p(page_table),
                         _p(seq_lens), _p(kmin), _p(kmax), _p(mean), _p(var))
    return kmin, kmax, mean, var


def score_pages(q, meta, page_table, seq_lens, Hkv, P):
    """bbox, mu, sigma float32 [B][Hq][max_pages] (NaN where not written)."""
    kmin, kmax, mean, var = meta
    q = _c(q, np.uint16)
    page_table = _c(page_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    max_pages = page_table.shape[1]
    out = [np.full((B, Hq, max_pages), np.nan, np.float32) for _ in range(3)]
    lib().orc_score_pages(B, Hq, Hkv, d, P, max_pages, _p(q), _p(_c(kmin, np.uint16)),
                          _p(_c(kmax, np.uint16)), _p(_c(mean, np.float32)),
                          _p(_c(var, np.float32)), _p(page_table), _p(seq_lens),
                          _p(out[0]), _p(out[1]), _p(out[2]))
    return tuple(out)


def gauss_J(r: int, c: float) -> float:
    return lib().orc_gauss_J(int(r), float(c))


def tau_hat(mu, sigma, n_tok, alpha):
    mu = _c(mu, np.float32)
    sigma = _c(sigma, np.float32)
    n_tok = _c(n_tok, np.int32)
    return lib().orc_tau_hat(len(mu), _p(mu), _p(sigma), _p(n_tok), float(alpha))


def select_topk(bbox, k):
    bbox = _c(bbox, np.float32)
    sel = np.zeros(max(1, len(bbox)), np.int32)
    n = lib().orc_select_topk(len(bbox), _p(bbox), int(k), _p(sel))
    return sel[:n]


def select_gauss(bbox, alpha, tau_hat_v, delta):
    bbox = _c(bbox, np.float32)
    sel = np.zeros(max(1, len(bbox)), np.int32)
    n = lib().orc_select_gauss(len(bbox), _p(bbox), float(alpha), float(tau_hat_v),
                               float(delta), _p(sel))
    return sel[:n]


def select_gauss_est(bbox, mu, sigma, n_tok, alpha, tau_hat_v, delta):
    """Gaussian rule with the capped Gaussian estimate of each page's max."""
    bbox, mu, sigma = (_c(x, np.float32) for x in (bbox, mu, sigma))
    n_tok = _c(n_tok, np.int32)
    sel = np.zeros(max(1, len(bbox)), np.int32)
    n = lib().orc_select_gauss_est(len(bbox), _p(bbox), _p(mu), _p(sigma), _p(n_tok), float(alpha),
                                   float(tau_hat_v), float(delta), _p(sel))
    return sel[:n]


def zmax_of(n: int) -> float:
    return lib().orc_zmax_of(int(n))


def select(seq_lens, bbox, mu, sigma, P, policy, k, alpha, delta):
    """Batched selection: sel [B][Hq][max_pages], cnt [B][Hq], tau_hat [B][Hq]."""
    seq_lens = _c(seq_lens, np.int32)
    bbox = _c(bbox, np.float32)
    B, Hq, max_pages = bbox.shape
    mu = _c(mu if mu is not None else np.zeros_like(bbox), np.float32)
    sigma = _c(sigma if sigma is not None else np.zeros_like(bbox), np.float32)
    sel = np.full((B, Hq, max_pages), -1, np.int32)
    cnt = np.zeros((B, Hq), np.int32)
    th = np.full((B, Hq), np.nan, np.float64)
    pol = {"topk": 0, "gauss": 1, "gauss_est": 2}[policy]
    lib().orc_select(B, Hq, P, max_pages, _p(seq_lens), _p(bbox), _p(mu), _p(sigma),
                     pol, int(k), float(alpha), float(delta), _p(sel), _p(cnt), _p(th))
    return sel, cnt, th


def sparsemax_tau(z):
    z = _c(z, np.float64)
    return lib().orc_sparsemax_tau(_p(z), len(z))


def entmax15_tau(z):
    z = _c(z, np.float64)
    return lib().orc_entmax15_tau(_p(z), len(z))


def entmax_tau(z, alpha):
    z = _c(z, np.float64)
    return lib().orc_entmax_tau(_p(z), len(z), float(alpha))


def decode(q, K, V, page_table, seq_lens, Hkv, P, alpha, sel=None, cnt=None,
           want_p=False, want_z=False):
    """o [B][Hq][d] fp64, tau [B][Hq], and optionally p / z in logical order."""
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    page_table = _c(page_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    max_pages = page_table.shape[1]
    o = np.zeros((B, Hq, d), np.float64)
    tau = np.zeros((B, Hq), np.float64)
    pw = np.zeros((B, Hq, max_pages * P), np.float64) if want_p else None
    zz = np.full((B, Hq, max_pages * P), -np.inf, np.float64) if want_z else None
    stride = 0
    if sel is not None:
        sel = _c(sel, np.int32)
        cnt = _c(cnt, np.int32)
        stride = sel.shape[-1]
    lib().orc_decode(B, Hq, Hkv, d, P, max_pages, _p(q), _p(K), _p(V),
                     _p(page_table), _p(seq_lens), _p(sel), _p(cnt), stride,
                     float(alpha), _p(o), _p(tau), _p(pw), _p(zz))
    return o, tau, pw, zz
