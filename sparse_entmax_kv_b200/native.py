"""ctypes binding of libentmaxkv.so (declarations in include/entmaxkv.h).

Argument marshalling only: every function here checks that the tensors it is
given live on a CUDA device with the dtype the C ABI expects, passes their
device pointers, the shape struct and the current CUDA stream, and raises
``EntmaxKVError`` on a non-zero return code.  All arithmetic happens in the
library's kernels; there is no CPU path.  Importing this module fails loudly
when the shared library has not been built.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libentmaxkv.so")

OK = 0
ERR = {0: "OK", -1: "ERR_NULL", -2: "ERR_SHAPE", -3: "ERR_ALPHA", -4: "ERR_POLICY",
       -5: "ERR_WORKSPACE", -6: "ERR_CUDA", -7: "ERR_UNSUPPORTED", -8: "ERR_ALIGN", -9: "ERR_TOO_LARGE"}
STATIC_SCRATCH_BYTES = 16 << 20
TOPK, GAUSS, GAUSS_EST = 0, 1, 2
CALL_SELECT, CALL_DECODE_SPARSE, CALL_DECODE_DENSE, CALL_DECODE_STEP = 2, 3, 4, 5
STATUS_BAD_PAGE, STATUS_BAD_SELECTION, STATUS_TIMEOUT, STATUS_OVERFLOW = 1, 2, 4, 8
STATUS_BAD_LENGTH, STATUS_NONFINITE = 16, 32

EXPORTED = ("entmaxkv_strerror", "entmaxkv_version", "entmaxkv_meta_bytes",
            "entmaxkv_workspace_size", "entmaxkv_get_status", "entmaxkv_build_meta", "entmaxkv_append",
            "entmaxkv_score_pages", "entmaxkv_select", "entmaxkv_decode_sparse",
            "entmaxkv_decode_sparse_static", "entmaxkv_decode_dense", "entmaxkv_decode_sparse_begin",
            "entmaxkv_decode_sparse_candidates", "entmaxkv_entmax_threshold", "entmaxkv_decode_sparse_finish",
            "entmaxkv_decode_sparse_kernels", "entmaxkv_selftest_wait", "entmaxkv_decode_step",
            "entmaxkv_decode_step_kernels")


class EntmaxKVError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn} returned {code} ({ERR.get(code, '?')}): {msg}")
        self.code = code


class Shape(C.Structure):
    """entmaxkv_shape; kv_begin / kv_count restrict a call to a kv-head range
    (both 0: every head)."""
    _fields_ = [("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("d", C.c_int32),
                ("page_size", C.c_int32), ("max_pages", C.c_int32), ("num_blocks", C.c_int32),
                ("kv_begin", C.c_int32), ("kv_count", C.c_int32)]

    def kv_range(self, kv_begin: int, kv_count: int) -> "Shape":
        """A copy restricted to kv heads [kv_begin, kv_begin + kv_count)."""
        t = Shape(*self.astuple())
        t.kv_begin, t.kv_count = int(kv_begin), int(kv_count)
        return t

    @classmethod
    def of(cls, q: torch.Tensor, k_cache: torch.Tensor, page_table: torch.Tensor) -> "Shape":
        B, Hq, d = q.shape
        nb, Hkv, P, d2 = k_cache.shape
        assert d == d2 and page_table.shape[0] == B
        return cls(B, Hq, Hkv, d, P, page_table.shape[1], nb)

    def astuple(self):
        return tuple(getattr(self, f) for f, _ in self._fields_)


_lib = None


def lib():
    """Load libentmaxkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_entmax_kv_b200.build_native`")
        L = C.CDLL(LIB_PATH)
        vp, i32, f32, sz = C.c_void_p, C.c_int32, C.c_float, C.c_size_t
        sp = C.POINTER(Shape)
        L.entmaxkv_strerror.restype = C.c_char_p
        L.entmaxkv_strerror.argtypes = [C.c_int]
        L.entmaxkv_version.restype = C.c_int
        L.entmaxkv_meta_bytes.restype = sz
        L.entmaxkv_meta_bytes.argtypes = [sp]
        L.entmaxkv_workspace_size.restype = sz
        L.entmaxkv_workspace_size.argtypes = [sp, C.c_int]
        L.entmaxkv_get_status.argtypes = [C.POINTER(i32), C.c_int, vp]
        L.entmaxkv_build_meta.argtypes = [sp, vp, vp, vp, i32, i32, vp, vp]
        L.entmaxkv_append.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.entmaxkv_score_pages.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp]
        L.entmaxkv_select.argtypes = [sp, vp, vp, vp, vp, i32, i32, f32, f32, vp, vp, vp, vp, sz, vp]
        L.entmaxkv_decode_sparse.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp, sz, vp]
        L.entmaxkv_decode_dense.argtypes = [sp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp, sz, vp]
        L.entmaxkv_decode_sparse_static.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp]
        L.entmaxkv_decode_sparse_begin.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, i32, i32, f32, vp, vp, sz, vp]
        L.entmaxkv_decode_sparse_candidates.argtypes = [sp, vp, vp, vp, vp, vp, f32, vp, i32, vp, vp, vp, sz, vp]
        L.entmaxkv_entmax_threshold.argtypes = [sp, i32, i32, vp, vp, vp, f32, vp, vp]
        L.entmaxkv_decode_sparse_finish.argtypes = [sp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp, vp, sz, vp]
        L.entmaxkv_decode_sparse_kernels.argtypes = [sp, f32]
        L.entmaxkv_selftest_wait.argtypes = [C.c_uint64, vp]
        L.entmaxkv_decode_step.argtypes = [sp, vp, vp, vp, vp, vp, vp, i32, i32, f32, f32, vp, vp, vp, vp, vp, vp,
                                           vp, vp, vp, vp, sz, vp]
        L.entmaxkv_decode_step_kernels.argtypes = [sp, i32, f32]
        for fn in EXPORTED:
            if fn not in ("entmaxkv_strerror", "entmaxkv_version", "entmaxkv_meta_bytes",
                          "entmaxkv_workspace_size"):
                getattr(L, fn).restype = C.c_int
        _lib = L
    return _lib


def _check(fn, rc):
    if rc != OK:
        raise EntmaxKVError(fn, rc, lib().entmaxkv_strerror(rc).decode())


def _ptr(t, dtype=None, name="tensor", pinned_ok=False):
    """Device pointer of t.  pinned_ok: a pinned host tensor is accepted too
    (with unified addressing its address is valid in kernels, which then
    read or write host memory directly over the bus)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.device.type != "cuda" and not (pinned_ok and t.device.type == "cpu" and t.is_pinned()):
        raise ValueError(f"{name}: must be a CUDA tensor (no CPU path exists)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def meta_bytes(shape: Shape) -> int:
    return lib().entmaxkv_meta_bytes(C.byref(shape))


def workspace_size(shape: Shape, call: int) -> int:
    return lib().entmaxkv_workspace_size(C.byref(shape), call)


def alloc_meta(shape: Shape, device) -> torch.Tensor:
    return torch.empty(meta_bytes(shape), dtype=torch.uint8, device=device)


def alloc_workspace(shape: Shape, call: int, device) -> torch.Tensor:
    n = workspace_size(shape, call)
    if n == (1 << 64) - 1:
        raise EntmaxKVError("entmaxkv_workspace_size", -2, "invalid shape or call")
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def entmaxkv_selftest_wait(limit_ns: int, stream=None):
    """One bounded on-device wait that nothing ends: the kernel returns after
    limit_ns nanoseconds and sets STATUS_TIMEOUT."""
    _check("entmaxkv_selftest_wait", lib().entmaxkv_selftest_wait(int(limit_ns), _stream(stream)))


def get_status(clear=True, stream=None) -> int:
    v = C.c_int32(0)
    _check("entmaxkv_get_status", lib().entmaxkv_get_status(C.byref(v), int(clear), _stream(stream)))
    return v.value


def entmaxkv_build_meta(shape, k_cache, page_table, seq_lens, first_page, n_pages, meta, stream=None):
    _check("entmaxkv_build_meta", lib().entmaxkv_build_meta(
        C.byref(shape), _ptr(k_cache, torch.bfloat16, "k_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(first_page), int(n_pages), _ptr(meta, None, "meta"),
        _stream(stream)))


def entmaxkv_append(shape, k_new, v_new, page_table, seq_lens, k_cache, v_cache, meta, q_in=None, q_out=None,
                    stream=None):
    """k_new, v_new and q_in may be pinned host tensors (read by the kernel over the bus)."""
    _check("entmaxkv_append", lib().entmaxkv_append(
        C.byref(shape), _ptr(k_new, torch.bfloat16, "k_new", pinned_ok=True),
        _ptr(v_new, torch.bfloat16, "v_new", pinned_ok=True),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(k_cache, torch.bfloat16, "k_cache"), _ptr(v_cache, torch.bfloat16, "v_cache"),
        _ptr(meta, None, "meta"), _ptr(q_in, torch.bfloat16, "q_in", pinned_ok=True),
        _ptr(q_out, torch.bfloat16, "q_out"), _stream(stream)))


def entmaxkv_score_pages(shape, q, meta, seq_lens, bbox, mu=None, sigma=None, stream=None):
    _check("entmaxkv_score_pages", lib().entmaxkv_score_pages(
        C.byref(shape), _ptr(q, torch.bfloat16, "q"), _ptr(meta, None, "meta"),
        _ptr(seq_lens, torch.int32, "seq_lens"),
        _ptr(bbox, torch.float32, "bbox"), _ptr(mu, torch.float32, "mu"), _ptr(sigma, torch.float32, "sigma"),
        _stream(stream)))


def entmaxkv_select(shape, seq_lens, bbox, mu, sigma, policy, k, alpha, delta, sel, cnt, tau_hat=None,
                    workspace=None, stream=None):
    ws = _ptr(workspace, None, "workspace")
    _check("entmaxkv_select", lib().entmaxkv_select(
        C.byref(shape), _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(bbox, torch.float32, "bbox"),
        _ptr(mu, torch.float32, "mu"), _ptr(sigma, torch.float32, "sigma"), int(policy), int(k),
        float(alpha), float(delta), _ptr(sel, torch.int32, "sel"), _ptr(cnt, torch.int32, "cnt"),
        _ptr(tau_hat, torch.float32, "tau_hat"), ws, 0 if workspace is None else workspace.numel(),
        _stream(stream)))


def entmaxkv_decode_sparse(shape, q, k_cache, v_cache, page_table, seq_lens, sel, cnt, alpha, out,
                           tau_out=None, p_out=None, workspace=None, stream=None):
    _check("entmaxkv_decode_sparse", lib().entmaxkv_decode_sparse(
        C.byref(shape), _ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(sel, torch.int32, "sel"), _ptr(cnt, torch.int32, "cnt"),
        float(alpha), _ptr(out, torch.float32, "out", pinned_ok=True), _ptr(tau_out, torch.float32, "tau_out"),
        _ptr(p_out, torch.float32, "p_out"), _ptr(workspace, None, "workspace"),
        0 if workspace is None else workspace.numel(), _stream(stream)))


def entmaxkv_decode_sparse_kernels(shape, alpha):
    """Kernel launches of one entmaxkv_decode_sparse call for this shape."""
    n = lib().entmaxkv_decode_sparse_kernels(C.byref(shape), float(alpha))
    _check("entmaxkv_decode_sparse_kernels", min(n, 0))
    return n


def entmaxkv_decode_step(shape, q, meta, k_cache, v_cache, page_table, seq_lens, policy, k, alpha, delta, bbox,
                         mu, sigma, sel, cnt, out, tau_hat=None, tau_out=None, p_out=None, workspace=None,
                         stream=None):
    """Scores, selection and sparse decode in one call (workspace of CALL_DECODE_STEP)."""
    _check("entmaxkv_decode_step", lib().entmaxkv_decode_step(
        C.byref(shape), _ptr(q, torch.bfloat16, "q"), _ptr(meta, None, "meta"),
        _ptr(k_cache, torch.bfloat16, "k_cache"), _ptr(v_cache, torch.bfloat16, "v_cache"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"), int(policy),
        int(k), float(alpha), float(delta), _ptr(bbox, torch.float32, "bbox"), _ptr(mu, torch.float32, "mu"),
        _ptr(sigma, torch.float32, "sigma"), _ptr(sel, torch.int32, "sel"), _ptr(cnt, torch.int32, "cnt"),
        _ptr(tau_hat, torch.float32, "tau_hat"), _ptr(out, torch.float32, "out", pinned_ok=True),
        _ptr(tau_out, torch.float32, "tau_out"), _ptr(p_out, torch.float32, "p_out"),
        _ptr(workspace, None, "workspace"), 0 if workspace is None else workspace.numel(), _stream(stream)))


def entmaxkv_decode_step_kernels(shape, policy, alpha):
    """Kernel launches of one entmaxkv_decode_step call."""
    n = lib().entmaxkv_decode_step_kernels(C.byref(shape), int(policy), float(alpha))
    _check("entmaxkv_decode_step_kernels", min(n, 0))
    return n


def _kv_args(q, k_cache, v_cache, page_table, seq_lens):
    return (_ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
            _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
            _ptr(seq_lens, torch.int32, "seq_lens"))


def entmaxkv_decode_sparse_begin(shape, q, k_cache, v_cache, page_table, seq_lens, sel, cnt, sel_max_pages,
                                 page_begin, alpha, zmax_out, workspace, stream=None):
    _check("entmaxkv_decode_sparse_begin", lib().entmaxkv_decode_sparse_begin(
        C.byref(shape), *_kv_args(q, k_cache, v_cache, page_table, seq_lens),
        _ptr(sel, torch.int32, "sel"), _ptr(cnt, torch.int32, "cnt"), int(sel_max_pages), int(page_begin),
        float(alpha), _ptr(zmax_out, torch.float32, "zmax_out"), _ptr(workspace, None, "workspace"),
        workspace.numel(), _stream(stream)))


def entmaxkv_decode_sparse_candidates(shape, q, k_cache, v_cache, page_table, seq_lens, alpha, zmax_in, cap,
                                      cand_z, cand_n, workspace, stream=None):
    _check("entmaxkv_decode_sparse_candidates", lib().entmaxkv_decode_sparse_candidates(
        C.byref(shape), *_kv_args(q, k_cache, v_cache, page_table, seq_lens), float(alpha),
        _ptr(zmax_in, torch.float32, "zmax_in"), int(cap), _ptr(cand_z, torch.float32, "cand_z"),
        _ptr(cand_n, torch.int32, "cand_n"), _ptr(workspace, None, "workspace"), workspace.numel(),
        _stream(stream)))


def entmaxkv_entmax_threshold(shape, n_shards, cap, cand_z, cand_n, zmax_in, alpha, tau_out, stream=None):
    _check("entmaxkv_entmax_threshold", lib().entmaxkv_entmax_threshold(
        C.byref(shape), int(n_shards), int(cap), _ptr(cand_z, torch.float32, "cand_z"),
        _ptr(cand_n, torch.int32, "cand_n"), _ptr(zmax_in, torch.float32, "zmax_in"), float(alpha),
        _ptr(tau_out, torch.float32, "tau_out"), _stream(stream)))


def entmaxkv_decode_sparse_finish(shape, q, k_cache, v_cache, page_table, seq_lens, alpha, zmax_in, tau_in, out,
                                  p_out, workspace, stream=None):
    _check("entmaxkv_decode_sparse_finish", lib().entmaxkv_decode_sparse_finish(
        C.byref(shape), *_kv_args(q, k_cache, v_cache, page_table, seq_lens), float(alpha),
        _ptr(zmax_in, torch.float32, "zmax_in"), _ptr(tau_in, torch.float32, "tau_in"),
        _ptr(out, torch.float32, "out"), _ptr(p_out, torch.float32, "p_out"), _ptr(workspace, None, "workspace"),
        workspace.numel(), _stream(stream)))


def entmaxkv_decode_dense(shape, q, k_cache, v_cache, page_table, seq_lens, alpha, out, tau_out=None,
                          p_out=None, workspace=None, stream=None):
    _check("entmaxkv_decode_dense", lib().entmaxkv_decode_dense(
        C.byref(shape), _ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), float(alpha), _ptr(out, torch.float32, "out"),
        _ptr(tau_out, torch.float32, "tau_out"), _ptr(p_out, torch.float32, "p_out"),
        _ptr(workspace, None, "workspace"), 0 if workspace is None else workspace.numel(), _stream(stream)))


def entmaxkv_decode_sparse_static(shape, q, k_cache, v_cache, page_table, seq_lens, sel, cnt, alpha, out,
                                  tau_out=None, p_out=None, stream=None):
    """entmaxkv_decode_sparse with the library's fixed on-device scratch instead of a workspace."""
    _check("entmaxkv_decode_sparse_static", lib().entmaxkv_decode_sparse_static(
        C.byref(shape), _ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(sel, torch.int32, "sel"), _ptr(cnt, torch.int32, "cnt"),
        float(alpha), _ptr(out, torch.float32, "out"), _ptr(tau_out, torch.float32, "tau_out"),
        _ptr(p_out, torch.float32, "p_out"), _stream(stream)))
