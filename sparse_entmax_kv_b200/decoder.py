"""One EntmaxKV decode step over a paged cache, as a sequence of C-ABI calls.

``EntmaxKVDecoder`` owns the device buffers the calls need (metadata, page
scores, selections, workspace, output) and issues, on the current stream:

  entmaxkv_append        (each sequence's new key/value row and its page's
                          metadata) or entmaxkv_build_meta (a page the caller
                          already wrote the token to)
  entmaxkv_decode_step   (scores, selection -- top-k or Gaussian tau_hat -
                          Delta -- and the sparse decode in one call)

or, with ``fused=False`` (and always for alpha = 1 or several kv-head
ranges), the three calls it stands for: entmaxkv_score_pages,
entmaxkv_select and entmaxkv_decode_sparse, with identical results.  It does
no arithmetic itself; see include/entmaxkv.h for what each call computes.
"""
from __future__ import annotations

import torch

from . import native as nv


class EntmaxKVDecoder:
    def __init__(self, k_cache, v_cache, page_table, seq_lens, Hq, *, alpha=1.5, policy="topk",
                 k=64, delta=0.5, kv_splits=1, fused=True):
        dev = k_cache.device
        nb, Hkv, P, d = k_cache.shape
        B, max_pages = page_table.shape
        self.shape = nv.Shape(B, Hq, Hkv, d, P, max_pages, nb)
        self.k_cache, self.v_cache = k_cache, v_cache
        self.page_table, self.seq_lens = page_table, seq_lens
        self.alpha, self.k, self.delta = float(alpha), int(k), float(delta)
        self.policy = {"topk": nv.TOPK, "gauss": nv.GAUSS, "gauss_est": nv.GAUSS_EST}[policy]
        gauss = self.policy in (nv.GAUSS, nv.GAUSS_EST)
        self.meta = nv.alloc_meta(self.shape, dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.bbox = torch.empty((B, Hq, max_pages), **f32)
        self.mu = torch.empty((B, Hq, max_pages), **f32) if gauss else None
        self.sigma = torch.empty((B, Hq, max_pages), **f32) if gauss else None
        self.sel = torch.empty((B, Hq, max_pages), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, Hq), dtype=torch.int32, device=dev)
        self.tau_hat = torch.empty((B, Hq), **f32)
        self.tau = torch.empty((B, Hq), **f32)
        self.out = torch.empty((B, Hq, d), **f32)
        self.launches_per_step = 0
        # kv-head ranges, each stepped on its own stream (disjoint heads: the
        # buffers and the workspace are shared); a range's scoring waits for
        # the previous range's, so its selection and decode overlap the next
        # range's metadata scan
        n = max(1, min(int(kv_splits), Hkv))
        cut = [(i * Hkv) // n for i in range(n + 1)]
        self.ranges = [(cut[i], cut[i + 1] - cut[i]) for i in range(n) if cut[i + 1] > cut[i]]
        self.shapes = [self.shape.kv_range(k0, nk) for k0, nk in self.ranges] if n > 1 else [self.shape]
        self.streams = [torch.cuda.Stream(device=dev) for _ in self.shapes] if n > 1 else None
        self.scored = [torch.cuda.Event() for _ in self.shapes] if n > 1 else None
        self.fused = bool(fused) and self.alpha > 1.0 and n == 1
        self.ws = nv.alloc_workspace(self.shape, nv.CALL_DECODE_STEP if self.fused else nv.CALL_DECODE_SPARSE, dev)

    def kernels_per_step(self, append: bool) -> int:
        """Kernel launches of one ``step`` of this decoder."""
        return kernels_per_step(self.shape, self.alpha, append, self.policy if self.fused else None)

    def build_meta(self, first_page=0, n_pages=-1):
        nv.entmaxkv_build_meta(self.shape, self.k_cache, self.page_table, self.seq_lens,
                               first_page, n_pages, self.meta)

    def step(self, q, append_page=None, p_out=None, new_kv=None, out=None, q_in=None):
        """One decode step for query q (bf16 [B, Hq, d]).  ``new_kv``: the
        (k_new, v_new) rows (bf16 [B, Hkv, d]) of the token each sequence just
        gained, at position seq_lens-1, written into the cache together with
        its page's metadata; or ``append_page``: a logical page whose metadata
        is refreshed (the caller wrote the token already); or neither.
        ``out``: where the output goes (fp32 [B, Hq, d]; device memory or
        pinned host memory, which the decode writes directly); default the
        decoder's own buffer.  ``q_in``: with ``new_kv``, the queries as they
        arrive (bf16 [B, Hq, d], possibly pinned host memory, like the new
        rows), copied into q by the append kernel."""
        dst = self.out if out is None else out
        if self.streams is None:
            self._step_range(self.shape, q, append_page, p_out, new_kv, None, None, dst, q_in)
            return dst
        cur = torch.cuda.current_stream()
        prev = None
        for shape, st, ev in zip(self.shapes, self.streams, self.scored):
            st.wait_stream(cur)
            with torch.cuda.stream(st):
                self._step_range(shape, q, append_page, p_out, new_kv, prev, ev, dst, q_in)
            prev = ev
        for st in self.streams:
            cur.wait_stream(st)
        return dst

    def _step_range(self, shape, q, append_page, p_out, new_kv, after, scored, out, q_in=None):
        if new_kv is not None:
            nv.entmaxkv_append(shape, new_kv[0], new_kv[1], self.page_table, self.seq_lens,
                               self.k_cache, self.v_cache, self.meta, q_in, None if q_in is None else q)
        elif append_page is not None:
            nv.entmaxkv_build_meta(shape, self.k_cache, self.page_table, self.seq_lens,
                                   append_page, 1, self.meta)
        if self.fused:
            nv.entmaxkv_decode_step(shape, q, self.meta, self.k_cache, self.v_cache, self.page_table,
                                    self.seq_lens, self.policy, self.k, self.alpha, self.delta, self.bbox,
                                    self.mu, self.sigma, self.sel, self.cnt, out, self.tau_hat, self.tau, p_out,
                                    self.ws)
            return
        if after is not None:
            torch.cuda.current_stream().wait_event(after)
        nv.entmaxkv_score_pages(shape, q, self.meta, self.seq_lens, self.bbox, self.mu, self.sigma)
        if scored is not None:  # the next range's scan follows this one
            scored.record(torch.cuda.current_stream())
        nv.entmaxkv_select(shape, self.seq_lens, self.bbox, self.mu, self.sigma, self.policy,
                           self.k, self.alpha, self.delta, self.sel, self.cnt, self.tau_hat)
        nv.entmaxkv_decode_sparse(shape, q, self.k_cache, self.v_cache, self.page_table,
                                  self.seq_lens, self.sel, self.cnt, self.alpha, out,
                                  self.tau, p_out, self.ws)


def last_token_rows(k_cache, v_cache, page_table, seq_lens):
    """(k, v) rows, bf16 [B, Hkv, d], of each sequence's token at position
    seq_lens-1 as the cache holds them (appending them again leaves the cache
    as it is).  Indexing only."""
    P = k_cache.shape[2]
    pos = (seq_lens.long() - 1).clamp(min=0)
    blk = page_table.long().gather(1, (pos // P)[:, None])[:, 0]
    tok = pos % P
    return k_cache[blk, :, tok].contiguous(), v_cache[blk, :, tok].contiguous()


def kernels_per_step(shape, alpha: float, append: bool, policy=None) -> int:
    """Kernel launches one ``step`` issues: append (1, if appending), then for
    the fused step (policy given) what entmaxkv_decode_step reports, else
    score (1), select (1) and decode_sparse (2 or 3, as the library reports
    for the shape)."""
    if policy is not None:
        return (1 if append else 0) + nv.entmaxkv_decode_step_kernels(shape, policy, alpha)
    return (1 if append else 0) + 1 + 1 + nv.entmaxkv_decode_sparse_kernels(shape, alpha)
