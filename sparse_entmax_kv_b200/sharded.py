"""Sequence-sharded sparse decode: one context split across ranks by
consecutive page ranges (EntmaxKV summary, section 2.C computed in pieces).

Rank r of S holds global pages [r*M, r*M + M) of every sequence (M =
ceil(max_pages / S)): its own paged K/V cache, page table and token counts,
and the metadata of its pages.  One step (``sharded_step``):

  1. score the rank's pages;
  2. all-gather the page scores; every rank runs the same global selection
     (so every rank holds the lists a single device would compute);
  3. union and q.K of the rank's selected pages -> the rank's max z per head;
  4. all-reduce max z;
  5. the rank's candidates (z > max z - 1, every token that can carry weight);
  6. all-gather the candidates; every rank solves the same exact tau;
  7. the rank's partial p.V (entmax weights are absolute, so partials add);
  8. all-reduce the outputs with sum.

Collectives go through a small communicator (``all_gather`` stacking the
ranks' tensors in rank order, ``all_reduce_max``, ``all_reduce_sum``):
``TorchComm`` wraps ``torch.distributed`` (NCCL between GPUs).  The compute of
every phase is a C-ABI call (``NativeShard``); this module only moves
arguments and reshapes the gathered scores.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import native as nv


class TorchComm:
    """Collectives over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)

    def all_gather(self, t):
        t = t.contiguous()
        parts = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(parts, t, group=self.group)
        return torch.stack(parts)

    def all_reduce_max(self, t):
        t = t.clone()
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=self.group)
        return t

    def all_reduce_sum(self, t):
        t = t.clone()
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
        return t


def shard_pages(max_pages: int, n_shards: int):
    """Pages per shard M and each shard's first global page."""
    M = -(-max_pages // n_shards)
    return M, [r * M for r in range(n_shards)]


def split_context(page_table, seq_lens, P: int, n_shards: int, rank: int):
    """This rank's page table [B][M], token counts [B] and first global page."""
    B, max_pages = page_table.shape
    M, begins = shard_pages(max_pages, n_shards)
    p0 = begins[rank]
    pt = torch.full((B, M), -1, dtype=torch.int32, device=page_table.device)
    w = max(0, min(M, max_pages - p0))
    if w:
        pt[:, :w] = page_table[:, p0:p0 + w]
    local = (seq_lens.long() - p0 * P).clamp(min=0, max=M * P).to(torch.int32)
    return pt.contiguous(), local.contiguous(), p0


class NativeShard:
    """One rank's shard and the library calls of each phase."""

    def __init__(self, k_cache, v_cache, page_table, seq_lens, seq_lens_global, Hq, page_begin,
                 max_pages_global, *, alpha=1.5, policy="gauss", k=64, delta=0.5, cap=2048):
        dev = k_cache.device
        nb, Hkv, P, d = k_cache.shape
        B, M = page_table.shape
        self.k_cache, self.v_cache, self.page_table = k_cache, v_cache, page_table
        self.seq_lens, self.seq_lens_global = seq_lens, seq_lens_global
        self.page_begin, self.max_pages_global, self.cap = int(page_begin), int(max_pages_global), int(cap)
        self.alpha, self.k, self.delta = float(alpha), int(k), float(delta)
        self.policy = {"topk": nv.TOPK, "gauss": nv.GAUSS, "gauss_est": nv.GAUSS_EST}[policy]
        gauss = self.policy != nv.TOPK
        self.shape = nv.Shape(B, Hq, Hkv, d, P, M, nb)
        self.gshape = nv.Shape(B, Hq, Hkv, d, P, self.max_pages_global, nb)
        f32 = dict(dtype=torch.float32, device=dev)
        i32 = dict(dtype=torch.int32, device=dev)
        self.meta = nv.alloc_meta(self.shape, dev)
        self.bbox = torch.empty((B, Hq, M), **f32)
        self.mu = torch.empty((B, Hq, M), **f32) if gauss else None
        self.sigma = torch.empty((B, Hq, M), **f32) if gauss else None
        self.sel = torch.empty((B, Hq, self.max_pages_global), **i32)
        self.cnt = torch.empty((B, Hq), **i32)
        self.zmax = torch.empty((B, Hq), **f32)
        self.cand_z = torch.empty((B, Hq, self.cap), **f32)
        self.cand_n = torch.empty((B, Hq), **i32)
        self.tau = torch.empty((B, Hq), **f32)
        self.out = torch.empty((B, Hq, d), **f32)
        self.ws = nv.alloc_workspace(self.shape, nv.CALL_DECODE_SPARSE, dev)

    def build_meta(self):
        nv.entmaxkv_build_meta(self.shape, self.k_cache, self.page_table, self.seq_lens, 0, -1, self.meta)

    def score(self, q):
        nv.entmaxkv_score_pages(self.shape, q, self.meta, self.seq_lens, self.bbox, self.mu, self.sigma)
        return self.bbox, self.mu, self.sigma

    def select(self, bbox, mu, sigma):
        nv.entmaxkv_select(self.gshape, self.seq_lens_global, bbox, mu, sigma, self.policy, self.k,
                           self.alpha, self.delta, self.sel, self.cnt)

    def begin(self, q):
        nv.entmaxkv_decode_sparse_begin(self.shape, q, self.k_cache, self.v_cache, self.page_table, self.seq_lens,
                                        self.sel, self.cnt, self.max_pages_global, self.page_begin, self.alpha,
                                        self.zmax, self.ws)
        return self.zmax

    def candidates(self, q, zmax):
        nv.entmaxkv_decode_sparse_candidates(self.shape, q, self.k_cache, self.v_cache, self.page_table,
                                             self.seq_lens, self.alpha, zmax, self.cap, self.cand_z, self.cand_n,
                                             self.ws)
        return self.cand_z, self.cand_n

    def threshold(self, cand_z_all, cand_n_all, zmax):
        nv.entmaxkv_entmax_threshold(self.shape, cand_z_all.shape[0], self.cap, cand_z_all.contiguous(),
                                     cand_n_all.contiguous(), zmax, self.alpha, self.tau)
        return self.tau

    def finish(self, q, zmax, tau):
        nv.entmaxkv_decode_sparse_finish(self.shape, q, self.k_cache, self.v_cache, self.page_table, self.seq_lens,
                                         self.alpha, zmax, tau, self.out, None, self.ws)
        return self.out


def gather_scores(comm, x, max_pages_global):
    """[S][B][Hq][M] gathered page scores -> [B][Hq][max_pages_global]."""
    g = comm.all_gather(x)
    S, B, Hq, M = g.shape
    return g.permute(1, 2, 0, 3).reshape(B, Hq, S * M)[:, :, :max_pages_global].contiguous()


def sharded_step(shard, comm, q):
    """One sequence-sharded decode step on this rank; returns the full output
    [B][Hq][d] (the same on every rank)."""
    bbox, mu, sigma = shard.score(q)
    G = shard.max_pages_global
    shard.select(gather_scores(comm, bbox, G), None if mu is None else gather_scores(comm, mu, G),
                 None if sigma is None else gather_scores(comm, sigma, G))
    zmax = comm.all_reduce_max(shard.begin(q))
    cz, cn = shard.candidates(q, zmax)
    tau = shard.threshold(comm.all_gather(cz), comm.all_gather(cn), zmax)
    return comm.all_reduce_sum(shard.finish(q, zmax, tau))
