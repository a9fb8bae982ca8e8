"""Seeded synthetic decode workloads shaped like the EntmaxKV efficiency setting.

This module only draws inputs: a paged bf16 K/V cache, one bf16 query per
(batch, query head), a page table and per-sequence lengths.  It holds none of
the method's arithmetic (no scores, no thresholds, no selection), so both the
CUDA path and the CPU oracle can be fed from it.

The five workload families follow the EntmaxKV technical summary (gist.science
paper 2605.21649, section 4 "Key results / Efficiency": long-context decode up
to 1M tokens).  The pages name no dataset shapes, so every shape below is a
synthetic stand-in:

* ``offset`` keys: N(0,1) per coordinate plus one scalar N(0, 0.5^2) offset per
  logical page added to every coordinate of that page.
* ``cluster`` keys: 256 centroids N(0,1)^d per (batch, kv head); the sequence is
  cut into page-contiguous runs of 1..8 pages, each run drawing one centroid,
  and every key is its centroid plus N(0, 0.3^2) noise.  The query of each head
  sits near one centroid of its kv head (plus N(0, 0.5^2)).
* needles: per query head, ``needles`` key slots (distinct across the heads of
  one GQA group) are overwritten with ``needle_scale * sqrt(d) * q / |q|`` so
  the entmax support is small and known to be there.

Values are N(0,1).  All draws come from one ``torch.Generator`` seeded by the
caller; bf16 rounding is round-to-nearest-even (``Tensor.to(torch.bfloat16)``).
Logical pages are scattered over physical blocks by a seeded permutation so
that page loads really are gathers.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L: int
    P: int
    alpha: float
    policy: str            # "topk", "gauss" or "dense"
    k: int = 0             # top-k budget in pages
    delta: float = 0.0     # Gaussian safety margin (z scale)
    keys: str = "offset"   # "offset" or "cluster"
    needles: int = 0       # per query head
    needle_scale: float = 3.0
    ragged: bool = False   # per-sequence lengths below L, not page aligned
    n_centroids: int = 256
    notes: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_pages(self) -> int:
        return (self.L + self.P - 1) // self.P

    @property
    def num_blocks(self) -> int:
        return self.B * self.max_pages

    def shrink(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workload shapes used by tests and the benchmark.
CONFIGS = {
    "tiny_h1_L4k": Workload("tiny_h1_L4k", B=1, Hq=1, Hkv=1, d=64, L=4096, P=16,
                            alpha=1.5, policy="topk", k=32, keys="offset",
                            needles=8, needle_scale=4.0),
    "dense_gqa_L32k": Workload("dense_gqa_L32k", B=4, Hq=32, Hkv=8, d=128, L=32768,
                               P=32, alpha=1.5, policy="dense", keys="offset",
                               needles=16, needle_scale=3.0),
    "topk_gqa_L128k": Workload("topk_gqa_L128k", B=8, Hq=32, Hkv=8, d=128,
                               L=131072, P=32, alpha=1.5, policy="topk", k=64,
                               keys="cluster", needles=32, needle_scale=3.0),
    "gauss_gqa_L1m": Workload("gauss_gqa_L1m", B=1, Hq=32, Hkv=8, d=128,
                              L=1048576, P=64, alpha=1.5, policy="gauss",
                              delta=0.5, keys="cluster", needles=64,
                              needle_scale=3.0),
    "sweep_mha_L64k": Workload("sweep_mha_L64k", B=16, Hq=32, Hkv=32, d=64,
                               L=65536, P=32, alpha=1.5, policy="topk", k=32,
                               keys="offset", needles=16, needle_scale=3.0),
}


def sweep_points():
    """The (alpha, page size, policy, needles) grid of the MHA sweep shape."""
    pts = []
    for alpha in (1.25, 1.5, 2.0):
        for P in (16, 32, 64):
            for pol in (("topk", 32, 0.0), ("topk", 128, 0.0),
                        ("gauss", 0, 0.25), ("gauss", 0, 1.0)):
                for nd in (1, 16, 256):
                    pts.append(dict(alpha=alpha, P=P, policy=pol[0], k=pol[1],
                                    delta=pol[2], needles=nd))
    return pts


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def make_inputs(wl: Workload, seed: int, device="cpu", sequential_pages: bool = False):
    """Draw one workload instance.  sequential_pages: logical page p of
    sequence b sits in block b * max_pages + p (an identity page table)
    instead of a seeded permutation of the blocks; every other draw is the
    same.

    Returns a dict of tensors on ``device``:
      q          bf16  [B, Hq, d]
      k_cache    bf16  [num_blocks, Hkv, P, d]
      v_cache    bf16  [num_blocks, Hkv, P, d]
      page_table int32 [B, max_pages]   (logical page -> physical block)
      seq_lens   int32 [B]
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    B, Hq, Hkv, d, P = wl.B, wl.Hq, wl.Hkv, wl.d, wl.P
    G = wl.G
    Np = wl.max_pages
    nb = wl.num_blocks

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    def randint(hi, shape):
        return torch.randint(0, hi, shape, generator=g, device=dev)

    perm = torch.randperm(nb, generator=g, device=dev).to(torch.int32)
    if sequential_pages:
        perm = torch.arange(nb, device=dev, dtype=torch.int32)
    page_table = perm.view(B, Np).contiguous()

    if wl.ragged:
        # every sequence shorter than L by a random amount that is not a
        # multiple of the page size (the last page is partial)
        cut = randint(max(1, 3 * P), (B,)) + 1
        seq = (wl.L - cut).clamp(min=1)
    else:
        seq = torch.full((B,), wl.L, device=dev, dtype=torch.int64)
    seq_lens = seq.to(torch.int32)

    k_cache = torch.empty((nb, Hkv, P, d), dtype=torch.bfloat16, device=dev)
    v_cache = torch.empty((nb, Hkv, P, d), dtype=torch.bfloat16, device=dev)
    q = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)

    for b in range(B):
        blocks = page_table[b].long()
        for kvh in range(Hkv):
            if wl.keys == "offset":
                kl = randn(Np, P, d) + 0.5 * randn(Np, 1, 1)
                qh = randn(G, d)
            elif wl.keys == "cluster":
                cents = randn(wl.n_centroids, d)
                # page-contiguous runs of 1..8 pages, one centroid per run
                run_len = randint(8, (Np,)) + 1
                run_cid = randint(wl.n_centroids, (Np,))
                starts = torch.cumsum(run_len, 0) - run_len
                page_run = torch.searchsorted(starts, torch.arange(Np, device=dev),
                                              right=True) - 1
                cid = run_cid[page_run]
                kl = cents[cid].unsqueeze(1) + 0.3 * randn(Np, P, d)
                jstar = randint(wl.n_centroids, (G,))
                qh = cents[jstar] + 0.5 * randn(G, d)
            else:
                raise ValueError(wl.keys)
            qh = _bf16(qh)
            q[b, kvh * G:(kvh + 1) * G] = qh
            vl = randn(Np, P, d)
            if wl.needles > 0:
                L_b = int(seq_lens[b])
                n_tot = G * wl.needles
                if n_tot > L_b:
                    raise ValueError("more needles than tokens")
                pos = torch.randperm(L_b, generator=g, device=dev)[:n_tot].view(G, wl.needles)
                qf = qh.float()
                nk = wl.needle_scale * math.sqrt(d) * qf / qf.norm(dim=1, keepdim=True)
                flat = kl.view(Np * P, d)
                for gi in range(G):
                    flat[pos[gi].long()] = nk[gi]
            k_cache[blocks, kvh] = _bf16(kl)
            v_cache[blocks, kvh] = _bf16(vl)

    return dict(q=q, k_cache=k_cache, v_cache=v_cache, page_table=page_table,
                seq_lens=seq_lens)


def to_host_u16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array holding the same bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")
