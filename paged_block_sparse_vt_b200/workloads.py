"""Seeded synthetic decode workloads shaped like the Vortex block top-k decode setting.

This module only draws inputs: it holds none of the method's arithmetic, and
both the CUDA path and the CPU oracle are fed from it.  All data comes from CPU
``torch.Generator`` objects: one seeded with ``seed = 1000 + cfg`` draws, in this
order, seq_lens, the page permutation, q and the per-page offsets (config 2
only); the K and V pools are drawn in fixed chunks of pages, chunk ``i`` of
pool ``s`` (1 = K, 2 = V) from its own generator seeded with
``seed * 1000003 + 7919 * s + i``, so the pools can be filled by several host
threads and still come out identical.

The five workloads (page size 16 everywhere; bf16 q/K/V; fp32 centroids):

====  =============================  ===========================================================
cfg   shape                          recipe
====  =============================  ===========================================================
1     B=1, Hq=2, Hkv=1, D=64         L=1024 (64 full pages) scattered in a 128-page pool; k=4+1+1
2     B=32, Hq=16, Hkv=8, D=128      L ~ U{4096..16384}; 40,000-page shuffled pool; k=30+1+1;
                                     K and V are N(0,1) plus an N(0, 0.5^2) offset vector drawn
                                     per (physical page, KV head), independently for K and V
3     B=128, Hq=32, Hkv=8, D=128     L=32768 (2048 pages) each; pool of exactly 262,144 pages; k=64+1+1
4     B=64, Hq=32, Hkv=1, D=576/512  MLA absorbed form: K row = [latent 512 ; rope 64], V = K[:512];
                                     L=16384 (1024 pages); 65,536-page pool; k=32+1+1
5     B=256, Hq=48, Hkv=8, D=128     L = floor(exp(U(ln 512, ln 65536))); 16 seeded requests end
                                     exactly on a page boundary (their last page fills this step),
                                     every other length that would end on a boundary is cut by one;
                                     pool = 1.25 x pages in use; k=30+1+1
====  =============================  ===========================================================

The pages' own measurements use real models on AMC23 / AIME24 / AIME26; none of
that is available here, and these synthetic batches stand in for them.

``poison=True`` (parity runs) fills every pool page that belongs to no request,
and every token slot past the end of a request's last page, with NaN, so that a
wrong gather shows up in the output instead of passing silently.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace
from typing import Optional

import torch

PAGE_SIZE = 16


@dataclass(frozen=True)
class Config:
    cfg: int
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    Dv: int
    topk: int
    bos: int
    eos: int
    sm_scale: float
    lengths: str            # "fixed", "uniform", "loguniform"
    len_lo: int             # tokens
    len_hi: int             # tokens (inclusive)
    pool_pages: Optional[int]   # None: 1.25 x pages in use
    page_offsets: float     # std of the per-(page, head) offset added to K and V (0: none)
    mla: bool = False       # V is the first Dv dims of the K row (one shared pool)
    filled: int = 0         # requests whose last page fills at this step (cfg 5 recipe)
    explicit: tuple = ()    # lengths="explicit": the seq_lens themselves (edge-case batches)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def kmax(self) -> int:
        return self.topk + self.bos + self.eos


CONFIGS = {
    1: Config(1, "tiny", B=1, Hq=2, Hkv=1, D=64, Dv=64, topk=4, bos=1, eos=1,
              sm_scale=1.0 / 8.0, lengths="fixed", len_lo=1024, len_hi=1024, pool_pages=128,
              page_offsets=0.0),
    2: Config(2, "qwen3-0.6b-like", B=32, Hq=16, Hkv=8, D=128, Dv=128, topk=30, bos=1, eos=1,
              sm_scale=1.0 / math.sqrt(128), lengths="uniform", len_lo=4096, len_hi=16384,
              pool_pages=40000, page_offsets=0.5),
    3: Config(3, "long-context", B=128, Hq=32, Hkv=8, D=128, Dv=128, topk=64, bos=1, eos=1,
              sm_scale=1.0 / math.sqrt(128), lengths="fixed", len_lo=32768, len_hi=32768,
              pool_pages=262144, page_offsets=0.0),
    4: Config(4, "mla-latent", B=64, Hq=32, Hkv=1, D=576, Dv=512, topk=32, bos=1, eos=1,
              sm_scale=1.0 / math.sqrt(576), lengths="fixed", len_lo=16384, len_hi=16384,
              pool_pages=65536, page_offsets=0.0, mla=True),
    5: Config(5, "heterogeneous", B=256, Hq=48, Hkv=8, D=128, Dv=128, topk=30, bos=1, eos=1,
              sm_scale=1.0 / math.sqrt(128), lengths="loguniform", len_lo=512, len_hi=65536,
              pool_pages=None, page_offsets=0.0, filled=16),
}


def config(cfg: int, **overrides) -> Config:
    """The named workload, optionally shrunk (B, lengths, pool size) for parity runs."""
    return replace(CONFIGS[cfg], **overrides)


def _seq_lens(c: Config, gen: torch.Generator) -> torch.Tensor:
    if c.lengths == "fixed":
        L = torch.full((c.B,), c.len_lo, dtype=torch.int64)
    elif c.lengths == "explicit":
        assert len(c.explicit) == c.B
        L = torch.tensor(c.explicit, dtype=torch.int64)
    elif c.lengths == "uniform":
        L = torch.randint(c.len_lo, c.len_hi + 1, (c.B,), generator=gen, dtype=torch.int64)
    elif c.lengths == "loguniform":
        u = torch.rand((c.B,), generator=gen, dtype=torch.float64)
        L = torch.floor(torch.exp(math.log(c.len_lo) + u * (math.log(c.len_hi) - math.log(c.len_lo))))
        L = L.to(torch.int64).clamp(c.len_lo, c.len_hi)
    else:
        raise ValueError(c.lengths)
    if c.filled:
        # the seeded requests whose newest token completes a page; nobody else ends on a boundary
        chosen = torch.randperm(c.B, generator=gen)[: c.filled]
        on_boundary = (L % PAGE_SIZE) == 0
        L = torch.where(on_boundary, L - 1, L)
        L[chosen] = ((L[chosen] + PAGE_SIZE - 1) // PAGE_SIZE) * PAGE_SIZE
    return L.to(torch.int32)


def _normal(n: int, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(n, generator=gen, device=device, dtype=torch.float32)


def _fill_pool(pool: torch.Tensor, seed: int, stream: int, offsets: Optional[torch.Tensor]) -> None:
    """pool[P,16,H,D] <- bf16(N(0,1) [+ offsets[p,h,:] broadcast over the page's tokens])."""
    P, T, H, D = pool.shape
    pages_per_chunk = max(1, (1 << 22) // (T * H * D))

    def chunk(i: int) -> None:
        p0, p1 = i * pages_per_chunk, min(P, (i + 1) * pages_per_chunk)
        g = torch.Generator(device="cpu")
        g.manual_seed(seed * 1000003 + 7919 * stream + i)
        x = _normal((p1 - p0) * T * H * D, g, "cpu").view(p1 - p0, T, H, D)
        if offsets is not None:
            x += offsets[p0:p1].unsqueeze(1)
        pool[p0:p1].copy_(x)

    n_chunks = (P + pages_per_chunk - 1) // pages_per_chunk
    workers = min(n_chunks, max(1, len(os.sched_getaffinity(0))))
    if workers <= 1:
        for i in range(n_chunks):
            chunk(i)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(chunk, range(n_chunks)))


def make_workload(cfg: int | Config, device="cpu", poison: bool = False, seed: Optional[int] = None,
                  **overrides) -> dict:
    """Draw one decode-step workload.  Returns a dict of tensors on ``device`` plus sizes.

    Keys: ``config`` (Config), ``q`` [B,Hq,D] bf16, ``k_pool`` [P,16,Hkv,D] bf16, ``v_pool``
    (the same tensor as ``k_pool`` for MLA, whose V is ``k_pool[..., :Dv]``), ``page_table``
    [B, max_pages] int32 (logical -> physical page; unused tail entries point at a spare page
    when one exists), ``seq_lens`` [B] int32 (tokens, including the one being decoded),
    ``prebuilt_pages`` (physical ids of pages that were full before this step),
    ``fill_pages`` (physical ids of pages that fill at this step), ``pad_page``.
    """
    c = cfg if isinstance(cfg, Config) else config(cfg, **overrides)
    gen_device = torch.device(device)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(1000 + c.cfg if seed is None else seed)

    L = _seq_lens(c, gen)
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    used = int(n.sum())
    P = c.pool_pages if c.pool_pages is not None else int(math.ceil(1.25 * used))
    if P < used:
        raise ValueError(f"pool of {P} pages cannot hold the {used} pages in use")
    perm = torch.randperm(P, generator=gen).to(torch.int32)

    max_pages = int(n.max())
    pad_page = int(perm[used]) if P > used else 0
    page_table = torch.full((c.B, max_pages), pad_page, dtype=torch.int32)
    # pages 0..n-2 of a request are full and were summarised at earlier steps; a request
    # whose length is a multiple of the page size has just completed its last page, whose
    # centroid is built at this step
    prebuilt, filled = [], []
    off = 0
    for b in range(c.B):
        nb = int(n[b])
        page_table[b, :nb] = perm[off: off + nb]
        prebuilt.append(perm[off: off + nb - 1])
        if int(L[b]) % PAGE_SIZE == 0:
            filled.append(perm[off + nb - 1: off + nb])
        off += nb
    prebuilt = torch.cat(prebuilt) if prebuilt else torch.zeros(0, dtype=torch.int32)
    filled = torch.cat(filled) if filled else torch.zeros(0, dtype=torch.int32)

    # values: q, then the per-page offsets (if any) from the main generator; K and V from
    # their per-chunk generators; always drawn on the host, whatever the target device
    q = _normal(c.B * c.Hq * c.D, gen, "cpu").view(c.B, c.Hq, c.D).to(torch.bfloat16)
    koff = voff = None
    if c.page_offsets:
        koff = (c.page_offsets * _normal(P * c.Hkv * c.D, gen, "cpu")).view(P, c.Hkv, c.D)
        voff = (c.page_offsets * _normal(P * c.Hkv * c.Dv, gen, "cpu")).view(P, c.Hkv, c.Dv)
    base_seed = 1000 + c.cfg if seed is None else seed
    k_pool = torch.empty((P, PAGE_SIZE, c.Hkv, c.D), dtype=torch.bfloat16)
    _fill_pool(k_pool, base_seed, 1, koff)
    if c.mla:
        v_pool = k_pool
    else:
        v_pool = torch.empty((P, PAGE_SIZE, c.Hkv, c.Dv), dtype=torch.bfloat16)
        _fill_pool(v_pool, base_seed, 2, voff)

    if poison:
        in_use = torch.zeros(P, dtype=torch.bool)
        in_use[perm[:used].long()] = True
        k_pool[~in_use] = float("nan")
        if not c.mla:
            v_pool[~in_use] = float("nan")
        for b in range(c.B):
            valid = int(L[b]) - PAGE_SIZE * (int(n[b]) - 1)
            last = int(page_table[b, int(n[b]) - 1])
            k_pool[last, valid:] = float("nan")
            if not c.mla:
                v_pool[last, valid:] = float("nan")

    out = dict(config=c, P=P, pad_page=pad_page, q=q, k_pool=k_pool, v_pool=v_pool,
               page_table=page_table, seq_lens=L, prebuilt_pages=prebuilt, fill_pages=filled)
    if gen_device.type != "cpu":
        for key in ("q", "k_pool", "page_table", "seq_lens", "prebuilt_pages", "fill_pages"):
            out[key] = out[key].to(gen_device)
        out["v_pool"] = out["k_pool"] if c.mla else out["v_pool"].to(gen_device)
    return out


def empty_centroids(c: Config, P: int, device="cpu", fill: float = float("nan")) -> torch.Tensor:
    """A centroid cache [P, Hkv, D] fp32, every row set to ``fill`` (NaN: "never built")."""
    return torch.full((P, c.Hkv, c.D), fill, dtype=torch.float32, device=device)
