"""Seeded synthetic inputs for the fp8 MQA indexer.

This module only draws random inputs; it holds none of the indexer's
arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle consume
what it returns, so they always see the same bytes.

Shapes and value distributions follow the "bench_mqa_logits_chunking.py"
page (`_build`, `SCENARIOS`): H = 32 index heads, D = 128, top-k = 2048;
q and k are standard normal samples clamped to [-2, 2] and cast to fp8
e4m3fn; key scales are U[0,1) + 0.5; head weights are U[0,1); ks = 0 and
ke[i] = rank_start + i + 1 clamped to n (the last context-parallel slice of
an 8-way in-sequence split sees the full key set).  Everything is drawn on
the CPU with a seeded ``torch.Generator`` so the data do not depend on the
GPU.  Draw order: q, k, s, w (prefill); lengths, page permutation, q,
key pages, page scales, w (paged).
"""
from __future__ import annotations

import dataclasses

import torch

H = 32
D = 128
TOPK = 2048
PAGE_SIZE = 64


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    name: str
    m: int
    n: int
    rank_start: int


@dataclasses.dataclass(frozen=True)
class PagedShape:
    name: str
    B: int
    R: int
    lmin: int
    lmax: int


# The five workloads, by index.  Seeds are 20260 + index.
WORKLOADS = {
    0: PrefillShape("tiny_ragged_prefill_m16_n4096", 16, 4096, 4096 - 16),
    1: PrefillShape("causal_prefill_m8192_n35000", 8192, 35000, 35000 - 8192),
    2: PrefillShape("cp8_rank_slice_m8192_n65536", 8192, 65536, 57344),
    3: PrefillShape("cp8_rank_slice_m7500_n210000", 7500, 210000, 202500),
    4: PagedShape("paged_decode_b64_r4_l4096_131072", 64, 4, 4096, 131072),
}


def seed_of(index: int) -> int:
    return 20260 + index


def _fp8_bytes(x: torch.Tensor) -> torch.Tensor:
    """clamp(-2, 2) then torch's e4m3fn cast; returned as raw bytes (uint8)."""
    return x.clamp(-2, 2).to(torch.float8_e4m3fn).view(torch.uint8)


def make_prefill(m: int, n: int, seed: int, rank_start: int | None = None, ks=None, ke=None,
                 heads: int = H, dim: int = D, duplicate_keys: bool = False,
                 signed_weights: bool = False) -> dict:
    """Ragged-prefill inputs as CPU tensors.

    q [m, heads, dim] uint8, k [n, dim] uint8, s [n] f32, w [m, heads] f32,
    ks/ke [m] int32.  By default ks = 0 and ke[i] = rank_start + i + 1
    clamped to n (rank_start defaults to n - m, a causal tail).  Explicit
    ks/ke override the defaults.  duplicate_keys=True makes every key the
    same vector with scale 1 (a degenerate all-ties case).
    signed_weights=True draws w ~ U[-1, 1) instead of U[0, 1).
    """
    g = torch.Generator().manual_seed(seed)
    q = _fp8_bytes(torch.randn(m, heads, dim, generator=g))
    k = _fp8_bytes(torch.randn(n, dim, generator=g))
    s = torch.rand(n, generator=g) + 0.5
    w = torch.rand(m, heads, generator=g)
    if signed_weights:
        w = 2.0 * w - 1.0
    if duplicate_keys and n > 0:
        k = k[:1].expand(n, dim).contiguous()
        s = torch.ones(n)
    if rank_start is None:
        rank_start = n - m
    if ks is None:
        ks = torch.zeros(m, dtype=torch.int32)
    if ke is None:
        ke = (torch.arange(m, dtype=torch.int64) + rank_start + 1).clamp(max=n).to(torch.int32)
    ks = torch.as_tensor(ks, dtype=torch.int32).contiguous()
    ke = torch.as_tensor(ke, dtype=torch.int32).contiguous()
    return dict(q=q.contiguous(), k=k.contiguous(), s=s.contiguous(), w=w.contiguous(), ks=ks,
                ke=ke, m=m, n=n)


def make_paged(B: int, R: int, lmin: int, lmax: int, seed: int, page_size: int = PAGE_SIZE,
               heads: int = H, dim: int = D, lengths=None, max_blocks: int | None = None,
               signed_weights: bool = False) -> dict:
    """Paged-decode inputs as CPU tensors.

    Context lengths L_b ~ U{lmin..lmax} (both ends inclusive) unless given.
    Request b owns ceil(L_b / page_size) pages; all pages are handed out by
    one seeded random permutation.  block_table [B, max_blocks] int32 holds
    the physical page of each logical page, padded with -1.  k_pages
    [P, page_size, dim] uint8, s_pages [P, page_size] f32, q [B*R, heads,
    dim] uint8, w [B*R, heads] f32, seq_lens [B] int32.  signed_weights=True
    draws w ~ U[-1, 1) instead of U[0, 1).
    """
    g = torch.Generator().manual_seed(seed)
    if lengths is None:
        lengths = torch.randint(lmin, lmax + 1, (B,), generator=g, dtype=torch.int64)
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    pages_per = (lengths + page_size - 1) // page_size
    P = int(pages_per.sum())
    if max_blocks is None:
        max_blocks = max(1, (lmax + page_size - 1) // page_size)
    perm = torch.randperm(P, generator=g).to(torch.int32)
    block_table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        c = int(pages_per[b])
        block_table[b, :c] = perm[off:off + c]
        off += c
    q = _fp8_bytes(torch.randn(B * R, heads, dim, generator=g))
    k_pages = _fp8_bytes(torch.randn(max(P, 1), page_size, dim, generator=g))
    s_pages = torch.rand(max(P, 1), page_size, generator=g) + 0.5
    w = torch.rand(B * R, heads, generator=g)
    if signed_weights:
        w = 2.0 * w - 1.0
    return dict(q=q.contiguous(), k_pages=k_pages.contiguous(), s_pages=s_pages.contiguous(),
                w=w.contiguous(), block_table=block_table.contiguous(),
                seq_lens=lengths.to(torch.int32).contiguous(), B=B, R=R, P=P,
                page_size=page_size, max_blocks=max_blocks)


def make_workload(index: int) -> dict:
    """The named workload `index` (0..4) with its fixed seed."""
    shape = WORKLOADS[index]
    if isinstance(shape, PrefillShape):
        d = make_prefill(shape.m, shape.n, seed_of(index), rank_start=shape.rank_start)
    else:
        d = make_paged(shape.B, shape.R, shape.lmin, shape.lmax, seed_of(index))
    d["name"] = shape.name
    d["seed"] = seed_of(index)
    return d
