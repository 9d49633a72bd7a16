"""Seeded synthetic inputs for the DSA workloads.

This module draws random numbers and lays out caches; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle may be fed from it.

Value distributions follow the workloads the method is sized for (Step-5-Preview's
full-attention layers): index_k, index_q, Q, K and V are bf16 ~ N(0, 1), indexer gates
z ~ U(0, 1); K/V live in a paged cache of 64-token pages whose block table is either the
identity or a seeded random permutation of the page pool.

Layouts (all contiguous):
  index_k      bf16  [tokens][4][256]       token rows of one or more requests
  index_q      bf16  [nq][16][256]
  gate         fp32  [nq][16]
  q            bf16  [nq][64][192]
  k_cache/v    bf16  [pages][4][64][192]
  block_table  int32 [B][max_pages]
  summaries    e4m3  [slots][4][256] (uint8), scales fp32 [slots][4]
"""
from __future__ import annotations

import math
import torch

REGION, G, DI, HI, HQ, D, PAGE = 8, 4, 256, 16, 64, 192, 64


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    """bf16 tensor ~ N(0,1), drawn in chunks to bound fp32 temporaries."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    chunk = 1 << 26
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        flat[s:e].copy_(torch.randn(e - s, generator=gen, device=device, dtype=torch.float32))
    return out


def uniform_f32(shape, gen: torch.Generator, device) -> torch.Tensor:
    return torch.rand(shape, generator=gen, device=device, dtype=torch.float32)


def paged_kv(capacity, gen, device, permute: bool) -> tuple:
    """Page pool for requests of the given token capacities.  Returns (block_table,
    k_cache, v_cache).  K/V of every page are N(0,1) bf16."""
    pages_per = [max(1, math.ceil(c / PAGE)) for c in capacity]
    n_pages = sum(pages_per)
    max_pages = max(pages_per)
    order = (torch.randperm(n_pages, generator=gen, device=gen.device)
             if permute else torch.arange(n_pages, device=device))
    order = order.to(device=device, dtype=torch.int32)
    bt = torch.zeros((len(capacity), max_pages), dtype=torch.int32, device=device)
    off = 0
    for b, n in enumerate(pages_per):
        bt[b, :n] = order[off: off + n]
        off += n
    kc = normal_bf16((n_pages, G, PAGE, D), gen, device)
    vc = normal_bf16((n_pages, G, PAGE, D), gen, device)
    return bt, kc, vc


def decode_batch(lengths, seed: int, device, permute: bool = True, extra_tokens: int = 0):
    """Inputs for one decode query per request.  Request b holds lengths[b] tokens
    (positions 0..L_b-1); its query sits at position L_b - 1 (its K/V and index_k are
    already in the cache).  extra_tokens reserves room for appended tokens.

    Returns a dict of tensors (see module docstring for layouts) plus bookkeeping:
      tok_base[b], sum_base[b], n_slots, q_pos, q_req."""
    gen = generator(seed, device)
    B = len(lengths)
    cap = [int(L) + int(extra_tokens) for L in lengths]
    bt, kc, vc = paged_kv(cap, gen, device, permute)
    tok_base, sum_base, t, s = [], [], 0, 0
    for c in cap:
        tok_base.append(t)
        sum_base.append(s)
        t += c
        s += math.ceil(c / REGION)
    index_k = normal_bf16((t, G, DI), gen, device)
    index_q = normal_bf16((B, HI, DI), gen, device)
    gate = uniform_f32((B, HI), gen, device)
    q = normal_bf16((B, HQ, D), gen, device)
    q_pos = torch.tensor([int(L) - 1 for L in lengths], dtype=torch.int32, device=device)
    q_req = torch.arange(B, dtype=torch.int32, device=device)
    return dict(block_table=bt, k_cache=kc, v_cache=vc, index_k=index_k, index_q=index_q,
                gate=gate, q=q, q_pos=q_pos, q_req=q_req,
                tok_base=tok_base, sum_base=torch.tensor(sum_base, dtype=torch.int64, device=device),
                n_slots=s, lengths=[int(L) for L in lengths], capacity=cap)


def complete_regions(lengths, tok_base, sum_base):
    """Host bookkeeping: for each request, the complete regions of its first L tokens.
    Returns (src_row, dst_slot) int64 lists: region r of request b is rows
    tok_base[b]+8r .. +7 and goes to slot sum_base[b]+r."""
    src, dst = [], []
    sb = [int(x) for x in (sum_base.tolist() if hasattr(sum_base, "tolist") else sum_base)]
    for b, L in enumerate(lengths):
        n = int(L) // REGION
        src.extend(int(tok_base[b]) + REGION * r for r in range(n))
        dst.extend(sb[b] + r for r in range(n))
    return src, dst


def prefill_chunk(ctx_len: int, n_new: int, seed: int, device, permute: bool = True, region_shared_q: bool = False):
    """One request with ctx_len tokens already cached and n_new new tokens appended in
    one chunk (positions ctx_len .. ctx_len+n_new-1).  index_k/K/V cover all
    ctx_len+n_new tokens; index_q/gate/Q exist for the n_new queries.
    region_shared_q: the queries of one region share their indexer query and gates (the
    locality variant: neighbouring tokens select the same regions)."""
    gen = generator(seed, device)
    total = ctx_len + n_new
    bt, kc, vc = paged_kv([total], gen, device, permute)
    index_k = normal_bf16((total, G, DI), gen, device)
    index_q = normal_bf16((n_new, HI, DI), gen, device)
    gate = uniform_f32((n_new, HI), gen, device)
    if region_shared_q:
        first = torch.arange(ctx_len, total, device=device) // REGION * REGION - ctx_len
        first = first.clamp(min=0)
        index_q = index_q[first].contiguous()
        gate = gate[first].contiguous()
    q = normal_bf16((n_new, HQ, D), gen, device)
    q_pos = torch.arange(ctx_len, total, dtype=torch.int32, device=device)
    q_req = torch.zeros(n_new, dtype=torch.int32, device=device)
    return dict(block_table=bt, k_cache=kc, v_cache=vc, index_k=index_k, index_q=index_q,
                gate=gate, q=q, q_pos=q_pos, q_req=q_req, tok_base=[0],
                sum_base=torch.zeros(1, dtype=torch.int64, device=device),
                n_slots=math.ceil(total / REGION), lengths=[total], capacity=[total],
                ctx_len=ctx_len, n_new=n_new)


def ragged_lengths(n_req: int, seed: int, lo: int = 4096, hi: int = 1 << 20):
    """Lengths log-uniform in [lo, hi]: L = 8*floor(exp(U(ln lo, ln hi))/8) + tail,
    tail ~ U{0..7}, so a request may end inside an incomplete region."""
    gen = generator(seed, "cpu")
    u = torch.rand(n_req, generator=gen, dtype=torch.float64)
    tails = torch.randint(0, REGION, (n_req,), generator=gen)
    out = []
    for i in range(n_req):
        x = math.exp(math.log(lo) + float(u[i]) * (math.log(hi) - math.log(lo)))
        L = REGION * int(x // REGION) + int(tails[i])
        out.append(max(REGION, min(L, hi - REGION)))
    return out
