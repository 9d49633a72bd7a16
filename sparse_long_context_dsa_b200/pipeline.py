"""Host orchestration of a DSA step over the C-ABI calls (no arithmetic of its own).

A decode step for a batch of requests, one query each, is
    compress the regions that this step completes  (A1, only if any are due)
    indexer scores over every complete region     (A2)  } one call: dsa_decode_select
    top-k with the own region forced              (A3)  }
    sparse attention over the selected regions    (A4)
([P2] Step-5-Preview 如何实现1M长上下文 §区域压缩CSA / §索引器打分).

The region a decode token completes is always the query's own region (token p completes
region p/8 exactly when p % 8 == 7), and the own region is forced, never scored.  So this
step's scan never reads what this step's compression writes, and the compression runs on
a parallel branch (a side stream joined at the end of the step); the next step sees it.
The branch forks after the selection, so the compression shares the GPU with the
attention (64 CTAs at batch 1, most SMs idle) rather than with the scan, whose slowest
CTAs it would delay.

All buffers are allocated once, so a step can be captured in a CUDA graph and replayed.
The per-step inputs live in one device arena (index_q, gate, q, q_pos and, optionally,
the 8-token tails whose regions complete), so a host caller refreshes them with a single
host-to-device copy of `arena`.
"""
from __future__ import annotations

import torch

from . import dsa
from .dsa import G, HQ, D, DI, HI, REGION


def _carve(arena: torch.Tensor, off: int, shape, dtype) -> tuple:
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.tensor([], dtype=dtype).element_size()
    view = arena[off: off + nbytes].view(dtype).view(*shape)
    return view, off + (nbytes + 255) // 256 * 256


class DecodeStep:
    """Buffers and launches of one decode step for fixed shapes.

    summaries/scales: the group-major pool; sum_base int64 [B]; block_table int32 [B][P];
    k_cache/v_cache bf16 [pages][4][64][192]; ld: score row length (>= max own region).
    tail_tokens = 8 gives the step an input tail buffer (bf16 [B*8][4][256]) whose
    regions are compressed when `set_compress` lists them.
    g0: first KV group of a group shard ([P2] §索引器打分: one GPU of a KV-group-sharded decode):
    with summaries [ng][slots][256] and caches [pages][ng][64][192] of groups g0 .. g0+ng-1
    the step runs the `_groups` calls and `out` holds those groups' 16*ng heads."""

    def __init__(self, summaries, scales, sum_base, block_table, k_cache, v_cache, ld, k=512,
                 tail_tokens=0, flags=0, g0=0):
        dev = summaries.device
        self.B = B = int(block_table.shape[0])
        self.g0, self.ng = int(g0), int(summaries.shape[0])
        self.sharded = self.ng != G
        ng = self.ng
        self.k = int(k)
        self.ld = int(ld)
        self.flags = flags
        self.summaries, self.scales, self.sum_base = summaries, scales, sum_base
        self.block_table, self.k_cache, self.v_cache = block_table, k_cache, v_cache
        # per-step inputs: one arena
        size = 0
        for shape, dt in (((B, HI, DI), torch.bfloat16), ((B, HI), torch.float32), ((B, HQ, D), torch.bfloat16),
                          ((B,), torch.int32), ((B * max(tail_tokens, 1), G, DI), torch.bfloat16)):
            n = 1
            for s in shape:
                n *= s
            size += (n * torch.tensor([], dtype=dt).element_size() + 255) // 256 * 256
        self.arena = torch.zeros(size, dtype=torch.uint8, device=dev)
        off = 0
        self.index_q, off = _carve(self.arena, off, (B, HI, DI), torch.bfloat16)
        self.gate, off = _carve(self.arena, off, (B, HI), torch.float32)
        self.q, off = _carve(self.arena, off, (B, HQ, D), torch.bfloat16)
        self.q_pos, off = _carve(self.arena, off, (B,), torch.int32)
        self.tail, off = _carve(self.arena, off, (B * max(tail_tokens, 1), G, DI), torch.bfloat16)
        self.tail_tokens = tail_tokens
        self.q_req = torch.arange(B, dtype=torch.int32, device=dev)
        self.scores = torch.zeros((B, ng, self.ld), dtype=torch.float32, device=dev)
        self.sel_idx = torch.empty((B, ng, self.k), dtype=torch.int32, device=dev)
        self.sel_count = torch.empty((B, ng), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, 16 * ng, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, 16 * ng), dtype=torch.float32, device=dev)
        self.n_compress = 0
        self.src_row = torch.zeros(max(1, B), dtype=torch.int64, device=dev)
        self.dst_slot = torch.zeros(max(1, B), dtype=torch.int64, device=dev)
        self.side = torch.cuda.Stream(device=dev)
        L = dsa.lib()
        self.ws_idx_n = L.dsa_indexer_workspace_size(B, self.ld)
        self.ws_topk_n = L.dsa_topk_workspace_size(B, self.ld, self.k)
        self.ws_sel_n = L.dsa_decode_select_workspace_size(B, self.ld, self.k)
        self.ws_attn_n = (L.dsa_attn_groups_workspace_size(B, self.k, ng) if self.sharded
                          else L.dsa_attn_workspace_size(B, self.k))
        self.ws_idx = torch.empty(max(1, self.ws_idx_n), dtype=torch.uint8, device=dev)
        self.ws_topk = torch.empty(max(1, self.ws_topk_n), dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(max(1, self.ws_attn_n), dtype=torch.uint8, device=dev)
        self.ws_sel = torch.empty(max(1, self.ws_sel_n), dtype=torch.uint8, device=dev)

    def load(self, index_q, gate, q, q_pos, tail=None):
        self.index_q.copy_(index_q, non_blocking=True)
        self.gate.copy_(gate, non_blocking=True)
        self.q.copy_(q, non_blocking=True)
        self.q_pos.copy_(q_pos, non_blocking=True)
        if tail is not None:
            self.tail.copy_(tail, non_blocking=True)

    def stage(self, host_arena):
        """Copies the step's inputs from a pinned host image of `arena` with one library
        kernel (the GPU reads the pinned memory directly), in the stream's kernel chain."""
        dsa.copy(self.arena, host_arena)

    def set_compress(self, requests, slots):
        """Regions to compress this step: tail block i (rows 8i..8i+7 of `tail`) of each
        listed request goes to pool slot slots[j]."""
        n = len(requests)
        if n:
            self.src_row[:n].copy_(torch.tensor([REGION * int(b) for b in requests], dtype=torch.int64))
            self.dst_slot[:n].copy_(torch.tensor([int(s) for s in slots], dtype=torch.int64))
        self.n_compress = n

    def run(self, out=None):
        """Launches the step on the current stream (capturable).  out: where the attention
        writes its output, bf16 [B][64][192], on the device (default `self.out`) or in pinned
        host memory, which the kernel then writes directly."""
        if out is None:
            out = self.out
        elif tuple(out.shape) != tuple(self.out.shape) or out.dtype != self.out.dtype or not (
                out.is_cuda or out.is_pinned()):
            raise ValueError("out must be bf16 [B][16*ng][192], on the device or in pinned host memory")
        L = dsa.lib()
        main = torch.cuda.current_stream()
        p = dsa._p
        st = dsa._stream()
        # scores and selection in one call (the scan's chunk maxima bound the selection)
        if self.sharded:
            dsa._check(L.dsa_decode_select_groups(p(self.index_q), p(self.gate), p(self.q_req), p(self.q_pos), self.B,
                                                  self.g0, self.ng, p(self.summaries), p(self.scales),
                                                  self.summaries.shape[1], p(self.sum_base), self.sum_base.numel(),
                                                  p(self.scores), self.ld, self.flags, self.k, p(self.sel_idx),
                                                  p(self.sel_count), p(self.ws_sel), self.ws_sel_n, st))
        else:
            dsa._check(L.dsa_decode_select(p(self.index_q), p(self.gate), p(self.q_req), p(self.q_pos), self.B,
                                           p(self.summaries), p(self.scales), self.summaries.shape[1],
                                           p(self.sum_base), self.sum_base.numel(), p(self.scores), self.ld,
                                           self.flags, self.k, p(self.sel_idx), p(self.sel_count), p(self.ws_sel),
                                           self.ws_sel_n, st))
        if self.n_compress:
            self.side.wait_stream(main)
            with torch.cuda.stream(self.side):
                t = self.tail
                if self.sharded:
                    dsa._check(L.dsa_compress_regions_groups(p(t), t[0].numel(), t.shape[0], p(self.src_row),
                                                             p(self.dst_slot), self.n_compress, self.g0, self.ng,
                                                             p(self.summaries), p(self.scales),
                                                             self.summaries.shape[1], dsa._stream()))
                else:
                    dsa._check(L.dsa_compress_regions(p(t), t[0].numel(), t.shape[0], p(self.src_row),
                                                      p(self.dst_slot), self.n_compress, p(self.summaries),
                                                      p(self.scales), self.summaries.shape[1], dsa._stream()))
        self.run_attention(out)
        if self.n_compress:
            main.wait_stream(self.side)
        return out

    def run_attention(self, out=None):
        """The step's attention alone, over the selection in sel_idx / sel_count."""
        L, p, st = dsa.lib(), dsa._p, dsa._stream()
        out = self.out if out is None else out
        if self.sharded:
            dsa._check(L.dsa_sparse_attn_decode_groups(p(self.q), p(self.k_cache), p(self.v_cache),
                                                       self.k_cache.shape[0], p(self.block_table),
                                                       self.block_table.shape[1], p(self.q_pos), self.B, self.g0,
                                                       self.ng, p(self.sel_idx), p(self.sel_count), self.k, p(out),
                                                       p(self.lse), p(self.ws_attn), self.ws_attn_n, st))
        else:
            dsa._check(L.dsa_sparse_attn_decode(p(self.q), p(self.k_cache), p(self.v_cache), self.k_cache.shape[0],
                                                p(self.block_table), self.block_table.shape[1], p(self.q_pos), self.B,
                                                p(self.sel_idx), p(self.sel_count), self.k, p(out), p(self.lse),
                                                p(self.ws_attn), self.ws_attn_n, st))
        return out


def compress_all(index_k, lengths, tok_base, sum_base, summaries, scales):
    """Compresses every complete region of every request (cache set-up)."""
    src, dst = [], []
    sb = sum_base.tolist()
    for b, L in enumerate(lengths):
        n = int(L) // REGION
        src.append(torch.arange(n, dtype=torch.int64) * REGION + int(tok_base[b]))
        dst.append(torch.arange(n, dtype=torch.int64) + int(sb[b]))
    src = torch.cat(src).to(index_k.device)
    dst = torch.cat(dst).to(index_k.device)
    dsa.compress_regions(index_k, src, dst, summaries, scales)


def due_regions(positions):
    """Requests whose appended token (at the given 0-based positions) completes a region:
    token p completes region p // 8 exactly when p % 8 == 7."""
    return [b for b, p in enumerate(positions) if int(p) % REGION == REGION - 1]


class StreamingDecode:
    """The streaming summary update of a ragged decode batch ([P2] Step-5-Preview 如何实现1M长上下文
    §区域压缩CSA, update_summaries_decode): a region is summarised exactly when its 8th token
    arrives; the tail of fewer than 8 tokens waits and is never summarised.

    lengths[b] tokens of request b are cached.  Each step appends one token per request at
    position p_b = lengths[b] (the caller writes its K/V into the paged cache and its
    index_k row into row p_b % 8 of tail block b of `step.tail`), queries at p_b, and
    compresses region p_b / 8 of the requests whose token completes it (p_b % 8 == 7) from
    their tail blocks.  That region is the query's own region, which its scan never reads,
    so the compression runs on the step's parallel branch."""

    def __init__(self, summaries, scales, sum_base, block_table, k_cache, v_cache, lengths, ld, k=512):
        self.lengths = [int(L) for L in lengths]
        self.sum_base = [int(x) for x in sum_base.tolist()]
        self.step = DecodeStep(summaries, scales, sum_base, block_table, k_cache, v_cache, ld, k=k, tail_tokens=8)

    def positions(self):
        """Positions of the tokens the next step appends (= its query positions)."""
        return list(self.lengths)

    def run(self, index_q, gate, q):
        """One step: the tail blocks must already hold the new tokens' index_k rows."""
        pos = self.positions()
        due = due_regions(pos)
        self.step.load(index_q, gate, q, torch.tensor(pos, dtype=torch.int32))
        self.step.set_compress(due, [self.sum_base[b] + pos[b] // REGION for b in due])
        out = self.step.run()
        self.lengths = [L + 1 for L in self.lengths]
        return out, due


def ring_block_table(batch: int, max_pages: int, ring_pages: int = 8, device="cuda") -> torch.Tensor:
    """Block table of per-request rings: request b's virtual page v maps to physical page
    b * ring_pages + v % ring_pages, so with 64-token pages a ring of 8 pages holds the last
    512 tokens and token t overwrites the slot of token t - 512 ([P2] Step-5-Preview
    如何实现1M长上下文 §第一招: the window layers' ring buffer)."""
    b = torch.arange(batch, dtype=torch.int32)[:, None]
    v = torch.arange(max_pages, dtype=torch.int32)[None, :]
    return (b * ring_pages + v % ring_pages).to(device)


class WindowDecodeStep:
    """One decode step of a window layer for a batch of requests, one token each: the new
    token's K/V into the request's ring, then GQA over its last `window` tokens, in one call
    (dsa_window_decode).  Buffers are allocated once (capturable in a CUDA graph).

    k_ring/v_ring: bf16 [B * ring_pages][4][64][192]; block_table: ring_block_table(...).
    Per-step inputs: q bf16 [B][64][192], new_k/new_v bf16 [B][4][192], q_pos int32 [B]."""

    def __init__(self, k_ring, v_ring, block_table, window: int = 512):
        dev = k_ring.device
        self.B = B = block_table.shape[0]
        self.k_ring, self.v_ring, self.block_table, self.window = k_ring, v_ring, block_table, window
        # per-step inputs in one arena (q, new_k, new_v, q_pos): one copy stages a step
        shapes = (((B, HQ, D), torch.bfloat16), ((B, G, D), torch.bfloat16), ((B, G, D), torch.bfloat16),
                  ((B,), torch.int32))
        size = 0
        for shape, dt in shapes:
            n = 1
            for x in shape:
                n *= x
            size += (n * torch.tensor([], dtype=dt).element_size() + 255) // 256 * 256
        self.arena = torch.zeros(size, dtype=torch.uint8, device=dev)
        off = 0
        self.q, off = _carve(self.arena, off, (B, HQ, D), torch.bfloat16)
        self.new_k, off = _carve(self.arena, off, (B, G, D), torch.bfloat16)
        self.new_v, off = _carve(self.arena, off, (B, G, D), torch.bfloat16)
        self.q_pos, off = _carve(self.arena, off, (B,), torch.int32)
        self.out = torch.empty((self.B, HQ, D), dtype=torch.bfloat16, device=dev)
        L = dsa.lib()
        self.ws_n = L.dsa_window_attn_workspace_size(self.B, window)
        self.ws = torch.empty(max(1, self.ws_n), dtype=torch.uint8, device=dev)

    def load(self, q, new_k, new_v, q_pos):
        self.q.copy_(q, non_blocking=True)
        self.new_k.copy_(new_k, non_blocking=True)
        self.new_v.copy_(new_v, non_blocking=True)
        self.q_pos.copy_(q_pos, non_blocking=True)

    def stage(self, host_arena):
        """Copies the step's inputs from a pinned host image of `arena` with one library
        kernel, in the stream's kernel chain."""
        dsa.copy(self.arena, host_arena)

    def run(self, out=None):
        """Launches the step (capturable).  out: bf16 [B][64][192] on the device (default
        `self.out`) or in pinned host memory, which the kernel then writes directly."""
        if out is None:
            out = self.out
        elif tuple(out.shape) != tuple(self.out.shape) or out.dtype != self.out.dtype or not (
                out.is_cuda or out.is_pinned()):
            raise ValueError("out must be bf16 [B][64][192], on the device or in pinned host memory")
        L, p, st = dsa.lib(), dsa._p, dsa._stream()
        kr, bt = self.k_ring, self.block_table
        # the append and the window attention in one call (one kernel where the clustered
        # window kernel serves the batch)
        dsa._check(L.dsa_window_decode(p(kr), p(self.v_ring), kr.shape[0], p(bt), bt.shape[1], self.B, None,
                                       p(self.q_pos), self.B, p(self.new_k), p(self.new_v), p(self.q), self.window,
                                       p(out), None, p(self.ws), self.ws_n, st))
        return out
