"""Host orchestration of a DSA step over the C-ABI calls (no arithmetic of its own).

A decode step for a batch of requests, one query each, is
    compress the regions that this step completes  (A1, only if any are due)
    indexer scores over every complete region     (A2)
    top-k with the own region forced              (A3)
    sparse attention over the selected regions    (A4)
([P2] Step-5-Preview 如何实现1M长上下文 §区域压缩CSA / §索引器打分).  All buffers are
allocated once, so a step can be captured in a CUDA graph and replayed.
"""
from __future__ import annotations

import torch

from . import dsa
from .dsa import G, HQ, D, REGION


class DecodeStep:
    """Buffers and launches of one decode step for fixed shapes.

    summaries/scales: the group-major pool; sum_base int64 [B]; block_table int32 [B][P];
    k_cache/v_cache bf16 [pages][4][64][192]; ld: score row length (>= max own region).
    Per-step inputs (index_q, gate, q, q_pos, compress lists) are copied into the
    step's own tensors by `load`, so graph replays see new values."""

    def __init__(self, summaries, scales, sum_base, block_table, k_cache, v_cache, ld, k=512,
                 max_compress=0, index_k=None, flags=0):
        dev = summaries.device
        self.B = int(block_table.shape[0])
        self.k = int(k)
        self.ld = int(ld)
        self.flags = flags
        self.summaries, self.scales, self.sum_base = summaries, scales, sum_base
        self.block_table, self.k_cache, self.v_cache = block_table, k_cache, v_cache
        self.index_k = index_k
        B = self.B
        self.index_q = torch.zeros((B, dsa.HI, dsa.DI), dtype=torch.bfloat16, device=dev)
        self.gate = torch.zeros((B, dsa.HI), dtype=torch.float32, device=dev)
        self.q = torch.zeros((B, HQ, D), dtype=torch.bfloat16, device=dev)
        self.q_pos = torch.zeros(B, dtype=torch.int32, device=dev)
        self.q_req = torch.arange(B, dtype=torch.int32, device=dev)
        self.scores = torch.zeros((B, G, self.ld), dtype=torch.float32, device=dev)
        self.sel_idx = torch.empty((B, G, self.k), dtype=torch.int32, device=dev)
        self.sel_count = torch.empty((B, G), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, HQ, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, HQ), dtype=torch.float32, device=dev)
        self.n_compress = 0
        self.src_row = torch.zeros(max(1, max_compress), dtype=torch.int64, device=dev)
        self.dst_slot = torch.zeros(max(1, max_compress), dtype=torch.int64, device=dev)
        # workspaces (allocated once)
        L = dsa.lib()
        self.ws_idx_n = L.dsa_indexer_workspace_size(B, self.ld)
        self.ws_topk_n = L.dsa_topk_workspace_size(B, self.ld, self.k)
        self.ws_attn_n = L.dsa_attn_workspace_size(B, self.k)
        self.ws_idx = torch.empty(max(1, self.ws_idx_n), dtype=torch.uint8, device=dev)
        self.ws_topk = torch.empty(max(1, self.ws_topk_n), dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(max(1, self.ws_attn_n), dtype=torch.uint8, device=dev)

    def load(self, index_q, gate, q, q_pos, src_row=None, dst_slot=None):
        self.index_q.copy_(index_q, non_blocking=True)
        self.gate.copy_(gate, non_blocking=True)
        self.q.copy_(q, non_blocking=True)
        self.q_pos.copy_(q_pos, non_blocking=True)
        n = 0 if src_row is None else int(src_row.numel())
        if n:
            self.src_row[:n].copy_(src_row, non_blocking=True)
            self.dst_slot[:n].copy_(dst_slot, non_blocking=True)
        self.n_compress = n

    def run(self, pre_scan=None, post_scan=None):
        """Launches the step on the current stream (capturable).  pre_scan/post_scan are
        optional callables invoked right before/after the indexer-scan launch (the
        benchmark records timing events there)."""
        L = dsa.lib()
        st = dsa._stream()
        p = dsa._p
        if self.n_compress:
            ik = self.index_k
            dsa._check(L.dsa_compress_regions(p(ik), ik[0].numel(), ik.shape[0], p(self.src_row), p(self.dst_slot),
                                              self.n_compress, p(self.summaries), p(self.scales),
                                              self.summaries.shape[1], st))
        if pre_scan is not None:
            pre_scan()
        dsa._check(L.dsa_indexer_scores(p(self.index_q), p(self.gate), p(self.q_req), p(self.q_pos), self.B,
                                        p(self.summaries), p(self.scales), self.summaries.shape[1],
                                        p(self.sum_base), self.sum_base.numel(), p(self.scores), self.ld,
                                        self.flags, p(self.ws_idx), self.ws_idx_n, st))
        if post_scan is not None:
            post_scan()
        dsa._check(L.dsa_topk_regions(p(self.scores), self.ld, p(self.q_pos), self.B, self.k, p(self.sel_idx),
                                      p(self.sel_count), p(self.ws_topk), self.ws_topk_n, st))
        dsa._check(L.dsa_sparse_attn_decode(p(self.q), p(self.k_cache), p(self.v_cache), self.k_cache.shape[0],
                                            p(self.block_table), self.block_table.shape[1], p(self.q_pos), self.B,
                                            p(self.sel_idx), p(self.sel_count), self.k, p(self.out), p(self.lse),
                                            p(self.ws_attn), self.ws_attn_n, st))
        return self.out


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
