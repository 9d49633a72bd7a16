"""Chunked prefill against the oracle.

A chunk of n_new query tokens is appended to a context of ctx tokens (one request):
  1. the regions the chunk completes are compressed before any scoring (the chunk's own
     queries see them: [P2] Step-5-Preview 如何实现1M长上下文 §区域压缩CSA);
  2. every query is scored against all complete regions before its own, with the query
     quantised per head to e4m3 (DSA_Q_FP8: the FP8 x FP8 indexer contraction);
  3. top-k with the own region forced;
  4. sparse GQA prefill attention.
Full size: 2,048 queries on a 262,144-token context (33,024 regions, 8,192 selection rows).
The oracle checks every compressed region, and for sampled queries the scores, the GPU
selector fed the oracle's scores, the selection made from the GPU's scores (differences
only within 1e-3 of the threshold score) and the attention outputs; every selection row
is checked for the structural invariants.  A small chunk is checked query by query.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa, pipeline
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits, bf16_from_bits_np, selection_differs_only_near_threshold

pytestmark = pytest.mark.gpu
G = 4


def run_chunk(ctx, n_new, seed, k=512, flags=dsa.Q_FP8):
    dev = torch.device("cuda")
    d = W.prefill_chunk(ctx, n_new, seed=seed, device=dev, permute=True)
    n_slots = d["n_slots"]
    S = torch.zeros((G, n_slots, 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, n_slots), dtype=torch.float32, device=dev)
    pipeline.compress_all(d["index_k"], [ctx], [0], d["sum_base"], S, C)          # the cached context
    total = ctx + n_new
    first, last = ctx // 8, total // 8                                          # regions the chunk completes
    src = torch.arange(first, last, dtype=torch.int64, device=dev) * 8
    dsa.compress_regions(d["index_k"], src, torch.arange(first, last, dtype=torch.int64, device=dev), S, C)
    ld = total // 8
    scores = torch.zeros((n_new, G, ld), dtype=torch.float32, device=dev)
    dsa.indexer_scores(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], scores, flags)
    sel, cnt = dsa.topk_regions(scores, d["q_pos"], k)
    lse = torch.empty((n_new, 64), dtype=torch.float32, device=dev)
    out = dsa.sparse_attn_prefill(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["q_req"], d["q_pos"],
                                  sel, cnt, lse=lse)
    dsa.check_device()
    return d, S, C, scores, sel, cnt, out, lse


def check_rows(sel, cnt, q_pos, k):
    own = q_pos // 8
    want = np.minimum(k, own + 1)
    assert np.array_equal(cnt, np.repeat(want[:, None], G, axis=1))
    for i in range(sel.shape[0]):
        for g in range(G):
            c = cnt[i, g]
            row = sel[i, g, :c]
            assert row[-1] == own[i]                        # own region last (largest index)
            assert np.all(np.diff(row) > 0)                 # ascending, distinct
            assert row[0] >= 0
            assert np.all(sel[i, g, c:] == -1)


def check_sampled(d, So, Co, scores, sel, cnt, out, lse, qi, k, flags):
    """So/Co: the oracle's own summaries (never the GPU's)."""
    dev = torch.device("cuda")
    qp_all = d["q_pos"].cpu().numpy()
    qp = qp_all[qi]
    ld = scores.shape[2]
    so = oracle.indexer_scores(bits(d["index_q"][qi]), d["gate"][qi].cpu().numpy(), [0] * len(qi), qp, So, Co,
                               [0], ld=ld, flags=flags)
    sg = scores[qi].cpu().numpy()
    for j, p in enumerate(qp):
        own = int(p) // 8
        err = np.abs(sg[j, :, :own] - so[j, :, :own]).max() / np.abs(so[j, :, :own]).max()
        assert err <= 1e-4, err
    so0 = np.nan_to_num(so)
    io, co = oracle.topk_regions(so0, qp, k)
    ig, cg = dsa.topk_regions(torch.from_numpy(so0).to(dev), torch.from_numpy(qp).to(dev), k)
    assert np.array_equal(cg.cpu().numpy(), co) and np.array_equal(ig.cpu().numpy(), io)
    s_sel, s_cnt = sel[qi].cpu().numpy(), cnt[qi].cpu().numpy()
    selection_differs_only_near_threshold(s_sel, s_cnt, io, co, so0, qp, k)
    oo, lo = oracle.sparse_attention(bits(d["q"][qi]), bits(d["k_cache"]), bits(d["v_cache"]),
                                     d["block_table"].cpu().numpy(), [0] * len(qi), qp, s_sel, s_cnt)
    og = out[qi].float().cpu().numpy()
    of = bf16_from_bits_np(oo)
    assert np.all(np.abs(og - of) <= 2e-2 + 1e-2 * np.abs(of))
    np.testing.assert_allclose(lse[qi].cpu().numpy(), lo, rtol=1e-3, atol=1e-3)


def check_compression(d, S, C):
    n = d["n_slots"]
    total = d["ctx_len"] + d["n_new"]
    src, dst = W.complete_regions([total], [0], [0])
    So, Co = oracle.compress_regions(bits(d["index_k"]), src, dst, n)
    assert np.array_equal(C.cpu().numpy(), Co) and np.array_equal(S.cpu().numpy(), So)
    return So, Co


def test_small_chunk_every_query():
    # 4,096-token context + 517 new tokens (the chunk ends inside a region); every query checked
    k = 64
    d, S, C, scores, sel, cnt, out, lse = run_chunk(4096, 517, seed=41, k=k)
    So, Co = check_compression(d, S, C)
    check_rows(sel.cpu().numpy(), cnt.cpu().numpy(), d["q_pos"].cpu().numpy(), k)
    check_sampled(d, So, Co, scores, sel, cnt, out, lse, np.arange(517), k, dsa.Q_FP8)


def test_full_chunk_2048_queries_on_262144_tokens():
    k = 512
    d, S, C, scores, sel, cnt, out, lse = run_chunk(262144, 2048, seed=1238, k=k)
    So, Co = check_compression(d, S, C)
    check_rows(sel.cpu().numpy(), cnt.cpu().numpy(), d["q_pos"].cpu().numpy(), k)
    qi = np.array([0, 1, 7, 8, 511, 1024, 1535, 2040, 2047])
    check_sampled(d, So, Co, scores, sel, cnt, out, lse, qi, k, dsa.Q_FP8)


def test_locality_variant_shares_selections():
    # the 8 queries of a region share index_q: their selections coincide (up to the own region's
    # causal eligibility), so the shared-selection attention streams one union per block
    k = 512
    dev = torch.device("cuda")
    d = W.prefill_chunk(65536, 256, seed=1240, device=dev, permute=True, region_shared_q=True)
    n_slots = d["n_slots"]
    S = torch.zeros((G, n_slots, 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, n_slots), dtype=torch.float32, device=dev)
    total = 65536 + 256
    src, dst = W.complete_regions([total], [0], [0])
    dsa.compress_regions(d["index_k"], torch.tensor(src, dtype=torch.int64, device=dev),
                         torch.tensor(dst, dtype=torch.int64, device=dev), S, C)
    ld = total // 8
    scores = torch.zeros((256, G, ld), dtype=torch.float32, device=dev)
    dsa.indexer_scores(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], scores, dsa.Q_FP8)
    sel, cnt = dsa.topk_regions(scores, d["q_pos"], k)
    lse = torch.empty((256, 64), dtype=torch.float32, device=dev)
    out = dsa.sparse_attn_prefill(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["q_req"], d["q_pos"],
                                  sel, cnt, lse=lse)
    dsa.check_device()
    s_np = sel.cpu().numpy()
    assert np.array_equal(s_np[8], s_np[9])                    # same region, same selection
    So, Co = check_compression(d, S, C)
    qi = np.array([0, 8, 9, 15, 100, 255])
    check_sampled(d, So, Co, scores, sel, cnt, out, lse, qi, k, dsa.Q_FP8)
