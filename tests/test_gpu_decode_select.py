"""dsa_decode_select (scan + selection in one call, the selection bounded by the scan's chunk
maxima) against the two separate calls and the oracle's selection.

The fused call must return exactly what dsa_indexer_scores followed by dsa_topk_regions
return: the same scores bit for bit and the same selection, which is the oracle's selection
over those scores ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: own region forced, ties
to the lower region).  Cases: decode batches whose rows take the chunk-maxima path (few long
rows: 16,384 .. 131,071 regions) and rows that do not (short rows, k = 1024, many rows), all-
zero queries (every score +0: the maxima tie in bulk and the selection falls back), identical
summaries (every score of a row equal), rows whose own region is below k, rows whose best
regions crowd into one stretch of the row (many chunk maxima tie near the bound, and whole
chunks are candidates), and rows where a run of regions shares the threshold score exactly
(copies of the summary at the threshold: the candidate bin at the threshold is taken whole,
ranked by one warp, or narrowed by the general levels).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa, pipeline
from sparse_long_context_dsa_b200 import workloads as W

pytestmark = pytest.mark.gpu
G = 4


def setup(lengths, seed, zero_q=False, same_summary=False):
    dev = torch.device("cuda")
    d = W.decode_batch(lengths, seed=seed, device=dev, permute=True)
    S = torch.zeros((G, d["n_slots"], 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, d["n_slots"]), dtype=torch.float32, device=dev)
    pipeline.compress_all(d["index_k"], d["lengths"], d["tok_base"], d["sum_base"], S, C)
    if same_summary:
        S[:] = S[:, :1].clone()
        C[:] = C[:, :1].clone()
    if zero_q:
        d["index_q"].zero_()
    return d, S, C


def both(d, S, C, k, ld):
    nq = d["q_pos"].numel()
    s1 = torch.full((nq, G, ld), -7.0, dtype=torch.float32, device="cuda")
    s2 = s1.clone()
    i1, c1 = dsa.decode_select(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], s1, k)
    dsa.indexer_scores(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], s2)
    i2, c2 = dsa.topk_regions(s2, d["q_pos"], k)
    dsa.check_device()
    return s1, i1, c1, s2, i2, c2


def check_against_oracle(s1, i1, c1, q_pos, k):
    sc = np.nan_to_num(s1.cpu().numpy())
    io, co = oracle.topk_regions(sc, q_pos.cpu().numpy(), k)
    assert np.array_equal(c1.cpu().numpy(), co) and np.array_equal(i1.cpu().numpy(), io)


@pytest.mark.parametrize("lengths,k", [
    ([1 << 20], 512),                                  # 4 cluster rows of 131,071 regions
    ([1 << 20, 131072 + 3], 512),                      # two requests, 8 cluster rows
    ([16384 * 8 + 7, 300000, 1 << 19], 64),            # mixed lengths
    ([1 << 20, 9, 200], 2),                            # a long row beside rows shorter than k
    ([1 << 20], 1024),                                 # k above the chunk-maxima path
    ([5000] * 12, 512),                                # many short rows
])
def test_matches_separate_calls_and_oracle(lengths, k):
    d, S, C = setup(lengths, seed=300 + k + len(lengths))
    ld = max(lengths) // 8
    s1, i1, c1, s2, i2, c2 = both(d, S, C, k, ld)
    assert torch.equal(s1, s2)
    assert torch.equal(c1, c2) and torch.equal(i1, i2)
    check_against_oracle(s1, i1, c1, d["q_pos"], k)


@pytest.mark.parametrize("case", ["zero_query", "same_summary"])
def test_equal_scores_take_the_lowest_regions(case):
    lengths = [1 << 20, 300000]
    d, S, C = setup(lengths, seed=41, zero_q=case == "zero_query", same_summary=case == "same_summary")
    k = 512
    ld = max(lengths) // 8
    s1, i1, c1, s2, i2, c2 = both(d, S, C, k, ld)
    assert torch.equal(s1, s2)
    assert torch.equal(c1, c2) and torch.equal(i1, i2)
    sel = i1.cpu().numpy()
    own = d["q_pos"].cpu().numpy() // 8
    for b in range(len(lengths)):
        for g in range(G):
            row = s1[b, g, : own[b]].cpu().numpy()
            if np.all(row == row[0]):                  # one tie: regions 0..k-2, then own
                assert np.array_equal(sel[b, g, : k - 1], np.arange(k - 1))
                assert sel[b, g, k - 1] == own[b]


def test_decode_step_uses_it():
    lengths = [1 << 20]
    d, S, C = setup(lengths, seed=5)
    ld = max(lengths) // 8
    st = pipeline.DecodeStep(S, C, d["sum_base"], d["block_table"], d["k_cache"], d["v_cache"], ld, k=512)
    st.load(d["index_q"], d["gate"], d["q"], d["q_pos"])
    st.run()
    s2 = torch.zeros_like(st.scores)
    dsa.indexer_scores(d["index_q"], d["gate"], st.q_req, d["q_pos"], S, C, d["sum_base"], s2)
    i2, c2 = dsa.topk_regions(s2, d["q_pos"], 512)
    dsa.check_device()
    own = int(d["q_pos"][0]) // 8
    assert torch.equal(st.scores[:, :, :own], s2[:, :, :own])
    assert torch.equal(st.sel_idx, i2) and torch.equal(st.sel_count, c2)


@pytest.mark.parametrize("lo,n", [(70000, 700), (0, 3000), (131071 - 600, 600)])
def test_crowded_best_regions_fall_back_exactly(lo, n):
    # scales of regions lo .. lo+n-1 times 64: their scores are 64x the others' (ReLU is
    # positively homogeneous), so the selection crowds into a few hundred whole chunks
    lengths = [1 << 20]
    d, S, C = setup(lengths, seed=77 + lo)
    C[:, lo:lo + n] *= 64.0
    k = 512
    ld = max(lengths) // 8
    s1, i1, c1, s2, i2, c2 = both(d, S, C, k, ld)
    assert torch.equal(s1, s2)
    assert torch.equal(c1, c2) and torch.equal(i1, i2)
    check_against_oracle(s1, i1, c1, d["q_pos"], k)
    sel = i1.cpu().numpy()[0]
    assert np.mean((sel[:, : k - 1] >= lo) & (sel[:, : k - 1] < lo + n)) > 0.9


@pytest.mark.parametrize("n_tied", [5, 31, 40])
def test_ties_at_the_threshold(n_tied):
    # each group's summary and scale at its (k-1)-th best region are copied over a run of
    # n_tied regions: their scores equal the threshold score bit for bit
    lengths = [1 << 20]
    d, S, C = setup(lengths, seed=900 + n_tied)
    k = 512
    ld = max(lengths) // 8
    own = int(d["q_pos"][0]) // 8
    s0 = torch.zeros((1, G, ld), dtype=torch.float32, device="cuda")
    dsa.indexer_scores(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], s0)
    dsa.check_device()
    base = int(d["sum_base"][0])
    for g in range(G):
        row = s0[0, g, :own].cpu().numpy()
        r = int(np.argsort(-row, kind="stable")[k - 2])
        x = 3000 + 20011 * g
        S[g, base + x:base + x + n_tied] = S[g, base + r]
        C[g, base + x:base + x + n_tied] = C[g, base + r]
    s1, i1, c1, s2, i2, c2 = both(d, S, C, k, ld)
    assert torch.equal(s1, s2)
    assert torch.equal(c1, c2) and torch.equal(i1, i2)
    check_against_oracle(s1, i1, c1, d["q_pos"], k)
    sc = s1.cpu().numpy()[0]
    for g in range(G):
        x = 3000 + 20011 * g
        assert np.all(sc[g, x:x + n_tied] == sc[g, x])       # the run is one tie
