"""GPU top-k (A3) fed the oracle's fp32 scores must reproduce the oracle's selection
bit for bit (indices, order, counts, padding)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa

pytestmark = pytest.mark.gpu
G = 4


def both(scores, q_pos, k):
    s = torch.from_numpy(np.ascontiguousarray(scores)).cuda()
    qp = torch.tensor(q_pos, dtype=torch.int32, device="cuda")
    ig, cg = dsa.topk_regions(s, qp, k)
    dsa.check_device()
    io, co = oracle.topk_regions(scores, q_pos, k)
    return ig.cpu().numpy(), cg.cpu().numpy(), io, co


def check(scores, q_pos, k):
    ig, cg, io, co = both(scores, q_pos, k)
    assert np.array_equal(cg, co)
    assert np.array_equal(ig, io)


@pytest.mark.parametrize("k", [1, 2, 64, 512, 2048])
def test_random_rows(k):
    rng = np.random.default_rng(k)
    ld = 20000
    s = rng.standard_normal((4, G, ld)).astype(np.float32)
    check(s, [8 * ld - 1, 8 * 3000 + 4, 7, 8 * 511], k)


def test_scores_like_the_indexer():
    # non-negative, ReLU zeros, gated sums: the distribution the decode path produces
    rng = np.random.default_rng(1)
    ld = 16383
    d = rng.standard_normal((2, G, 4, ld)) * 5.6
    z = rng.uniform(0, 1, (2, G, 4, 1))
    s = (np.maximum(d, 0) * z).sum(axis=2).astype(np.float32) / 16
    check(s, [8 * ld + 7, 8 * ld], 512)


def test_heavy_ties_and_all_zero_rows():
    rng = np.random.default_rng(2)
    s = rng.integers(0, 5, (2, G, 9000)).astype(np.float32)
    s[1] = 0.0
    s[1, 2, 100:200] = -0.0
    check(s, [8 * 9000, 8 * 9000 + 3], 512)


def test_negative_and_mixed_sign_scores():
    rng = np.random.default_rng(3)
    s = (rng.standard_normal((1, G, 5000)) * 1e3).astype(np.float32)
    s[0, 1] = -np.abs(s[0, 1])
    check(s, [8 * 5000], 300)


def test_own_region_smaller_than_k():
    rng = np.random.default_rng(4)
    s = rng.standard_normal((3, G, 600)).astype(np.float32)
    check(s, [0, 8 * 100 + 1, 8 * 511 + 7], 512)


def test_one_million_token_row():
    rng = np.random.default_rng(5)
    ld = 131071
    d = rng.standard_normal((1, G, 4, ld)).astype(np.float32) * 5.6
    s = (np.maximum(d, 0) * rng.uniform(0, 1, (1, G, 4, 1)).astype(np.float32)).sum(axis=2) / 16
    check(s.astype(np.float32), [8 * 131072 - 1], 512)


def test_many_rows_take_the_per_row_path():
    # more (query, group) rows than the cluster path takes, rows of at most 65,536 scores:
    # one CTA per row (group-maxima bound, candidates in smem)
    rng = np.random.default_rng(6)
    nq, ld = 100, 3000
    s = rng.standard_normal((nq, G, ld)).astype(np.float32)
    s[::7] = np.round(s[::7])                     # some tie-heavy rows
    q_pos = [int(x) for x in rng.integers(0, 8 * ld + 1, nq)]
    check(s, q_pos, 512)


def test_per_row_path_unaligned_rows():
    # rows that do not start on 16-byte boundaries (ld not a multiple of 4) are loaded
    # directly instead of streamed through the smem ring; same selection either way
    rng = np.random.default_rng(11)
    nq, ld = 100, 3001
    s = rng.standard_normal((nq, G, ld)).astype(np.float32)
    s[::5] = np.round(s[::5] * 2) / 2             # tie-heavy rows
    q_pos = [int(x) for x in rng.integers(0, 8 * ld + 1, nq)]
    check(s, q_pos, 512)


@pytest.mark.parametrize("k", [2, 64, 512, 1024])
def test_per_row_path_prefill_like_rows(k):
    # prefill-shaped: 160 rows of 33,024 scores, indexer-like non-negative scores, rows with
    # all scores equal (the whole-row fallback), rows ending in every region of a chunk
    rng = np.random.default_rng(k)
    nq, ld = 40, 33024
    z = rng.standard_normal((nq, G, 4, ld)).astype(np.float32)
    s = (np.maximum(z, 0) * rng.uniform(0, 1, (nq, G, 4, 1)).astype(np.float32)).sum(2) / 16
    s = s.astype(np.float32)
    s[3] = 0.0
    s[4] = 0.5
    q_pos = [8 * ld - 1 - 3 * i for i in range(nq)]
    check(s, q_pos, k)


def test_many_long_rows_take_the_workspace_path():
    # many rows longer than 65,536 scores: histogram + select kernels with a workspace
    rng = np.random.default_rng(16)
    nq, ld = 20, 70000
    s = rng.standard_normal((nq, G, ld)).astype(np.float32)
    s[::5] = np.round(s[::5])
    q_pos = [int(x) for x in rng.integers(0, 8 * ld + 1, nq)]
    check(s, q_pos, 512)


def test_cluster_path_long_rows_and_ties():
    # rows long enough for 8-CTA clusters, with a plateau of equal scores at the threshold
    rng = np.random.default_rng(7)
    ld = 120000
    s = rng.standard_normal((2, G, ld)).astype(np.float32)
    s[0, 0, :5000] = 2.5
    s[1, 3, :] = 0.0
    check(s, [8 * ld, 8 * 70000 + 3], 512)


def test_own_beyond_ld_is_flagged():
    s = np.zeros((1, G, 10), np.float32)
    sc = torch.from_numpy(s).cuda()
    idx, cnt = dsa.topk_regions(sc, torch.tensor([8 * 50], dtype=torch.int32, device="cuda"), 4)
    with pytest.raises(dsa.DsaError):
        dsa.check_device()
    assert np.all(cnt.cpu().numpy() == 0) and np.all(idx.cpu().numpy() == -1)


@pytest.mark.parametrize("ld", [16000, 16384, 60000, 131071])
def test_equal_scores_take_the_lowest_regions(ld):
    # every score of a row equal (one row +0, one row a positive constant, one row two values
    # in alternating blocks): the exact threshold must narrow through several histogram
    # levels of the (score, region) composite, on the single-CTA rows (ld <= 16,384) and on
    # the cluster rows
    k = 512
    s = np.zeros((3, G, ld), np.float32)
    s[1] = 0.75
    s[2] = np.where((np.arange(ld) // 97) % 2 == 0, 1.5, 1.25).astype(np.float32)
    check(s, [8 * ld - 1, 8 * ld - 3, 8 * (ld - 5)], k)


@pytest.mark.parametrize("n_tied", [5, 31, 33, 40])
def test_cluster_path_ties_at_the_threshold(n_tied):
    # n_tied regions take exactly the score of the need-th best one, so the bin of the
    # candidate histogram that holds the threshold holds n_tied + 1 equal keys: taken whole,
    # ranked by one warp (<= 32) or narrowed by the general levels (> 32); the lowest regions
    # of the tie win
    rng = np.random.default_rng(100 + n_tied)
    ld, k = 120000, 512
    s = rng.standard_normal((2, G, ld)).astype(np.float32)
    q_pos = [8 * ld, 8 * ld - 5]                              # own regions ld and ld - 1
    for b in range(2):
        own = q_pos[b] // 8
        for g in range(G):
            v = np.sort(s[b, g, :own])[::-1][k - 2]           # the (k-1)-th largest: need = k - 1
            x = 1000 + 7919 * (b * G + g)
            s[b, g, x:x + n_tied] = v
    check(s, q_pos, k)
