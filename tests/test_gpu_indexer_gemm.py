"""The prefill indexer GEMM (tcgen05 FP8 x FP8, one request's chunk) against the oracle and
against the streaming scan.

A prefill chunk is scored with the query quantised per (query, head) to e4m3 (DSA_Q_FP8,
[P1] kwkr.cn/news/601179 §DSA ③: the indexer is an FP8 contraction).  Cases span several
128-row query tiles and 256-region blocks with ragged tails, a pool offset (sum_base > 0),
a score row length that is not a multiple of 4 (scalar stores), a request's first chunk
(queries whose own region is 0 write nothing) and an invalid query (flagged, skipped).
Tolerance as for the scan: 1e-4 of the row's largest |score|.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits

pytestmark = pytest.mark.gpu
G = 4
SENTINEL = -12345.0


def chunk_pool(ctx, n_new, seed, base):
    """Chunk inputs with every complete region of the ctx+n_new tokens compressed into
    pool slots base .. base+n-1 of a pool with some slack after them."""
    dev = torch.device("cuda")
    d = W.prefill_chunk(ctx, n_new, seed=seed, device=dev, permute=False)
    total = ctx + n_new
    n = total // 8
    n_slots = base + n + 5
    S = torch.zeros((G, n_slots, 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, n_slots), dtype=torch.float32, device=dev)
    src = torch.arange(n, dtype=torch.int64, device=dev) * 8
    dsa.compress_regions(d["index_k"], src, src // 8 + base, S, C)
    d["sum_base"] = torch.tensor([base], dtype=torch.int64, device=dev)
    return d, S, C


def scores_via(d, S, C, ld, use_gemm, q_pos=None):
    """Raw C-ABI call: use_gemm=False passes no workspace, which takes the streaming scan."""
    qp = d["q_pos"] if q_pos is None else q_pos
    nq = qp.numel()
    sc = torch.full((nq, G, ld), SENTINEL, dtype=torch.float32, device="cuda")
    L = dsa.lib()
    nbytes = L.dsa_indexer_workspace_size(nq, ld) if use_gemm else 0
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    p = dsa._p
    dsa._check(L.dsa_indexer_scores(p(d["index_q"]), p(d["gate"]), p(d["q_req"]), p(qp), nq, p(S), p(C),
                                    S.shape[1], p(d["sum_base"]), 1, p(sc), ld, dsa.Q_FP8,
                                    p(ws) if use_gemm else None, nbytes, dsa._stream()))
    return sc


def oracle_scores(d, S_host, C_host, ld, qi):
    qp = d["q_pos"].cpu().numpy()[qi]
    base = int(d["sum_base"][0])
    return oracle.indexer_scores(bits(d["index_q"][qi]), d["gate"][qi].cpu().numpy(), [0] * len(qi), qp,
                                 S_host, C_host, [base], ld=ld, flags=dsa.Q_FP8), qp


def compare(sg, so, q_pos, tol=1e-4):
    for i, p in enumerate(q_pos):
        own = int(p) // 8
        for g in range(G):
            if own:
                a, b = sg[i, g, :own], so[i, g, :own]
                err = np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)
                assert err <= tol, (i, g, err)
            assert np.all(sg[i, g, own:] == SENTINEL), (i, g)


def oracle_pool(d, ctx, n_new, base, n_slots):
    n = (ctx + n_new) // 8
    return oracle.compress_regions(bits(d["index_k"]), [8 * r for r in range(n)], [base + r for r in range(n)],
                                   n_slots)


@pytest.mark.parametrize("ctx,n_new,base,pad", [(3003, 333, 37, 3), (1024, 640, 0, 0), (0, 200, 11, 1)])
def test_gemm_every_query_matches_oracle(ctx, n_new, base, pad):
    d, S, C = chunk_pool(ctx, n_new, seed=ctx + n_new, base=base)
    ld = (ctx + n_new) // 8 + pad
    sg = scores_via(d, S, C, ld, use_gemm=True)
    dsa.check_device()
    So, Co = oracle_pool(d, ctx, n_new, base, S.shape[1])
    assert np.array_equal(So, S.cpu().numpy()) and np.array_equal(Co, C.cpu().numpy())
    qi = np.arange(n_new)
    so, qp = oracle_scores(d, So, Co, ld, qi)
    compare(sg.cpu().numpy(), so, qp)


def test_gemm_agrees_with_scan():
    ctx, n_new = 20000, 1000
    d, S, C = chunk_pool(ctx, n_new, seed=5, base=3)
    ld = (ctx + n_new) // 8
    a = scores_via(d, S, C, ld, use_gemm=True).cpu().numpy()
    b = scores_via(d, S, C, ld, use_gemm=False).cpu().numpy()
    dsa.check_device()
    qp = d["q_pos"].cpu().numpy()
    for i in range(0, n_new, 37):
        own = int(qp[i]) // 8
        for g in range(G):
            err = np.abs(a[i, g, :own] - b[i, g, :own]).max() / np.abs(b[i, g, :own]).max()
            assert err <= 2e-5, (i, g, err)
    assert np.array_equal(a == SENTINEL, b == SENTINEL)


def test_gemm_invalid_query_is_flagged_and_skipped():
    ctx, n_new = 2048, 128
    d, S, C = chunk_pool(ctx, n_new, seed=9, base=0)
    ld = (ctx + n_new) // 8
    qp = d["q_pos"].clone()
    qp[5] = 8 * (ld + 1)                 # own region beyond the score row
    sg = scores_via(d, S, C, ld, use_gemm=True, q_pos=qp)
    with pytest.raises(dsa.DsaError):
        dsa.check_device()
    sg = sg.cpu().numpy()
    assert np.all(sg[5] == SENTINEL)
    So, Co = oracle_pool(d, ctx, n_new, 0, S.shape[1])
    qi = np.array([0, 4, 6, 127])
    so, qpo = oracle_scores(d, So, Co, ld, qi)
    compare(sg[qi], so, qpo)
