"""GPU indexer scores (A2) against the oracle.

The oracle accumulates in double; the GPU contracts e4m3 summaries with an exact e4m3
hi/lo split of the bf16 query on the tensor cores in fp32.  Tolerance: |gpu - oracle| <=
1e-4 * max|oracle score| of the row (the dot products cancel, so per-entry relative error
is not meaningful; the top-k contract is a 1e-3 relative gap at the threshold).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa, pipeline
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits

pytestmark = pytest.mark.gpu
G = 4
SENTINEL = -12345.0


def setup(lengths, seed, dev="cuda"):
    d = W.decode_batch(lengths, seed=seed, device=dev, permute=True)
    S = torch.zeros((G, d["n_slots"], 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, d["n_slots"]), dtype=torch.float32, device=dev)
    pipeline.compress_all(d["index_k"], d["lengths"], d["tok_base"], d["sum_base"], S, C)
    return d, S, C


def gpu_scores(d, S, C, ld, flags=0, q_pos=None, q_req=None):
    qp = d["q_pos"] if q_pos is None else q_pos
    qr = d["q_req"] if q_req is None else q_req
    nq = qp.numel()
    sc = torch.full((nq, G, ld), SENTINEL, dtype=torch.float32, device="cuda")
    dsa.indexer_scores(d["index_q"][:nq].contiguous(), d["gate"][:nq].contiguous(), qr, qp, S, C,
                       d["sum_base"], sc, flags)
    dsa.check_device()
    return sc.cpu().numpy()


def compare(sg, so, q_pos, tol=1e-4):
    worst = 0.0
    for i, p in enumerate(q_pos):
        own = int(p) // 8
        for g in range(G):
            a, b = sg[i, g, :own], so[i, g, :own]
            if own:
                scale = max(np.abs(b).max(), 1e-30)
                err = np.abs(a - b).max() / scale
                worst = max(worst, err)
                assert err <= tol, (i, g, err)
            assert np.all(sg[i, g, own:] == SENTINEL)            # r >= own untouched
    return worst


@pytest.mark.parametrize("flags", [0, dsa.Q_FP8])
def test_scores_match_oracle(flags):
    lengths = [5000, 1037, 64, 9, 4096 * 2 + 3]
    d, S, C = setup(lengths, seed=21)
    ld = max(lengths) // 8 + 3
    sg = gpu_scores(d, S, C, ld, flags)
    qp = d["q_pos"].cpu().numpy()
    so = oracle.indexer_scores(bits(d["index_q"]), d["gate"].cpu().numpy(), d["q_req"].cpu().numpy(), qp,
                               S.cpu().numpy(), C.cpu().numpy(), d["sum_base"].cpu().numpy(), ld=ld, flags=flags)
    w = compare(sg, so, qp)
    print(f"max normalised score error {w:.3e} (flags={flags})")


def test_queries_mid_region_and_shared_request():
    lengths = [3000]
    d, S, C = setup(lengths, seed=22)
    pos = torch.tensor([2999, 1500, 17, 8, 7, 0, 2047], dtype=torch.int32, device="cuda")
    req = torch.zeros(7, dtype=torch.int32, device="cuda")
    d["index_q"] = W.normal_bf16((7, 16, 256), W.generator(5, "cuda"), "cuda")
    d["gate"] = W.uniform_f32((7, 16), W.generator(6, "cuda"), "cuda")
    ld = 400
    sg = gpu_scores(d, S, C, ld, q_pos=pos, q_req=req)
    so = oracle.indexer_scores(bits(d["index_q"]), d["gate"].cpu().numpy(), req.cpu().numpy(),
                               pos.cpu().numpy(), S.cpu().numpy(), C.cpu().numpy(),
                               d["sum_base"].cpu().numpy(), ld=ld)
    compare(sg, so, pos.cpu().numpy())


def test_extreme_query_magnitudes():
    d, S, C = setup([2048], seed=23)
    q = d["index_q"].float()
    q[0, 0] *= 1e-20                              # tiny head
    q[0, 1] *= 1e20                               # huge head
    q[0, 2] = 0                                   # zero head
    q[0, 3, 5] = 1e-3                             # one large component among tiny ones
    d["index_q"] = q.to(torch.bfloat16)
    sg = gpu_scores(d, S, C, 256)
    qp = d["q_pos"].cpu().numpy()
    so = oracle.indexer_scores(bits(d["index_q"]), d["gate"].cpu().numpy(), [0], qp, S.cpu().numpy(),
                               C.cpu().numpy(), [0], ld=256)
    compare(sg, so, qp)


def test_invalid_query_is_flagged():
    d, S, C = setup([512], seed=24)
    sc = torch.full((1, G, 10), SENTINEL, dtype=torch.float32, device="cuda")
    dsa.indexer_scores(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], sc)  # own 63 > ld 10
    with pytest.raises(dsa.DsaError):
        dsa.check_device()
    assert np.all(sc.cpu().numpy() == SENTINEL)
