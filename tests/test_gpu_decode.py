"""End-to-end decode steps at the workloads' full sizes, every stage against the oracle.

  * compression: bytes and scales bit-exact over the whole cache;
  * indexer scores: within 1e-4 of the row's largest oracle score;
  * top-k: the GPU selector fed the oracle's scores reproduces the oracle bit for bit,
    and the selection made from the GPU's own scores differs from the oracle's only for
    regions whose score is within 1e-3 (relative) of the threshold score;
  * attention on the GPU's selection: within 2e-2 abs + 1e-2 rel of the oracle on the
    same selection.
Workloads: decode B=1 at 16,384 tokens (identity block table), B=8 at 131,072 tokens
and B=1 at 1,048,576 tokens (random page permutations); k = 512, query at L-1.
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
CASES = {
    "b1_16k": dict(lengths=[16384], permute=False, seed=1235),
    "b8_128k": dict(lengths=[131072] * 8, permute=True, seed=1236),
    "b1_1m": dict(lengths=[1 << 20], permute=True, seed=1237),
}


@pytest.mark.parametrize("case", list(CASES))
def test_decode_step_against_oracle(case):
    cfg = CASES[case]
    dev = torch.device("cuda")
    k = 512
    d = W.decode_batch(cfg["lengths"], seed=cfg["seed"], device=dev, permute=cfg["permute"])
    n_slots = d["n_slots"]
    S = torch.zeros((G, n_slots, 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, n_slots), dtype=torch.float32, device=dev)
    # cache set-up: every complete region except the one the step itself completes
    lengths_before = [L - 1 for L in d["lengths"]]
    pipeline.compress_all(d["index_k"], lengths_before, d["tok_base"], d["sum_base"], S, C)
    ld = max(d["lengths"]) // 8
    step = pipeline.DecodeStep(S, C, d["sum_base"], d["block_table"], d["k_cache"], d["v_cache"], ld, k=k,
                               tail_tokens=8)
    # tail block b = the last 8 tokens of request b; compressed when the query completes it
    tail = torch.cat([d["index_k"][int(d["tok_base"][b]) + L - 8: int(d["tok_base"][b]) + L]
                      for b, L in enumerate(d["lengths"])])
    step.load(d["index_q"], d["gate"], d["q"], d["q_pos"], tail)
    due = [b for b, L in enumerate(d["lengths"]) if L % 8 == 0]
    step.set_compress(due, [int(d["sum_base"][b]) + (d["lengths"][b] - 1) // 8 for b in due])
    step.run()
    dsa.check_device()

    # --- compression over the whole cache
    src, dst = W.complete_regions(d["lengths"], d["tok_base"], d["sum_base"])
    So, Co = oracle.compress_regions(bits(d["index_k"]), src, dst, n_slots)
    assert np.array_equal(C.cpu().numpy(), Co)
    assert np.array_equal(S.cpu().numpy(), So)

    # --- scores
    qp = d["q_pos"].cpu().numpy()
    so = oracle.indexer_scores(bits(d["index_q"]), d["gate"].cpu().numpy(), d["q_req"].cpu().numpy(), qp, So, Co,
                               d["sum_base"].cpu().numpy(), ld=ld)
    sg = step.scores.cpu().numpy()
    for i, p in enumerate(qp):
        own = int(p) // 8
        err = np.abs(sg[i, :, :own] - so[i, :, :own]).max() / np.abs(so[i, :, :own]).max()
        assert err <= 1e-4, err

    # --- top-k: bit-exact on the oracle's scores, near-threshold-only differences on ours
    io, co = oracle.topk_regions(np.nan_to_num(so), qp, k)
    ig, cg = dsa.topk_regions(torch.from_numpy(np.nan_to_num(so)).to(dev), d["q_pos"], k)
    assert np.array_equal(cg.cpu().numpy(), co) and np.array_equal(ig.cpu().numpy(), io)
    sel, cnt = step.sel_idx.cpu().numpy(), step.sel_count.cpu().numpy()
    n_diff = selection_differs_only_near_threshold(sel, cnt, io, co, np.nan_to_num(so), qp, k)
    print(f"{case}: rows whose selection differs near the threshold: {n_diff}/{sel.shape[0] * G}")

    # --- attention on the GPU's own selection
    oo, lo = oracle.sparse_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                     d["block_table"].cpu().numpy(), d["q_req"].cpu().numpy(), qp, sel, cnt)
    og = step.out.float().cpu().numpy()
    of = bf16_from_bits_np(oo)
    assert np.all(np.abs(og - of) <= 2e-2 + 1e-2 * np.abs(of))
    np.testing.assert_allclose(step.lse.cpu().numpy(), lo, rtol=1e-3, atol=1e-3)
