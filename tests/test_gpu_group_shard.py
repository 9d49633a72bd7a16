"""KV-group-sharded decode on one GPU: the `_groups` calls run on one shard's data (the
summaries and K/V of groups g0 .. g0 + ng - 1 only) and must give exactly the rows of the
4-group calls for those groups ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: regions and
indexer heads map one to one onto the 4 KV groups, so every step is per group).

Per case and shard plan ({0,1} + {2,3}, and the four single groups):
  * the shard's compression equals its groups' rows of the 4-group pool, byte for byte;
  * its scores, selection, attention output and LSE equal the 4-group call's rows for its
    groups bit for bit, and the shards' union is the 4-group call;
  * (smaller cases) each shard against the oracle: scores within 1e-4 of the row's largest
    oracle score, and attention on the shard's selection within 2e-2 abs + 1e-2 rel.
Cases: B = 2 (131,072 and 20,000 tokens: the clustered attention), B = 8 at 16,384 (the
per-row attention with splits) and B = 1 at 1,048,576 (the chunk-maxima selection)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa, pipeline
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits, bf16_from_bits_np

pytestmark = pytest.mark.gpu
G, K = 4, 512
CASES = {
    "b2_ragged": dict(lengths=[131072, 20000], seed=1401, oracle=True),
    "b8_16k": dict(lengths=[16384] * 8, seed=1402, oracle=True),
    "b1_1m": dict(lengths=[1 << 20], seed=1403, oracle=False),
}
PLANS = [[(0, 2), (2, 2)], [(0, 1), (1, 1), (2, 1), (3, 1)], [(0, 4)]]


def full_step(d, ld):
    dev = d["index_k"].device
    S = torch.zeros((G, d["n_slots"], 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, d["n_slots"]), dtype=torch.float32, device=dev)
    pipeline.compress_all(d["index_k"], d["lengths"], d["tok_base"], d["sum_base"], S, C)
    nq = d["q_pos"].numel()
    scores = torch.zeros((nq, G, ld), dtype=torch.float32, device=dev)
    sel, cnt = dsa.decode_select(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], scores, K)
    lse = torch.empty((nq, 64), dtype=torch.float32, device=dev)
    out = dsa.sparse_attn_decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["q_pos"], sel, cnt, lse=lse)
    dsa.check_device()
    return S, C, scores, sel, cnt, out, lse


def shard_step(d, ld, g0, ng):
    dev = d["index_k"].device
    src, dst = W.complete_regions(d["lengths"], d["tok_base"], d["sum_base"])
    src, dst = torch.as_tensor(src, dtype=torch.int64, device=dev), torch.as_tensor(dst, dtype=torch.int64, device=dev)
    S = torch.zeros((ng, d["n_slots"], 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((ng, d["n_slots"]), dtype=torch.float32, device=dev)
    dsa.compress_regions_groups(d["index_k"], src, dst, S, C, g0)
    nq = d["q_pos"].numel()
    scores = torch.zeros((nq, ng, ld), dtype=torch.float32, device=dev)
    sel, cnt = dsa.decode_select_groups(d["index_q"], d["gate"], d["q_req"], d["q_pos"], S, C, d["sum_base"], scores,
                                        K, g0)
    kc = d["k_cache"][:, g0:g0 + ng].contiguous()
    vc = d["v_cache"][:, g0:g0 + ng].contiguous()
    lse = torch.empty((nq, 16 * ng), dtype=torch.float32, device=dev)
    out = dsa.sparse_attn_decode_groups(d["q"], kc, vc, d["block_table"], d["q_pos"], sel, cnt, g0, lse=lse)
    dsa.check_device()
    return S, C, scores, sel, cnt, out, lse


@pytest.mark.parametrize("case", list(CASES))
def test_group_shards_equal_the_four_group_calls(case):
    cfg = CASES[case]
    dev = torch.device("cuda")
    d = W.decode_batch(cfg["lengths"], seed=cfg["seed"], device=dev, permute=True)
    ld = max(d["lengths"]) // 8
    S, C, scores, sel, cnt, out, lse = full_step(d, ld)
    qp = d["q_pos"].cpu().numpy()
    own = [int(p) // 8 for p in qp]
    if cfg["oracle"]:
        src, dst = W.complete_regions(d["lengths"], d["tok_base"], d["sum_base"])
        So, Co = oracle.compress_regions(bits(d["index_k"]), src, dst, d["n_slots"])
        so = oracle.indexer_scores(bits(d["index_q"]), d["gate"].cpu().numpy(), d["q_req"].cpu().numpy(), qp, So, Co,
                                   d["sum_base"].cpu().numpy(), ld=ld)
    for plan in PLANS:
        parts = []
        for g0, ng in plan:
            Ss, Cs, ss, sl, cn, o, ls = shard_step(d, ld, g0, ng)
            gs = slice(g0, g0 + ng)
            hs = slice(16 * g0, 16 * (g0 + ng))
            assert torch.equal(Ss, S[gs]) and torch.equal(Cs, C[gs])
            for i, ow in enumerate(own):
                assert torch.equal(ss[i, :, :ow], scores[i, gs, :ow])
            assert torch.equal(cn, cnt[:, gs]) and torch.equal(sl, sel[:, gs])
            assert torch.equal(o, out[:, hs]) and torch.equal(ls, lse[:, hs])
            if cfg["oracle"]:
                sgn = ss.cpu().numpy()
                for i, ow in enumerate(own):
                    ref = so[i, gs, :ow]
                    assert np.abs(sgn[i, :, :ow] - ref).max() <= 1e-4 * np.abs(ref).max()
                # attention on the shard's selection against the oracle (other groups empty)
                sel_f = np.full((len(qp), G, K), -1, np.int32)
                cnt_f = np.zeros((len(qp), G), np.int32)
                sel_f[:, gs] = sl.cpu().numpy()
                cnt_f[:, gs] = cn.cpu().numpy()
                oo, lo = oracle.sparse_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                                 d["block_table"].cpu().numpy(), d["q_req"].cpu().numpy(), qp, sel_f,
                                                 cnt_f)
                of = bf16_from_bits_np(oo)[:, hs]
                og = o.float().cpu().numpy()
                assert np.all(np.abs(og - of) <= 2e-2 + 1e-2 * np.abs(of))
                np.testing.assert_allclose(ls.cpu().numpy(), lo[:, hs], rtol=1e-3, atol=1e-3)
            parts.append((sl, cn, o))
        # the union of the shards is the 4-group call
        assert torch.equal(torch.cat([p[0] for p in parts], dim=1), sel)
        assert torch.equal(torch.cat([p[1] for p in parts], dim=1), cnt)
        assert torch.equal(torch.cat([p[2] for p in parts], dim=1), out)

