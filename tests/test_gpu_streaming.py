"""Ragged batched decode with the streaming summary update, against the oracle.

32 requests, lengths log-uniform in [4,096, 1,048,576] with tails of 0-7 tokens (their last
region incomplete, hence unsummarised), 8 decode steps each appending one token per request
([P2] Step-5-Preview 如何实现1M长上下文 §区域压缩CSA, update_summaries_decode: a region is
summarised when its 8th token arrives).  Paged 64-token K/V with a random page
permutation, k = 512.

Every step: every region completed by the step is compared byte for byte with the oracle's
compression of the same 8 rows, and no other slot changes.  For the shortest, the median
and the longest request the oracle keeps its own summaries (compressed from index_k, updated
as regions complete) and checks scores, the GPU selector on the oracle's scores, the
selection from the GPU's scores and the attention output.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa, pipeline
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits, bf16_from_bits_np, selection_differs_only_near_threshold

pytestmark = pytest.mark.gpu
G, PAGE = 4, 64


def compact_cache(kc, vc, bt_row, regions, p):
    """Host copies of only the pages the given regions' tokens (t <= p) touch, with the
    block-table row remapped to them (input marshalling for the oracle)."""
    toks = (np.asarray(regions, np.int64)[:, None] * 8 + np.arange(8)[None, :]).ravel()
    toks = toks[(toks >= 0) & (toks <= p)]
    jp = np.unique(toks // PAGE)
    pages = bt_row[jp]
    idx = torch.from_numpy(pages.astype(np.int64)).to(kc.device)
    kcs, vcs = bits(kc[idx]), bits(vc[idx])
    row = np.full(bt_row.shape[0], -1, np.int32)
    row[jp] = np.arange(len(jp), dtype=np.int32)
    return kcs, vcs, row[None, :]


def test_ragged_streaming_decode_8_steps():
    dev = torch.device("cuda")
    k, n_req, n_steps = 512, 32, 8
    lengths = W.ragged_lengths(n_req, seed=1239)
    d = W.decode_batch(lengths, seed=1239, device=dev, permute=True, extra_tokens=n_steps + 8)
    n_slots = d["n_slots"]
    S = torch.zeros((G, n_slots, 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((G, n_slots), dtype=torch.float32, device=dev)
    pipeline.compress_all(d["index_k"], lengths, d["tok_base"], d["sum_base"], S, C)
    ld = max(L + n_steps for L in lengths) // 8
    sd = pipeline.StreamingDecode(S, C, d["sum_base"], d["block_table"], d["k_cache"], d["v_cache"], lengths, ld, k)
    order = np.argsort(lengths)
    sampled = [int(order[0]), int(order[n_req // 2]), int(order[-1])]
    tb = [int(x) for x in d["tok_base"]]
    sb = [int(x) for x in d["sum_base"].tolist()]
    bt = d["block_table"].cpu().numpy()
    # the oracle's own summaries for the sampled requests (request-local pools)
    ik = {}
    pools = {}
    for b in sampled:
        cap = lengths[b] + n_steps + 8
        ik[b] = bits(d["index_k"][tb[b]: tb[b] + cap])
        n = lengths[b] // 8
        pools[b] = oracle.compress_regions(ik[b], [8 * r for r in range(n)], list(range(n)), (cap + 7) // 8)
    gen = W.generator(77, dev)
    for s in range(n_steps):
        pos = sd.positions()
        # the new tokens' index_k rows: the tail block of each request holds its region so far
        tail = torch.stack([d["index_k"][tb[b] + 8 * (p // 8): tb[b] + 8 * (p // 8) + 8] for b, p in enumerate(pos)])
        sd.step.tail.copy_(tail.view(-1, G, 256))
        index_q = W.normal_bf16((n_req, 16, 256), gen, dev)
        gate = W.uniform_f32((n_req, 16), gen, dev)
        q = W.normal_bf16((n_req, 64, 192), gen, dev)
        S_before = S.clone()
        out, due = sd.run(index_q, gate, q)
        dsa.check_device()
        assert due == [b for b, p in enumerate(pos) if p % 8 == 7]
        # compression: the completed regions, byte for byte; nothing else changed
        changed = torch.zeros(n_slots, dtype=torch.bool, device=dev)
        for b in due:
            slot = sb[b] + pos[b] // 8
            rows = bits(d["index_k"][tb[b] + 8 * (pos[b] // 8): tb[b] + 8 * (pos[b] // 8) + 8])
            So1, Co1 = oracle.compress_regions(rows, [0], [0], 1)
            assert np.array_equal(S[:, slot].cpu().numpy(), So1[:, 0])
            assert np.array_equal(C[:, slot].cpu().numpy(), Co1[:, 0])
            changed[slot] = True
        assert torch.equal(S[:, ~changed], S_before[:, ~changed])
        # sampled requests: scores, selection, attention
        sel = sd.step.sel_idx.cpu().numpy()
        cnt = sd.step.sel_count.cpu().numpy()
        sg = sd.step.scores.cpu().numpy()
        for b in sampled:
            p = pos[b]
            own = p // 8
            Sb, Cb = pools[b]
            so = oracle.indexer_scores(bits(index_q[b: b + 1]), gate[b: b + 1].cpu().numpy(), [0], [p], Sb, Cb, [0],
                                       ld=ld)
            err = np.abs(sg[b, :, :own] - so[0, :, :own]).max() / np.abs(so[0, :, :own]).max()
            assert err <= 1e-4, (s, b, err)
            so0 = np.nan_to_num(so)
            io, co = oracle.topk_regions(so0, [p], k)
            ig, cg = dsa.topk_regions(torch.from_numpy(so0).to(dev), torch.tensor([p], dtype=torch.int32, device=dev), k)
            assert np.array_equal(cg.cpu().numpy(), co) and np.array_equal(ig.cpu().numpy(), io)
            selection_differs_only_near_threshold(sel[b: b + 1], cnt[b: b + 1], io, co, so0, [p], k)
            regs = np.unique(sel[b, :, : cnt[b].max()].ravel())
            regs = regs[regs >= 0]
            kcs, vcs, row = compact_cache(d["k_cache"], d["v_cache"], bt[b], regs, p)
            oo, lo = oracle.sparse_attention(bits(q[b: b + 1]), kcs, vcs, row, [0], [p], sel[b: b + 1], cnt[b: b + 1])
            og = out[b: b + 1].float().cpu().numpy()
            of = bf16_from_bits_np(oo)
            assert np.all(np.abs(og - of) <= 2e-2 + 1e-2 * np.abs(of)), (s, b)
            np.testing.assert_allclose(sd.step.lse[b: b + 1].cpu().numpy(), lo, rtol=1e-3, atol=1e-3)
            # the oracle's pool learns the region this step completed
            if p % 8 == 7:
                oracle.compress_regions(ik[b], [8 * own], [own], Sb.shape[1], Sb, Cb)
