"""Pins for the oracle's sparse GQA attention (step A4) and the whole oracle pipeline.

[P1] kwkr.cn/news/601179 §DSA ④: exact attention over the real K/V of the selected
regions only; [P3] 100 万 token 上下文实测 §一: 64 query heads / 4 KV groups, paged
K/V gathered through the block_table.  Fixed reading: softmax(q K^T / sqrt(192)) V over
the selected tokens t <= p, head h using KV group h // 16.

The central pin: when k covers every region (L <= 4096 with k = 512), DSA equals dense
causal GQA, evaluated here by torch's scaled_dot_product_attention in float64.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits, f64

G, HQ, D, PAGE = 4, 64, 192, 64


def gather_tokens(kc, bt_row, n):
    """[n tokens][4][192] view of a request's cache (t -> page bt[t//64], row t%64)."""
    t = torch.arange(n)
    return kc[bt_row[t // PAGE].long(), :, t % PAGE, :]      # [n][4][192]


def dense_reference(q, kc, vc, bt_row, p):
    """torch SDPA, float64, over tokens 0..p: the query is the last row."""
    K = gather_tokens(kc, bt_row, p + 1).to(torch.float64)    # [T][4][192]
    V = gather_tokens(vc, bt_row, p + 1).to(torch.float64)
    Qh = q.to(torch.float64)[None]                            # [1][64][192]
    Kh = K.permute(1, 0, 2).repeat_interleave(HQ // G, dim=0)  # [64][T][192]
    Vh = V.permute(1, 0, 2).repeat_interleave(HQ // G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(
        Qh.permute(1, 0, 2), Kh, Vh)                          # [64][1][192]
    logits = (Qh.permute(1, 0, 2) @ Kh.transpose(1, 2)) / np.sqrt(D)
    lse = torch.logsumexp(logits, dim=-1)[:, 0]
    return o[:, 0, :].numpy(), lse.numpy()


def run_pipeline(d, k):
    """Oracle A1..A4 for the decode batch d (one query per request)."""
    src, dst = W.complete_regions(d["lengths"], d["tok_base"], d["sum_base"])
    S, C = oracle.compress_regions(bits(d["index_k"]), src, dst, d["n_slots"])
    qp = d["q_pos"].numpy()
    sc = oracle.indexer_scores(bits(d["index_q"]), d["gate"].numpy(), d["q_req"].numpy(), qp, S, C,
                               d["sum_base"].numpy(), ld=max(1, int(qp.max()) // 8))
    idx, cnt = oracle.topk_regions(np.nan_to_num(sc, nan=0.0), qp, k)
    out, lse, o64 = oracle.sparse_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                            d["block_table"].numpy(), d["q_req"].numpy(), qp, idx,
                                            cnt, want_f64=True)
    return out, lse, o64, idx, cnt


@pytest.mark.parametrize("L,permute", [(200, False), (517, True), (1024, True), (4096, True)])
def test_dense_equivalence_when_k_covers_every_region(L, permute):
    d = W.decode_batch([L], seed=100 + L, device="cpu", permute=permute)
    out, lse, o64, idx, cnt = run_pipeline(d, k=512)
    assert np.all(cnt[0] == (L - 1) // 8 + 1)
    if L == 4096:
        # the boundary: k = 512 equals the region count R = L / 8, so every region is selected
        assert np.all(cnt[0] == 512) and L // 8 == 512
        assert np.array_equal(idx[0], np.tile(np.arange(512, dtype=idx.dtype), (G, 1)))
    ref, ref_lse = dense_reference(d["q"][0], d["k_cache"], d["v_cache"], d["block_table"][0], L - 1)
    np.testing.assert_allclose(o64[0], ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_lse, rtol=1e-6)
    # out is o64 rounded once to bf16
    assert np.array_equal(out[0], oracle.f64_to_bf16(o64[0].ravel()).reshape(HQ, D))


def test_two_regions_by_hand():
    # L = 16, p = 12: with k = 1 only the own region (tokens 8..12) is attended,
    # with k = 2 tokens 0..12
    d = W.decode_batch([13], seed=5, device="cpu", permute=False)
    kc, vc, bt = d["k_cache"], d["v_cache"], d["block_table"][0]
    q = bits(d["q"])
    for k, first in ((1, 8), (2, 0)):
        sel = np.full((1, G, k), -1, np.int32)
        sel[0, :, :k] = [1] if k == 1 else [0, 1]
        cnt = np.full((1, G), k, np.int32)
        out, lse, o64 = oracle.sparse_attention(q, bits(kc), bits(vc), bt[None].numpy(), [0], [12],
                                                sel, cnt, want_f64=True)
        K = gather_tokens(kc, bt, 13)[first:13].to(torch.float64)
        V = gather_tokens(vc, bt, 13)[first:13].to(torch.float64)
        for h in (0, 17, 63):
            g = h // 16
            lg = (K[:, g, :] @ torch.from_numpy(f64(q[0, h]))) / np.sqrt(D)
            w = torch.softmax(lg, 0)
            np.testing.assert_allclose(o64[0, h], (w[:, None] * V[:, g, :]).sum(0).numpy(), rtol=1e-12,
                                       atol=1e-14)


def test_single_token_returns_its_value_exactly():
    d = W.decode_batch([1], seed=6, device="cpu", permute=False)
    sel = np.zeros((1, G, 1), np.int32)
    cnt = np.ones((1, G), np.int32)
    out, lse = oracle.sparse_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                       d["block_table"].numpy(), [0], [0], sel, cnt)
    v0 = bits(d["v_cache"])[d["block_table"][0, 0], :, 0, :]          # [4][192]
    for h in range(HQ):
        assert np.array_equal(out[0, h], v0[h // 16])
    kq = f64(bits(d["k_cache"])[d["block_table"][0, 0], :, 0, :])
    qq = f64(bits(d["q"])[0])
    np.testing.assert_allclose(lse[0], [(qq[h] @ kq[h // 16]) / np.sqrt(D) for h in range(HQ)], rtol=1e-6)


def test_zero_query_averages_the_selected_values():
    d = W.decode_batch([64], seed=7, device="cpu", permute=True)
    q = np.zeros((1, HQ, D), np.uint16)
    sel = np.full((1, G, 3), -1, np.int32)
    sel[0, :, :2] = [2, 7]
    cnt = np.full((1, G), 2, np.int32)
    out, lse, o64 = oracle.sparse_attention(q, bits(d["k_cache"]), bits(d["v_cache"]),
                                            d["block_table"].numpy(), [0], [60], sel, cnt, want_f64=True)
    V = gather_tokens(d["v_cache"], d["block_table"][0], 64).to(torch.float64).numpy()
    toks = list(range(16, 24)) + list(range(56, 61))                    # t <= p = 60
    for h in range(HQ):
        np.testing.assert_allclose(o64[0, h], V[toks, h // 16].mean(0), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse[0], np.log(len(toks)), rtol=1e-7)


def test_empty_selection_gives_zero_and_minus_infinity():
    d = W.decode_batch([16], seed=8, device="cpu", permute=False)
    sel = np.full((1, G, 4), -1, np.int32)
    cnt = np.zeros((1, G), np.int32)
    out, lse = oracle.sparse_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                       d["block_table"].numpy(), [0], [15], sel, cnt)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_page_permutation_is_transparent():
    a = W.decode_batch([300], seed=9, device="cpu", permute=False)
    perm = torch.randperm(a["k_cache"].shape[0], generator=torch.Generator().manual_seed(1))
    kc = torch.empty_like(a["k_cache"])
    vc = torch.empty_like(a["v_cache"])
    kc[perm] = a["k_cache"]
    vc[perm] = a["v_cache"]
    bt = perm[a["block_table"].long()].to(torch.int32)
    sel = np.tile(np.array([0, 9, 20, 37], np.int32), (1, G, 1))
    cnt = np.full((1, G), 4, np.int32)
    o1, l1 = oracle.sparse_attention(bits(a["q"]), bits(a["k_cache"]), bits(a["v_cache"]),
                                     a["block_table"].numpy(), [0], [299], sel, cnt)
    o2, l2 = oracle.sparse_attention(bits(a["q"]), bits(kc), bits(vc), bt.numpy(), [0], [299], sel, cnt)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_kv_head_map_16_query_heads_per_group():
    # changing group g's K/V changes exactly heads 16g..16g+15
    d = W.decode_batch([40], seed=10, device="cpu", permute=False)
    sel = np.tile(np.arange(5, dtype=np.int32), (1, G, 1))
    cnt = np.full((1, G), 5, np.int32)
    args = (bits(d["q"]), bits(d["k_cache"]), d["block_table"].numpy(), [0], [39], sel, cnt)
    vc = bits(d["v_cache"])
    o1, _ = oracle.sparse_attention(args[0], args[1], vc, *args[2:])
    vc2 = vc.copy()
    vc2[:, 2] ^= 0x0001                      # perturb group 2's values in every page
    o2, _ = oracle.sparse_attention(args[0], args[1], vc2, *args[2:])
    changed = [h for h in range(HQ) if not np.array_equal(o1[0, h], o2[0, h])]
    assert set(changed) <= set(range(32, 48)) and len(changed) > 8
