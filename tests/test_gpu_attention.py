"""GPU sparse attention (A4) against the oracle on the same selections: bf16 outputs
within 2e-2 absolute + 1e-2 relative, lse within 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits, bf16_from_bits_np

pytestmark = pytest.mark.gpu
G = 4


def random_selection(q_pos, k, seed, force_own=True):
    rng = np.random.default_rng(seed)
    nq = len(q_pos)
    idx = np.full((nq, G, k), -1, np.int32)
    cnt = np.zeros((nq, G), np.int32)
    for i, p in enumerate(q_pos):
        own = p // 8
        for g in range(G):
            n = min(k, own + 1)
            pick = rng.choice(own, size=n - 1, replace=False) if n > 1 else np.array([], np.int64)
            s = np.sort(np.concatenate([pick, [own]]).astype(np.int32))
            idx[i, g, :n] = s
            cnt[i, g] = n
    return idx, cnt


def run(d, idx, cnt, q_req=None, prefill=False):
    dev = "cuda"
    si = torch.from_numpy(idx).to(dev)
    sc = torch.from_numpy(cnt).to(dev)
    nq = idx.shape[0]
    lse = torch.empty((nq, 64), dtype=torch.float32, device=dev)
    q = d["q"][:nq].contiguous()
    if prefill:
        out = dsa.sparse_attn_prefill(q, d["k_cache"], d["v_cache"], d["block_table"], q_req, d["q_pos"], si, sc,
                                      lse=lse)
    else:
        out = dsa.sparse_attn_decode(q, d["k_cache"], d["v_cache"], d["block_table"], d["q_pos"], si, sc, lse=lse)
    dsa.check_device()
    qr = np.arange(nq) if q_req is None else q_req.cpu().numpy()
    oo, lo = oracle.sparse_attention(bits(q), bits(d["k_cache"]), bits(d["v_cache"]), d["block_table"].cpu().numpy(),
                                     qr, d["q_pos"].cpu().numpy(), idx, cnt)
    og = out.float().cpu().numpy()
    of = bf16_from_bits_np(oo)
    err = np.abs(og - of)
    assert np.all(err <= 2e-2 + 1e-2 * np.abs(of)), err.max()
    lg = lse.cpu().numpy()
    fin = np.isfinite(lo)
    assert np.array_equal(np.isfinite(lg), fin)
    np.testing.assert_allclose(lg[fin], lo[fin], rtol=1e-3, atol=1e-3)
    return err.max()


@pytest.mark.parametrize("k", [1, 5, 16, 64, 512])
def test_decode_random_selections(k):
    lengths = [16384, 9000 + 3, 600 + 7]
    d = W.decode_batch(lengths, seed=30 + k, device="cuda", permute=True)
    idx, cnt = random_selection(d["q_pos"].cpu().numpy(), k, seed=k)
    e = run(d, idx, cnt)
    print(f"k={k} max abs err {e:.3e}")


def test_prefill_many_rows_single_pass():
    # >= 2 * SMs (query, group) rows: each CTA covers a whole selection (no split)
    ctx = 4096
    d = W.prefill_chunk(ctx, 160, seed=33, device="cuda", permute=True)
    qp = d["q_pos"].cpu().numpy()
    idx, cnt = random_selection(qp, 64, seed=3)
    run(d, idx, cnt, q_req=d["q_req"], prefill=True)


def test_causal_mask_inside_the_own_region():
    # queries at every offset of a region; the own region alone is selected
    d = W.decode_batch([8 * 20 + 8], seed=34, device="cuda", permute=False)
    dev = "cuda"
    nq = 8
    pos = torch.arange(8 * 20, 8 * 21, dtype=torch.int32, device=dev)
    d["q_pos"] = pos
    d["q"] = W.normal_bf16((nq, 64, 192), W.generator(9, dev), dev)
    idx = np.full((nq, G, 2), -1, np.int32)
    idx[:, :, 0] = 20
    cnt = np.ones((nq, G), np.int32)
    run(d, idx, cnt, q_req=torch.zeros(nq, dtype=torch.int32, device=dev), prefill=True)


def test_empty_selection_and_bad_region():
    d = W.decode_batch([1000], seed=35, device="cuda")
    idx = np.full((1, G, 4), -1, np.int32)
    cnt = np.zeros((1, G), np.int32)
    idx[0, 1, :2] = [3, 124]
    cnt[0, 1] = 2
    run(d, idx, cnt)
    idx[0, 2, 0] = 99999                       # beyond the block table: flagged, skipped
    cnt[0, 2] = 1
    si = torch.from_numpy(idx).cuda()
    sc = torch.from_numpy(cnt).cuda()
    dsa.sparse_attn_decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["q_pos"], si, sc)
    with pytest.raises(dsa.DsaError):
        dsa.check_device()


def test_prefill_queries_of_several_requests_in_one_block():
    # 40 queries cycling over 3 requests: every block of 8 serves its queries in one pass per
    # request (the shared-selection kernel); random, unrelated selections (k = 64) mask most of
    # each union away from each query
    dev = "cuda"
    d = W.decode_batch([5000, 3000 + 5, 7000], seed=36, device=dev, permute=True)
    nq = 40
    rng = np.random.default_rng(7)
    lens = [5000, 3005, 7000]
    q_req = np.arange(nq, dtype=np.int32) % 3
    q_pos = np.array([rng.integers(8, lens[b]) for b in q_req], np.int32)
    d["q_pos"] = torch.from_numpy(q_pos).to(dev)
    d["q"] = W.normal_bf16((nq, 64, 192), W.generator(10, dev), dev)
    idx, cnt = random_selection(q_pos, 64, seed=8)
    run(d, idx, cnt, q_req=torch.from_numpy(q_req).to(dev), prefill=True)


def test_prefill_shared_block_with_empty_and_overlapping_selections():
    # 48 queries of one request: neighbours share most of their regions, some rows select
    # nothing at all, one query's last block is partial
    dev = "cuda"
    ctx = 6000
    d = W.prefill_chunk(ctx, 45, seed=37, device=dev, permute=True)
    qp = d["q_pos"].cpu().numpy()
    idx, cnt = random_selection(qp, 128, seed=9)
    base = idx[0, :, :100].copy()                  # a common core for everyone
    for i in range(1, len(qp)):
        idx[i, :, :100] = base
        idx[i] = np.sort(np.where(idx[i] < 0, 10 ** 9, idx[i]), axis=1)
        idx[i] = np.where(idx[i] == 10 ** 9, -1, idx[i])
        for g in range(G):
            row = np.unique(idx[i, g][idx[i, g] >= 0])
            idx[i, g] = -1
            idx[i, g, : len(row)] = row
            cnt[i, g] = len(row)
    cnt[5, 2] = 0
    idx[5, 2] = -1
    cnt[17] = 0
    idx[17] = -1
    run(d, idx, cnt, q_req=d["q_req"], prefill=True)


def test_prefill_shared_block_running_max_grows():
    # 48 queries in six blocks of 8 (one region each), every block sharing one selection of
    # 200 regions; the K rows of region r are scaled by 1 + r / 16, so along the union (in
    # region order) each row's running max climbs past the lazy-rescale slack again and again
    # and the shared kernel rescales O in TMEM several times per row
    dev = "cuda"
    ctx = 6000
    d = W.prefill_chunk(ctx, 48, seed=41, device=dev, permute=True)
    bt = d["block_table"][0]
    n_log = (ctx + 48 + 63) // 64
    rows = torch.arange(n_log * 64, device=dev) // 8                 # region of each logical row
    scale = (1.0 + rows.float() / 16).view(n_log, 1, 64, 1)
    kc = d["k_cache"].float()
    kc[bt[:n_log].long()] *= scale
    d["k_cache"] = kc.to(torch.bfloat16)
    qp = d["q_pos"].cpu().numpy()
    rng = np.random.default_rng(12)
    k = 256
    idx = np.full((48, G, k), -1, np.int32)
    cnt = np.zeros((48, G), np.int32)
    for b in range(6):
        own = int(qp[8 * b]) // 8
        for g in range(G):
            sel = np.sort(np.concatenate([rng.choice(own, 199, replace=False), [own]])).astype(np.int32)
            idx[8 * b: 8 * b + 8, g, :200] = sel
            cnt[8 * b: 8 * b + 8, g] = 200
    run(d, idx, cnt, q_req=d["q_req"], prefill=True)


@pytest.mark.parametrize("grow", [False, True])
def test_prefill_rows_on_tcgen05(grow):
    # 96 queries x 4 groups = 384 rows (more than two per SM: the tcgen05 per-row kernel, each
    # persistent CTA streaming two or three rows back to back), selections of 512 regions (32
    # tiles of 128 tokens) beside ragged ones (1, 17, 129 regions) and empty rows; with grow, K
    # of region r is scaled by 1 + r/64 so every row's running max
    # passes the slack many times (O^T rescaled in TMEM)
    ctx, n_new = 16384, 96
    dev = "cuda"
    d = W.prefill_chunk(ctx, n_new, seed=51 + grow, device=dev, permute=True)
    if grow:
        kc = d["k_cache"].float()
        bt = d["block_table"][0].long()
        rs = torch.zeros(kc.shape[0], device=dev)
        rs[bt] = torch.arange(bt.numel(), device=dev, dtype=torch.float32)   # page -> its first region / 8
        scale = 1.0 + (rs[:, None, None, None] * 8 + torch.arange(64, device=dev)[None, None, :, None] // 8) / 64.0
        d["k_cache"] = (kc * scale).to(torch.bfloat16)
    qp = d["q_pos"].cpu().numpy()
    idx, cnt = random_selection(qp, 512, seed=7 + grow)
    for i, n in ((3, 1), (10, 17), (20, 129), (33, 0), (47, 0)):
        for g in range(G):
            if n:
                own = qp[i] // 8
                keep = np.sort(np.concatenate([idx[i, g, : cnt[i, g] - 1][:n - 1], [own]]))
                idx[i, g, :] = -1
                idx[i, g, :n] = keep
            else:
                idx[i, g, :] = -1
            cnt[i, g] = n
    run(d, idx, cnt, q_req=d["q_req"], prefill=True)
