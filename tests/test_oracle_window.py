"""Pins for the oracle's sliding-window attention (the window layers beside DSA).

[P1] kwkr.cn/news/601179 §滑窗注意力: the window layers read only the most recent 512
tokens (sliding_window 512), and their cache is a ring buffer that keeps nothing older;
[P2] Step-5-Preview 如何实现1M长上下文 §第一招: the ring buffer writes a new token over the
slot `position mod 512`, and decode runs attention inside the window.  Fixed reading: a
query at position p attends tokens max(0, p - 511) .. p (the window holds the query's own
token and the 511 before it), softmax(q K^T / sqrt(192)) V, head h using KV group h // 16.

Pins: dense attention over the window's tokens (torch's scaled_dot_product_attention in
float64, a library routine the oracle does not use), a one-token window returning v_p
exactly, an aligned window equal to the DSA oracle over the window's regions, a 512-slot
ring buffer (8 pages used cyclically, later tokens overwriting earlier ones) giving the same
result as the linear cache, and tokens outside the window having no effect.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits, f64

G, HQ, D, PAGE = 4, 64, 192, 64


def gather_tokens(kc, bt_row, lo, hi):
    """[hi - lo][4][192] rows of tokens lo .. hi-1 (t -> page bt[t//64], row t%64)."""
    t = torch.arange(lo, hi)
    return kc[bt_row[t // PAGE].long(), :, t % PAGE, :]


def dense_window(q, kc, vc, bt_row, p, window):
    """torch SDPA in float64 over tokens max(0, p-window+1) .. p (the query is the last row)."""
    lo = max(0, p - window + 1)
    K = gather_tokens(kc, bt_row, lo, p + 1).to(torch.float64)
    V = gather_tokens(vc, bt_row, lo, p + 1).to(torch.float64)
    Qh = q.to(torch.float64)[:, None, :]                               # [64][1][192]
    Kh = K.permute(1, 0, 2).repeat_interleave(HQ // G, dim=0)          # [64][T][192]
    Vh = V.permute(1, 0, 2).repeat_interleave(HQ // G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(Qh, Kh, Vh)[:, 0, :]
    lse = torch.logsumexp((Qh @ Kh.transpose(1, 2)) / np.sqrt(D), dim=-1)[:, 0]
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("L,window", [(300, 512), (1500, 512), (777, 100), (2048, 512)])
def test_equals_dense_attention_over_the_window(L, window):
    d = W.decode_batch([L], seed=L + window, device="cpu", permute=True)
    p = L - 1
    out, lse, o64 = oracle.window_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                            d["block_table"].numpy(), [0], [p], window, want_f64=True)
    ref, ref_lse = dense_window(d["q"][0], d["k_cache"], d["v_cache"], d["block_table"][0], p, window)
    np.testing.assert_allclose(o64[0], ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_lse, rtol=1e-6)
    assert np.array_equal(out[0], oracle.f64_to_bf16(o64[0].ravel()).reshape(HQ, D))


def test_one_token_window_returns_v_exactly():
    d = W.decode_batch([200], seed=3, device="cpu", permute=False)
    p = 137
    out, lse = oracle.window_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                       d["block_table"].numpy(), [0], [p], 1)
    v = bits(d["v_cache"][p // PAGE, :, p % PAGE, :])                   # [4][192]
    k = f64(bits(d["k_cache"][p // PAGE, :, p % PAGE, :]))
    q = f64(bits(d["q"][0]))
    for h in range(HQ):
        assert np.array_equal(out[0, h], v[h // 16])
        assert np.isclose(lse[0, h], q[h] @ k[h // 16] / np.sqrt(D), rtol=1e-6)


@pytest.mark.parametrize("p,window", [(1023, 512), (1535, 256), (519, 512)])
def test_region_aligned_window_equals_dsa_over_its_regions(p, window):
    # window start p - window + 1 a multiple of 8: the window is whole regions
    assert (p - window + 1) % 8 == 0 or p < window
    d = W.decode_batch([p + 1], seed=p, device="cpu", permute=True)
    lo = max(0, p - window + 1)
    regs = np.arange(lo // 8, p // 8 + 1, dtype=np.int32)
    sel = np.tile(regs, (1, G, 1))
    cnt = np.full((1, G), regs.size, np.int32)
    a = oracle.window_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                d["block_table"].numpy(), [0], [p], window, want_f64=True)
    b = oracle.sparse_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                d["block_table"].numpy(), [0], [p], sel, cnt, want_f64=True)
    if p >= window:
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2])
    else:                                  # window covers 0..p: every region selected
        np.testing.assert_allclose(a[2], b[2], rtol=1e-12, atol=1e-14)


def ring_cache(kc, vc, bt, lengths, n_ring_pages=8):
    """The same tokens written one by one into per-request rings of n_ring_pages pages:
    token t of request b goes to ring page ring[b][(t // 64) % n], row t % 64, overwriting
    whatever was there.  Returns (k_ring, v_ring, cyclic block table)."""
    B = len(lengths)
    max_pages = int(bt.shape[1])
    kr = torch.zeros((B * n_ring_pages, G, PAGE, D), dtype=kc.dtype)
    vr = torch.zeros_like(kr)
    cyc = torch.zeros((B, max_pages), dtype=torch.int32)
    for b, L in enumerate(lengths):
        for vp in range(max_pages):
            cyc[b, vp] = b * n_ring_pages + vp % n_ring_pages
        for t in range(L):
            src_page = int(bt[b, t // PAGE])
            dst_page = b * n_ring_pages + (t // PAGE) % n_ring_pages
            kr[dst_page, :, t % PAGE, :] = kc[src_page, :, t % PAGE, :]
            vr[dst_page, :, t % PAGE, :] = vc[src_page, :, t % PAGE, :]
    return kr, vr, cyc


def test_ring_buffer_equals_linear_cache():
    lengths = [1500, 700, 200]
    d = W.decode_batch(lengths, seed=17, device="cpu", permute=True)
    kr, vr, cyc = ring_cache(d["k_cache"], d["v_cache"], d["block_table"], lengths)
    qp = d["q_pos"].numpy()
    lin = oracle.window_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                  d["block_table"].numpy(), d["q_req"].numpy(), qp, 512)
    rng = oracle.window_attention(bits(d["q"]), bits(kr), bits(vr), cyc.numpy(), d["q_req"].numpy(), qp, 512)
    assert np.array_equal(lin[0], rng[0]) and np.array_equal(lin[1], rng[1])
    # the ring really was overwritten: a window of 600 reads slots that now hold newer tokens
    wide = oracle.window_attention(bits(d["q"][:1]), bits(kr), bits(vr), cyc.numpy(), [0], [qp[0]], 600)
    lin_wide = oracle.window_attention(bits(d["q"][:1]), bits(d["k_cache"]), bits(d["v_cache"]),
                                       d["block_table"].numpy(), [0], [qp[0]], 600)
    assert not np.array_equal(wide[0], lin_wide[0])


def test_tokens_outside_the_window_have_no_effect():
    d = W.decode_batch([1100], seed=23, device="cpu", permute=False)
    p, window = 1099, 512
    lo = p - window + 1
    base = oracle.window_attention(bits(d["q"]), bits(d["k_cache"]), bits(d["v_cache"]),
                                   d["block_table"].numpy(), [0], [p], window)
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    for t in (0, 17, lo - 1):                                   # outside: no change at all
        kc[t // PAGE, :, t % PAGE, :] = 40.0
        vc[t // PAGE, :, t % PAGE, :] = -40.0
    same = oracle.window_attention(bits(d["q"]), bits(kc), bits(vc), d["block_table"].numpy(), [0], [p], window)
    assert np.array_equal(base[0], same[0]) and np.array_equal(base[1], same[1])
    vc[lo // PAGE, :, lo % PAGE, :] = -40.0                      # the first token inside: changes
    diff = oracle.window_attention(bits(d["q"]), bits(kc), bits(vc), d["block_table"].numpy(), [0], [p], window)
    assert not np.array_equal(base[0], diff[0])
