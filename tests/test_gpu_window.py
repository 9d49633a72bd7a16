"""GPU sliding-window attention of the window layers (dsa_window_attn) and the ring buffer
write (dsa_kv_append) against the oracle's window attention.

[P1] kwkr.cn/news/601179 §滑窗注意力: the window layers read the most recent 512 tokens;
[P2] Step-5-Preview 如何实现1M长上下文 §第一招: their cache is a ring buffer written by a
modulo of the position.  Bar as for the sparse attention: bf16 outputs within 2e-2
absolute + 1e-2 relative of the oracle's, lse within 1e-3.  Cases: decode batches on a
linear paged cache (windows shorter than, equal to and longer than the context, window
sizes 1 .. 4,096, a 1M-token context; up to 624 tokens the clustered kernel with its in-kernel
merge, beyond it the split kernel and the combine), many queries of one request (the per-row kernel
without splits, a prefill chunk's shape), a ring of 8 pages per request filled token by
token through dsa_kv_append across several wraps, and an append beyond the block table
(flagged, nothing written).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa
from sparse_long_context_dsa_b200 import workloads as W

from _util import bits, bf16_from_bits_np

pytestmark = pytest.mark.gpu
G, PAGE = 4, 64


def check(q, kc, vc, bt, q_req, q_pos, window, out, lse):
    oo, lo = oracle.window_attention(bits(q), bits(kc), bits(vc), bt.cpu().numpy(), q_req, q_pos, window)
    og = out.float().cpu().numpy()
    of = bf16_from_bits_np(oo)
    err = np.abs(og - of)
    assert np.all(err <= 2e-2 + 1e-2 * np.abs(of)), err.max()
    lg = lse.cpu().numpy()
    fin = np.isfinite(lo)
    assert np.array_equal(np.isfinite(lg), fin)
    np.testing.assert_allclose(lg[fin], lo[fin], rtol=1e-3, atol=1e-3)


@pytest.mark.parametrize("lengths,window", [
    ([200, 511, 512, 513, 1500], 512),
    ([1500, 3000], 1),
    ([1500, 3000], 100),
    ([9000, 5000, 40000], 4096),
    ([1 << 20], 512),
    ([5000, 700, 2000], 600),            # 77 regions: the clustered kernel's last CTAs partly filled
    ([3000, 640, 625], 624),             # 80 regions: every region slot of the clustered kernel
])
def test_decode_batch_matches_oracle(lengths, window):
    d = W.decode_batch(lengths, seed=sum(lengths) % 1000 + window, device="cuda", permute=True)
    nq = len(lengths)
    lse = torch.empty((nq, 64), dtype=torch.float32, device="cuda")
    out = dsa.window_attn(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["q_pos"], window, lse=lse)
    dsa.check_device()
    check(d["q"], d["k_cache"], d["v_cache"], d["block_table"], np.arange(nq), d["q_pos"].cpu().numpy(), window,
          out, lse)


def test_many_queries_of_one_request():
    # a chunk's shape: 1,200 consecutive positions of one request (enough rows for one CTA
    # per row), checked on a sample of rows
    ctx, n_new = 3000, 1200
    d = W.prefill_chunk(ctx, n_new, seed=8, device="cuda", permute=True)
    lse = torch.empty((n_new, 64), dtype=torch.float32, device="cuda")
    out = dsa.window_attn(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["q_pos"], 512, q_req=d["q_req"],
                          lse=lse)
    dsa.check_device()
    rows = np.array([0, 1, 7, 8, 300, 511, 512, 999, n_new - 1])
    qp = d["q_pos"].cpu().numpy()[rows]
    check(d["q"][rows], d["k_cache"], d["v_cache"], d["block_table"], np.zeros(len(rows), np.int64), qp, 512,
          out[rows], lse[rows])


def test_ring_buffer_through_kv_append():
    # requests of different lengths; each step appends one token per request into an
    # 8-page ring (512 slots) and attends over the last 512 tokens; the reference reads the
    # same tokens from the linear cache they came from
    lengths = [700, 1030, 60]
    steps = 40
    d = W.decode_batch([L + steps for L in lengths], seed=31, device="cuda", permute=True)
    B = len(lengths)
    ring_pages = 8
    max_pages = d["block_table"].shape[1]
    cyc = (torch.arange(B, dtype=torch.int32)[:, None] * ring_pages +
           torch.arange(max_pages, dtype=torch.int32)[None] % ring_pages).to("cuda")
    kr = torch.zeros((B * ring_pages, G, PAGE, 192), dtype=torch.bfloat16, device="cuda")
    vr = torch.zeros_like(kr)
    bt = d["block_table"]

    def token_rows(cache, b, t):
        t = torch.as_tensor(t, device="cuda")
        return cache[bt[b, t // PAGE].long(), :, t % PAGE, :]            # [n][4][192]

    # fill each ring with its request's first L tokens, one append call per request
    for b, L in enumerate(lengths):
        pos = torch.arange(L, dtype=torch.int32, device="cuda")
        # slots repeat every 512 tokens: append in order, one window's worth per call
        for s in range(0, L, 512):
            p = pos[s:s + 512]
            req = torch.full_like(p, b)
            dsa.kv_append(kr, vr, cyc, p, token_rows(d["k_cache"], b, p.long()).contiguous(),
                          token_rows(d["v_cache"], b, p.long()).contiguous(), q_req=req)
    dsa.check_device()
    for step in range(steps):
        pos = torch.tensor([L + step for L in lengths], dtype=torch.int32, device="cuda")
        newk = torch.stack([token_rows(d["k_cache"], b, int(pos[b])) for b in range(B)]).contiguous()
        newv = torch.stack([token_rows(d["v_cache"], b, int(pos[b])) for b in range(B)]).contiguous()
        dsa.kv_append(kr, vr, cyc, pos, newk, newv)
        lse = torch.empty((B, 64), dtype=torch.float32, device="cuda")
        out = dsa.window_attn(d["q"], kr, vr, cyc, pos, 512, lse=lse)
        dsa.check_device()
        if step in (0, 1, 17, steps - 1):
            check(d["q"], d["k_cache"], d["v_cache"], bt, np.arange(B), pos.cpu().numpy(), 512, out, lse)


def test_append_beyond_the_block_table_is_flagged_and_skipped():
    kr = torch.zeros((2, G, PAGE, 192), dtype=torch.bfloat16, device="cuda")
    vr = torch.zeros_like(kr)
    bt = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    pos = torch.tensor([2 * PAGE], dtype=torch.int32, device="cuda")          # page 2: beyond the table
    new = torch.ones((1, G, 192), dtype=torch.bfloat16, device="cuda")
    dsa.kv_append(kr, vr, bt, pos, new, new)
    with pytest.raises(dsa.DsaError):
        dsa.check_device()
    assert not kr.any() and not vr.any()


@pytest.mark.parametrize("window", [512, 4096])
def test_window_decode_equals_append_then_attention(window):
    # dsa_window_decode (the append folded into the clustered kernel at 512 tokens; the two
    # calls at 4,096) against kv_append + window_attn on a copy of the same rings, step by
    # step: outputs, LSE and ring contents bit for bit, and the oracle on some steps
    lengths = [700, 1030, 60, 4200]
    steps = 12
    d = W.decode_batch([L + steps for L in lengths], seed=57 + window, device="cuda", permute=True)
    B = len(lengths)
    ring_pages = (window + PAGE - 1) // PAGE + 1
    max_pages = d["block_table"].shape[1]
    cyc = (torch.arange(B, dtype=torch.int32)[:, None] * ring_pages +
           torch.arange(max_pages, dtype=torch.int32)[None] % ring_pages).to("cuda")
    bt = d["block_table"]

    def token_rows(cache, b, t):
        t = torch.as_tensor(t, device="cuda")
        return cache[bt[b, t // PAGE].long(), :, t % PAGE, :]

    kr = torch.zeros((B * ring_pages, G, PAGE, 192), dtype=torch.bfloat16, device="cuda")
    vr = torch.zeros_like(kr)
    slots = ring_pages * PAGE
    for b, L in enumerate(lengths):
        pos = torch.arange(max(0, L - slots), L, dtype=torch.int32, device="cuda")
        dsa.kv_append(kr, vr, cyc, pos, token_rows(d["k_cache"], b, pos.long()).contiguous(),
                      token_rows(d["v_cache"], b, pos.long()).contiguous(), q_req=torch.full_like(pos, b))
    kr2, vr2 = kr.clone(), vr.clone()
    dsa.check_device()
    for step in range(steps):
        pos = torch.tensor([L + step for L in lengths], dtype=torch.int32, device="cuda")
        newk = torch.stack([token_rows(d["k_cache"], b, int(pos[b])) for b in range(B)]).contiguous()
        newv = torch.stack([token_rows(d["v_cache"], b, int(pos[b])) for b in range(B)]).contiguous()
        lse = torch.empty((B, 64), dtype=torch.float32, device="cuda")
        out = dsa.window_decode(d["q"], kr, vr, cyc, pos, newk, newv, window, lse=lse)
        dsa.kv_append(kr2, vr2, cyc, pos, newk, newv)
        lse2 = torch.empty((B, 64), dtype=torch.float32, device="cuda")
        out2 = dsa.window_attn(d["q"], kr2, vr2, cyc, pos, window, lse=lse2)
        dsa.check_device()
        assert torch.equal(out, out2) and torch.equal(lse, lse2)
        assert torch.equal(kr, kr2) and torch.equal(vr, vr2)
        if step in (0, steps - 1):
            check(d["q"], d["k_cache"], d["v_cache"], bt, np.arange(B), pos.cpu().numpy(), window, out, lse)
    assert dsa.lib().dsa_window_decode_launches(B, window) == (1 if window == 512 else 3)


def test_window_step_runner_from_pinned_host_memory():
    # pipeline.WindowDecodeStep: inputs staged from a pinned host image of its arena by the
    # library's copy kernel, the output written into pinned host memory by the attention
    # kernel; equal to dsa.window_decode on a copy of the same rings
    from sparse_long_context_dsa_b200 import pipeline
    B, ring_pages, window = 3, 9, 512
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    bt = pipeline.ring_block_table(B, 20000, ring_pages, "cuda")
    kr = torch.randn((B * ring_pages, G, PAGE, 192), generator=g, device="cuda").to(torch.bfloat16)
    vr = torch.randn(kr.shape, generator=g, device="cuda").to(torch.bfloat16)
    kr2, vr2 = kr.clone(), vr.clone()
    st = pipeline.WindowDecodeStep(kr, vr, bt, window)
    q = torch.randn((B, 64, 192), generator=g, device="cuda").to(torch.bfloat16)
    nk = torch.randn((B, G, 192), generator=g, device="cuda").to(torch.bfloat16)
    nv = torch.randn((B, G, 192), generator=g, device="cuda").to(torch.bfloat16)
    pos = torch.tensor([1000, 70000, 511], dtype=torch.int32, device="cuda")
    st.load(q, nk, nv, pos)
    host = st.arena.cpu().pin_memory()
    st.arena.zero_()
    out_host = torch.empty((B, 64, 192), dtype=torch.bfloat16).pin_memory()
    st.stage(host)
    st.run(out_host)
    torch.cuda.synchronize()
    dsa.check_device()
    want = dsa.window_decode(q, kr2, vr2, bt, pos, nk, nv, window)
    dsa.check_device()
    assert torch.equal(out_host, want.cpu())
    assert torch.equal(kr, kr2) and torch.equal(vr, vr2)
