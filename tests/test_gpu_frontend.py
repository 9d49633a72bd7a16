"""GPU indexer front end (dsa_indexer_frontend: tcgen05 bf16 GEMM with RMSNorm, partial RoPE
and sigmoid gates in its epilogue) against the oracle's front end.

[P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: index_q / index_k / index_z projected from
the hidden state, normalised, RoPE on part of the dimensions.  Bar: index_q and index_k are
bf16 outputs of fp32 arithmetic against the oracle's double rounded once to bf16, so they may
differ by one bf16 step (2^-8 relative) where the double lands near a rounding boundary:
within 2^-7 relative + 2e-3 absolute; gates within 1e-5.  Cases: one token, ragged token
tiles (130, 300), hidden sizes that are and are not multiples of the 64-element k-step, large
positions (up to 2^20), and the benchmark's shape (2,048 tokens, hidden 6,144) on sampled
tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_dsa_b200 import dsa

from _util import bits, bf16_from_bits_np

pytestmark = pytest.mark.gpu
ROWS = 16 * 256 + 4 * 256 + 16


def make(T, hid, seed, max_pos=1 << 20):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    hidden = torch.randn((T, hid), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((ROWS, hid), generator=g, device="cuda") / hid ** 0.5).to(torch.bfloat16)
    gq = (1.0 + 0.1 * torch.randn(256, generator=g, device="cuda")).to(torch.bfloat16)
    gk = (1.0 + 0.1 * torch.randn(256, generator=g, device="cuda")).to(torch.bfloat16)
    pos = torch.randint(0, max_pos, (T,), generator=g, device="cuda", dtype=torch.int32)
    return hidden, w, gq, gk, pos


def compare(got_q, got_k, got_z, ref, rows):
    rq, rk, rz = ref
    for got, want in ((got_q, rq), (got_k, rk)):
        g = got[rows].float().cpu().numpy()
        o = bf16_from_bits_np(want)
        err = np.abs(g - o)
        assert np.all(err <= 2 ** -7 * np.abs(o) + 2e-3), err.max()
    np.testing.assert_allclose(got_z[rows].cpu().numpy(), rz, atol=1e-5, rtol=0)


@pytest.mark.parametrize("T,hid", [(1, 64), (130, 200), (300, 512), (129, 1000)])
def test_matches_oracle(T, hid):
    hidden, w, gq, gk, pos = make(T, hid, seed=T + hid)
    iq, ik, z = dsa.indexer_frontend(hidden, w, gq, gk, pos)
    dsa.check_device()
    ref = oracle.indexer_frontend(bits(hidden), bits(w), bits(gq), bits(gk), pos.cpu().numpy())
    compare(iq, ik, z, ref, np.arange(T))


def test_benchmark_shape_on_sampled_tokens():
    T, hid = 2048, 6144
    hidden, w, gq, gk, pos = make(T, hid, seed=77)
    iq, ik, z = dsa.indexer_frontend(hidden, w, gq, gk, pos)
    dsa.check_device()
    rows = np.array([0, 1, 127, 128, 1000, 2047])
    ref = oracle.indexer_frontend(bits(hidden[rows]), bits(w), bits(gq), bits(gk), pos.cpu().numpy()[rows])
    compare(iq, ik, z, ref, rows)


def test_position_zero_leaves_dims_unrotated_and_norm_is_scale_free():
    T, hid = 64, 256
    hidden, w, gq, gk, _ = make(T, hid, seed=5)
    zero = torch.zeros(T, dtype=torch.int32, device="cuda")
    a = dsa.indexer_frontend(hidden, w, gq, gk, zero)
    b = dsa.indexer_frontend((hidden.float() * 4).to(torch.bfloat16), w, gq, gk, zero)
    dsa.check_device()
    # x4 is exact in bf16; RMSNorm removes it up to eps: one bf16 step at most
    for x, y in ((a[0], b[0]), (a[1], b[1])):
        assert torch.all((x.float() - y.float()).abs() <= 2 ** -7 * x.float().abs() + 1e-3)
