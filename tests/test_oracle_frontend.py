"""Pins for the oracle's indexer front end ([P2] Step-5-Preview 如何实现1M长上下文
§索引器打分: the indexer projects the hidden state to index_q / index_k / index_z, then
normalises and applies RoPE to part of the dimensions).

Fixed reading (the pages give no constants): index_q (16 x 256) and index_k (4 x 256) are
RMSNorm-ed per 256-d head (eps 1e-6, learned weight per side), the first 64 dimensions are
rotated in rotate-half pairs (i, i + 32) by pos * 10000^(-2i/64), and the gates are
z = sigmoid(W_z h).

Pins: the projection and norm at position 0 against numpy's float64 matmul (a library routine
the oracle does not use); the rotation angle itself on hand-built one-hot head vectors (the
pair (i, i + 32) must come out as the plane rotation by pos * 10000^(-2i/64), evaluated here
with numpy's cos/sin, for i = 0, 1, 31 at positions 1, 1000 and 2^20 - 1, so a wrong frequency
table, base or pair map fails); the unrotated dimensions identical at every position; every rotated
pair keeping its norm; the score-relevant dot product over the rotated dimensions depending on
the positions only through their difference; RMSNorm's invariance to scaling the hidden state;
zero gate weights giving z = 1/2 and negated ones 1 - z.
"""
import numpy as np
import pytest

import oracle

from _util import bf16_from_bits_np

HI, G, DI = 16, 4, 256
ROWS = HI * DI + G * DI + HI


def to_bits(x):
    """float -> bf16 bits, round to nearest even (test inputs only)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def inputs(T, hid, seed, gamma_one=False):
    rng = np.random.default_rng(seed)
    h = to_bits(rng.standard_normal((T, hid)))
    w = to_bits(rng.standard_normal((ROWS, hid)) / np.sqrt(hid))
    gq = to_bits(np.ones(DI) if gamma_one else 1.0 + 0.1 * rng.standard_normal(DI))
    gk = to_bits(np.ones(DI) if gamma_one else 1.0 + 0.1 * rng.standard_normal(DI))
    return h, w, gq, gk


def f64(bits):
    return bf16_from_bits_np(bits).astype(np.float64)


def test_position_zero_equals_numpy_projection_and_rmsnorm():
    T, hid = 5, 96
    h, w, gq, gk = inputs(T, hid, 1)
    iq, ik, z = oracle.indexer_frontend(h, w, gq, gk, np.zeros(T, np.int32))
    a = f64(w) @ f64(h).T                                   # [ROWS][T] float64 (numpy)
    for t in range(T):
        heads = a[: (HI + G) * DI, t].reshape(HI + G, DI)
        y = heads / np.sqrt((heads ** 2).mean(axis=1, keepdims=True) + 1e-6)
        y[:HI] *= f64(gq)
        y[HI:] *= f64(gk)
        got = np.concatenate([f64(iq[t]), f64(ik[t])])
        np.testing.assert_allclose(got, y, rtol=2 ** -8, atol=1e-30)
        np.testing.assert_allclose(z[t], 1.0 / (1.0 + np.exp(-a[(HI + G) * DI:, t])), rtol=1e-6)


def test_unrotated_dimensions_do_not_depend_on_position():
    T, hid = 3, 64
    h, w, gq, gk = inputs(T, hid, 2)
    base = oracle.indexer_frontend(h, w, gq, gk, np.zeros(T, np.int32))
    for p in (1, 777, 1_048_575):
        other = oracle.indexer_frontend(h, w, gq, gk, np.full(T, p, np.int32))
        assert np.array_equal(base[0][..., 64:], other[0][..., 64:])
        assert np.array_equal(base[1][..., 64:], other[1][..., 64:])
        assert not np.array_equal(base[0][..., :64], other[0][..., :64])
        assert np.array_equal(base[2], other[2])                 # gates: no rotation


def test_rotation_keeps_every_pair_norm():
    T, hid = 2, 64
    h, w, gq, gk = inputs(T, hid, 3)
    a = oracle.indexer_frontend(h, w, gq, gk, np.zeros(T, np.int32))
    b = oracle.indexer_frontend(h, w, gq, gk, np.full(T, 12345, np.int32))
    for x, y in ((a[0], b[0]), (a[1], b[1])):
        nx = f64(x[..., :32]) ** 2 + f64(x[..., 32:64]) ** 2
        ny = f64(y[..., :32]) ** 2 + f64(y[..., 32:64]) ** 2
        np.testing.assert_allclose(ny, nx, rtol=2 ** -6, atol=1e-3)


def test_rotated_dot_product_depends_on_position_difference():
    # q of token 0 at p1 against k of token 1 at p2: only p1 - p2 matters
    T, hid = 2, 64
    h, w, gq, gk = inputs(T, hid, 4)
    dots = []
    for p1, p2 in ((7, 3), (1007, 1003), (500_004, 500_000)):
        iq, ik, _ = oracle.indexer_frontend(h, w, gq, gk, np.array([p1, p2], np.int32))
        dots.append(np.einsum("hd,gd->hg", f64(iq[0, :, :64]), f64(ik[1, :, :64])))
    scale = np.abs(dots[0]).max()          # outputs are bf16: compare on the products' scale
    for d in dots[1:]:
        assert np.abs(d - dots[0]).max() <= 0.01 * scale
    # and a different difference gives a different product
    iq, ik, _ = oracle.indexer_frontend(h, w, gq, gk, np.array([9, 3], np.int32))
    d6 = np.einsum("hd,gd->hg", f64(iq[0, :, :64]), f64(ik[1, :, :64]))
    assert np.abs(d6 - dots[0]).max() > 0.1 * scale


def test_rmsnorm_ignores_the_scale_of_the_hidden_state():
    T, hid = 3, 80
    h, w, gq, gk = inputs(T, hid, 5, gamma_one=True)
    h2 = to_bits(2.0 * f64(h))                                  # exact doubling in bf16
    a = oracle.indexer_frontend(h, w, gq, gk, np.arange(T, dtype=np.int32))
    b = oracle.indexer_frontend(h2, w, gq, gk, np.arange(T, dtype=np.int32))
    # equal but for eps (1e-6 against a mean square 4x larger): within one bf16 step
    for x, y in ((a[0], b[0]), (a[1], b[1])):
        np.testing.assert_allclose(f64(y), f64(x), rtol=2 ** -7, atol=1e-6)
    # with gamma = 1 every head vector has mean square 1 (eps aside), at any position
    ms = (f64(a[0]) ** 2).mean(axis=-1)
    np.testing.assert_allclose(ms, 1.0, rtol=2e-2)


def test_gates_are_sigmoids():
    T, hid = 4, 32
    h, w, gq, gk = inputs(T, hid, 6)
    w0 = w.copy()
    w0[(HI + G) * DI:] = 0
    _, _, z0 = oracle.indexer_frontend(h, w0, gq, gk, np.zeros(T, np.int32))
    assert np.all(z0 == 0.5)
    _, _, z = oracle.indexer_frontend(h, w, gq, gk, np.zeros(T, np.int32))
    wn = w.copy()
    wn[(HI + G) * DI:] ^= np.uint16(0x8000)                     # negate the gate rows
    _, _, zn = oracle.indexer_frontend(h, wn, gq, gk, np.zeros(T, np.int32))
    np.testing.assert_allclose(zn, 1.0 - z, rtol=1e-6, atol=1e-7)


def one_hot_case(dim, val=16.0, hid=8):
    """Hidden state e_0 and weights whose only non-zero entry puts `val` at `dim` of every
    q head and k group: each pre-norm head vector is val * e_dim (mean square val^2 / 256,
    so with val = 16 the RMSNorm leaves it at 16 up to eps, and gamma = 1)."""
    h = np.zeros((1, hid), np.uint16)
    h[0, 0] = to_bits(1.0)
    w = np.zeros((ROWS, hid), np.uint16)
    for v in range(HI + G):
        w[v * DI + dim, 0] = to_bits(val)
    ones = to_bits(np.ones(DI))
    return h, w, ones, ones


@pytest.mark.parametrize("i", [0, 1, 31])
@pytest.mark.parametrize("p", [1, 1000, (1 << 20) - 1])
def test_rotation_angle_by_hand(i, p):
    # RoPE on the first 64 dims in rotate-half pairs (i, i + 32), angle p * 10000^(-2i/64)
    # ([P2] §索引器打分 names RoPE on part of the dims; the frequency table is the reading).
    th = p * 10000.0 ** (-2.0 * i / 64.0)
    c, s = np.cos(th), np.sin(th)
    mag = 16.0 / np.sqrt(1.0 + 1e-6)                           # the RMSNorm's eps, exactly
    for dim, exp_i, exp_j in ((i, mag * c, mag * s), (i + 32, -mag * s, mag * c)):
        h, w, gq, gk = one_hot_case(dim)
        iq, ik, _ = oracle.indexer_frontend(h, w, gq, gk, np.array([p], np.int32))
        for out in (f64(iq[0]), f64(ik[0])):                    # every q head and k group
            want = np.zeros(DI)
            want[i], want[i + 32] = exp_i, exp_j
            # one bf16 rounding of each output (8 significant bits): half an ulp, <= 2^-8 relative
            tol = np.abs(want) * 2.0 ** -8 + 1e-30
            assert np.all(np.abs(out - want[None, :]) <= tol[None, :]), (dim, p, out[0, [i, i + 32]], want[[i, i + 32]])
