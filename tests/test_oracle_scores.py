"""Pins for the oracle's indexer score (step A2).

[P1] kwkr.cn/news/601179 §DSA ③ and [P2] Step-5-Preview 如何实现1M长上下文 §索引器打分:
a 16-head indexer scores the query against every region summary of its request; the
regions and the indexer heads map onto the 4 KV groups (num_provider_groups: 4).
Fixed reading: score(r,g) = sum_{h=4g}^{4g+3} z_h * ReLU(q_h . s_{r,g}) / 16.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle

from _util import f64

G, DI, HI = 4, 256, 16


def bits_of(x):
    x = np.asarray(x, np.float32)
    u = x.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


def rand_bf16(rng, shape):
    x = rng.standard_normal(shape).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def one_hot_pool(n_slots, j=0, c=448.0 * 2 ** -6):
    """Group-major pool whose every summary is c * e_j exactly: code 0x7E at j, scale c/448."""
    S = np.zeros((G, n_slots, DI), np.uint8)
    S[:, :, j] = 0x7E
    C = np.full((G, n_slots), np.float32(c / 448.0), np.float32)
    return S, C


def random_pool(rng, n_slots, lo=0, hi=0x7E):
    S = rng.integers(lo, hi, (G, n_slots, DI), dtype=np.uint8)
    C = rng.uniform(0.001, 0.01, (G, n_slots)).astype(np.float32)
    return S, C


def test_closed_form_one_hot_summary():
    S, C = one_hot_pool(4, j=3)
    c = 448.0 * 2 ** -6                      # exactly 448 * scale
    q = np.zeros((1, HI, DI), np.float32)
    a = np.array([1.5, -2.0, 0.25, 3.0] * 4, np.float32)
    q[0, :, 3] = a
    q[0, :, 100] = 7.0                       # where the summary is zero: no contribution
    z = np.linspace(0.1, 0.9, HI).astype(np.float32)
    sc = oracle.indexer_scores(bits_of(q), z[None], [0], [4 * 8 + 2], S, C, [0])
    for g in range(G):
        h = np.arange(4 * g, 4 * g + 4)
        expect = np.float32(np.sum(z[h].astype(np.float64) * np.maximum(a[h] * c, 0.0)) / 16.0)
        assert np.all(sc[0, g, :4] == expect)


def test_negative_dot_products_score_zero():
    S, C = one_hot_pool(3)
    q = np.zeros((1, HI, DI), np.float32)
    q[0, :, 0] = -1.0
    sc = oracle.indexer_scores(bits_of(q), np.ones((1, HI), np.float32), [0], [3 * 8], S, C, [0])
    assert np.all(sc[0, :, :3] == 0.0) and not np.any(np.signbit(sc[0, :, :3]))


def test_head_to_group_map():
    # only head h has a non-zero gate: only group h // 4 scores anything
    S, C = one_hot_pool(2)
    q = np.zeros((1, HI, DI), np.float32)
    q[0, :, 0] = 1.0
    for h in range(HI):
        z = np.zeros((1, HI), np.float32)
        z[0, h] = 1.0
        sc = oracle.indexer_scores(bits_of(q), z, [0], [16], S, C, [0])
        nz = [g for g in range(G) if np.any(sc[0, g, :2] != 0)]
        assert nz == [h // 4]


def test_only_regions_before_the_own_region_are_scored():
    rng = np.random.default_rng(0)
    n = 10
    S, C = random_pool(rng, n)
    q = rand_bf16(rng, (3, HI, DI))
    z = rng.uniform(0, 1, (3, HI)).astype(np.float32)
    pos = [0, 23, 79]                          # own regions 0, 2, 9
    sc = oracle.indexer_scores(q, z, [0, 0, 0], pos, S, C, [0], ld=n)
    for i, p in enumerate(pos):
        own = p // 8
        assert np.all(np.isfinite(sc[i, :, :own]))
        assert np.all(np.isnan(sc[i, :, own:]))


def test_request_base_selects_the_request_slots():
    rng = np.random.default_rng(1)
    S, C = random_pool(rng, 12)
    q = rand_bf16(rng, (1, HI, DI))
    z = rng.uniform(0, 1, (1, HI)).astype(np.float32)
    a = oracle.indexer_scores(q, z, [1], [40], S, C, [0, 7])      # request 1: slots 7..11
    b = oracle.indexer_scores(q, z, [0], [40], S[:, 7:], C[:, 7:], [0])
    assert np.array_equal(a, b)


def test_exact_scalings():
    # doubling every gate, or every query, doubles every score exactly (powers of two)
    rng = np.random.default_rng(2)
    S, C = random_pool(rng, 6)
    q = rand_bf16(rng, (1, HI, DI))
    z = rng.uniform(0, 1, (1, HI)).astype(np.float32)
    s0 = oracle.indexer_scores(q, z, [0], [48], S, C, [0])
    s1 = oracle.indexer_scores(q, z * 2, [0], [48], S, C, [0])
    q2 = bits_of(f64(q).astype(np.float32) * 2)
    s2 = oracle.indexer_scores(q2, z, [0], [48], S, C, [0])
    assert np.array_equal(s1, 2 * s0) and np.array_equal(s2, 2 * s0)


def test_brute_force_from_library_decode():
    # decoded with ml_dtypes, evaluated with numpy float64 einsum
    rng = np.random.default_rng(3)
    n, nq = 33, 4
    S, C = random_pool(rng, n, 0, 256)
    S[(S & 0x7F) == 0x7F] = 0x11               # no NaN codes
    q = rand_bf16(rng, (nq, HI, DI))
    z = rng.uniform(0, 1, (nq, HI)).astype(np.float32)
    pos = [8 * n + 1, 70, 8, 200]
    sc = oracle.indexer_scores(q, z, [0] * nq, pos, S, C, [0], ld=n)
    s = S.view(ml_dtypes.float8_e4m3fn).astype(np.float64) * C[..., None].astype(np.float64)  # [g][r][d]
    qd = f64(q)
    for i in range(nq):
        own = pos[i] // 8
        dots = np.einsum("hd,grd->rgh", qd[i], s)               # [r][g][h]
        for g in range(G):
            h = np.arange(4 * g, 4 * g + 4)
            ref = (np.maximum(dots[:own, g, h], 0) * z[i, h]).sum(axis=1) / 16
            np.testing.assert_allclose(sc[i, g, :own], ref, rtol=1e-6, atol=0)


def test_fp8_query_mode_is_exact_for_representable_queries():
    # a query head whose values are e4m3 values times a power of two with absmax
    # exactly 448 * 2^-5 quantises without error: both modes give the same scores
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 0x7E, (1, HI, DI), dtype=np.uint8)
    codes[..., 0] = 0x7E                      # absmax code 448 in every head
    vals = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32) * np.float32(2.0 ** -5)
    q = bits_of(vals)
    S, C = random_pool(rng, 5)
    z = rng.uniform(0, 1, (1, HI)).astype(np.float32)
    a = oracle.indexer_scores(q, z, [0], [40], S, C, [0], flags=0)
    b = oracle.indexer_scores(q, z, [0], [40], S, C, [0], flags=oracle.Q_FP8)
    np.testing.assert_allclose(b, a, rtol=1e-6)


def test_fp8_query_mode_error_bound():
    # e4m3 keeps 4 significant bits: each quantised query value is within 2^-4 of it
    # (relative) or within half a subnormal step; scores move accordingly
    rng = np.random.default_rng(5)
    S, C = one_hot_pool(2, j=0, c=1.0 * 448 * 2 ** -8)
    q = rand_bf16(rng, (1, HI, DI))
    z = np.ones((1, HI), np.float32)
    a = oracle.indexer_scores(q, z, [0], [16], S, C, [0])
    b = oracle.indexer_scores(q, z, [0], [16], S, C, [0], flags=oracle.Q_FP8)
    np.testing.assert_allclose(b, a, rtol=2 ** -4, atol=1e-3)
