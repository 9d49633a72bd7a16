"""Pins for the oracle's region compression (step A1).

[P1] kwkr.cn/news/601179 §DSA ②: every complete 8-token region becomes one 256-d FP8
summary; [P2] Step-5-Preview 如何实现1M长上下文 §区域压缩CSA: only regions that hold 8
tokens are summarised.  The fixed reading: summary = e4m3(mean / scale), one fp32
scale = absmax/448 per (region, group).

Every test here checks the oracle against something it does not compute itself:
closed forms, exact invariances of the definition, the e4m3 error bound, and an
independent library evaluation (numpy + ml_dtypes).
"""
import ml_dtypes
import numpy as np
import pytest

import oracle

from _util import f64

G, DI = 4, 256


def bf16_bits(x):
    """float array exactly representable in bf16 -> bit patterns (truncation is exact)."""
    x = np.asarray(x, np.float32)
    u = x.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def rand_bf16(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)   # truncate to a bf16 value


def compress(tokens_bits, n_regions=None):
    """tokens [T][4][256] -> summaries [r][g][256] / scales [r][g] of regions 0..T/8-1
    (the oracle's group-major pool, transposed to region-major for indexing here)."""
    T = tokens_bits.shape[0]
    n = T // 8 if n_regions is None else n_regions
    S, C = oracle.compress_regions(tokens_bits, [8 * r for r in range(n)], list(range(n)), n)
    return S.transpose(1, 0, 2), C.T


def test_rows_of_region_r_are_8r_to_8r_plus_7():
    # token t carries the value t in every coordinate: region r's mean is 8r + 3.5
    T = 64
    vals = np.repeat(np.arange(T, dtype=np.float32)[:, None, None], G * DI, axis=1).reshape(T, G, DI)
    S, C = compress(bf16_bits(vals))
    for r in range(T // 8):
        mean = 8 * r + 3.5
        for g in range(G):
            assert C[r, g] == np.float32(np.float32(mean) / np.float32(448.0))
            assert np.all(S[r, g] == 0x7E)    # every coordinate is the absmax -> 448


def test_identical_tokens_mean_is_the_token():
    rng = np.random.default_rng(1)
    tok = rand_bf16(rng, (1, G, DI))
    S, C = compress(np.repeat(tok, 8, axis=0))
    m = f64(tok[0]).astype(np.float32)
    for g in range(G):
        scale = np.float32(np.abs(m[g]).max() / np.float32(448.0))
        assert C[0, g] == scale
        amax = int(np.argmax(np.abs(m[g])))
        assert S[0, g, amax] in (0x7E, 0xFE)
        deq = oracle.e4m3_to_f64(S[0, g]) * float(scale)
        # e4m3 error bound: half a step of 2^(E-3) around each value, 2^-10 for subnormals
        q = m[g].astype(np.float64) / float(scale)
        step = np.where(np.abs(q) >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(q), 1e-300))) - 3),
                        2.0 ** -9)
        assert np.all(np.abs(deq / float(scale) - q) <= step / 2 + 1e-6 * np.abs(q))


def test_zero_region_has_zero_scale_and_codes():
    S, C = compress(np.zeros((16, G, DI), np.uint16))
    assert np.all(C == 0) and np.all(S == 0)


def test_power_of_two_homogeneity_and_negation():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((8, G, DI))).astype(np.float32)
    x = (x.view(np.uint32) & 0xFFFF0000).view(np.float32)
    S0, C0 = compress(bf16_bits(x))
    S1, C1 = compress(bf16_bits(x * np.float32(2.0 ** 5)))
    S2, C2 = compress(bf16_bits(-x))
    assert np.array_equal(S0, S1) and np.array_equal(C1, C0 * np.float32(32.0))
    assert np.array_equal(S2, S0 ^ np.uint8(0x80) * (S0 != 0))
    assert np.array_equal(C2, C0)


def test_token_order_inside_a_region_does_not_matter():
    rng = np.random.default_rng(3)
    x = rand_bf16(rng, (8, G, DI))
    S0, C0 = compress(x)
    S1, C1 = compress(x[rng.permutation(8)])
    assert np.array_equal(S0, S1) and np.array_equal(C0, C1)


def test_groups_are_independent():
    rng = np.random.default_rng(4)
    x = rand_bf16(rng, (8, G, DI))
    S0, C0 = compress(x)
    y = x.copy()
    y[:, 2] = rand_bf16(rng, (8, DI))
    S1, C1 = compress(y)
    for g in (0, 1, 3):
        assert np.array_equal(S0[0, g], S1[0, g]) and C0[0, g] == C1[0, g]


def test_matches_library_evaluation():
    # numpy float64 mean -> fp32, numpy fp32 division, ml_dtypes RNE cast to e4m3
    rng = np.random.default_rng(5)
    T = 8 * 40
    x = rand_bf16(rng, (T, G, DI))
    S, C = compress(x)
    v = f64(x).reshape(T // 8, 8, G, DI)
    m = v.mean(axis=1).astype(np.float32)
    scale = (np.abs(m).max(axis=2) / np.float32(448.0)).astype(np.float32)
    q = (m / scale[..., None]).astype(np.float32)
    ref = q.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(C, scale)
    assert np.array_equal(S, ref)


def test_strided_rows_and_scattered_slots():
    # rows taken with a row stride larger than 4*256 and written to arbitrary slots
    rng = np.random.default_rng(6)
    x = rand_bf16(rng, (40, G, DI))
    wide = np.zeros((40, G * DI + 128), np.uint16)
    wide[:, : G * DI] = x.reshape(40, G * DI)
    Sa, Ca = oracle.compress_regions(wide, [0, 8, 24], [5, 0, 2], 7)
    Sb, Cb = oracle.compress_regions(x, [0, 8, 24], [5, 0, 2], 7)
    assert np.array_equal(Sa, Sb) and np.array_equal(Ca, Cb)
    Sa, Ca = Sa.transpose(1, 0, 2), Ca.T
    Sr, Cr = compress(x)
    assert np.array_equal(Sa[5], Sr[0]) and np.array_equal(Sa[0], Sr[1]) and np.array_equal(Sa[2], Sr[3])
    for s in (1, 3, 4, 6):
        assert np.all(Sa[s] == 0) and np.all(Ca[s] == 0)


def test_region_geometry_against_the_pages():
    # 1M tokens make 131,072 regions ([P3] 100 万 token 上下文实测 §一); 512 regions
    # of 8 tokens make 4,096 tokens ([P2] FAQ)
    assert (1 << 20) // 8 == 131072 and 512 * 8 == 4096
