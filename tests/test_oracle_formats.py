"""Pins for the oracle's number formats: OCP E4M3 and bf16 codecs.

The summaries are stored as FP8 ([P2] Step-5-Preview 如何实现1M长上下文, §区域压缩CSA;
[P1] kwkr.cn/news/601179 §DSA ②), the e4m3 variant with absmax/448 scaling.  The codec
is pinned against two independent library implementations (ml_dtypes and torch) and
against properties that fix round-to-nearest-even exhaustively.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

pytestmark = []


def all_finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_decode_matches_libraries():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    th = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    fin = np.array([(c & 0x7F) != 0x7F for c in range(256)])
    assert np.array_equal(ours[fin], ml[fin])
    assert np.array_equal(ours[fin], th[fin])
    assert np.all(np.isnan(ours[~fin]))


def test_hand_values():
    # largest finite, smallest subnormal, smallest normal, one, saturation
    assert oracle.f32_to_e4m3([448.0])[0] == 0x7E
    assert oracle.f32_to_e4m3([-448.0])[0] == 0xFE
    assert oracle.f32_to_e4m3([2.0 ** -9])[0] == 0x01
    assert oracle.f32_to_e4m3([2.0 ** -6])[0] == 0x08
    assert oracle.f32_to_e4m3([1.0])[0] == 0x38
    assert oracle.f32_to_e4m3([464.0])[0] == 0x7E
    assert oracle.f32_to_e4m3([1e30])[0] == 0x7E
    assert oracle.f32_to_e4m3([-1e30])[0] == 0xFE
    assert oracle.f32_to_e4m3([0.0])[0] == 0x00
    assert oracle.f32_to_e4m3([-0.0])[0] == 0x80
    assert oracle.e4m3_to_f64([0x7E])[0] == 448.0


def test_round_trip_every_code():
    codes = np.array(all_finite_codes(), dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes).astype(np.float32)
    back = oracle.f32_to_e4m3(vals)
    assert np.array_equal(back, codes)


def test_midpoints_round_to_even_and_neighbours_to_nearest():
    pos = sorted(set(oracle.e4m3_to_f64(np.arange(0, 0x7F, dtype=np.uint8)).tolist()))
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = np.float32((lo + hi) / 2)          # exact: both have <= 4 significant bits
        assert float(mid) == (lo + hi) / 2
        clo, chi = oracle.f32_to_e4m3([lo, hi])
        even = clo if clo % 2 == 0 else chi
        assert oracle.f32_to_e4m3([mid])[0] == even, (lo, hi)
        below = np.nextafter(mid, np.float32(-np.inf))
        above = np.nextafter(mid, np.float32(np.inf))
        assert oracle.f32_to_e4m3([below])[0] == clo
        assert oracle.f32_to_e4m3([above])[0] == chi
        # the negative side mirrors the positive side
        assert oracle.f32_to_e4m3([-mid])[0] == (even | 0x80)


def test_random_values_match_libraries():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 100,
        rng.uniform(-448, 448, 4000).astype(np.float32),
        (rng.standard_normal(2000) * 2.0 ** -8).astype(np.float32),
    ])
    ours = oracle.f32_to_e4m3(x)
    ml = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    th = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ml)
    assert np.array_equal(ours, th)


def test_saturation_above_max():
    x = np.array([448.0, 448.5, 460.0, 463.99, 464.0, 500.0, 1e6, 3.4e38], np.float32)
    assert np.all(oracle.f32_to_e4m3(x) == 0x7E)
    assert np.all(oracle.f32_to_e4m3(-x) == 0xFE)


def test_bf16_round_trip_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = ((pats >> 7) & 0xFF) != 0xFF
    vals = oracle.bf16_to_f64(pats)
    with np.errstate(invalid="ignore"):
        ref = (pats.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(vals[finite], ref[finite])
    sel = pats[finite][::97]
    back = oracle.f64_to_bf16(oracle.bf16_to_f64(sel))
    # -0.0 and +0.0 keep their signs
    assert np.array_equal(back, sel)


def test_bf16_rounding_matches_torch_from_fp32():
    # an fp32 input reaches the oracle exactly (fp32 -> f64 is exact), so one rounding
    # to bf16 must agree with torch's fp32 -> bf16 conversion (RNE)
    rng = np.random.default_rng(3)
    with np.errstate(over="ignore"):
        x = np.concatenate([rng.standard_normal(5000).astype(np.float32),
                            (rng.standard_normal(500) * 1e-39).astype(np.float32),
                            rng.standard_normal(500).astype(np.float32) * np.float32(3e38)])
    ours = oracle.f64_to_bf16(x.astype(np.float64))
    th = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, th)


def test_bf16_rounds_once_from_double():
    # 1 + 2^-8 + 2^-30 is just above the bf16 midpoint between 1 and 1 + 2^-7: a double
    # rounded via fp32 would land on the midpoint and tie to 1.0; one rounding gives 1+2^-7
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle.bf16_to_f64(oracle.f64_to_bf16([x]))[0] == 1.0 + 2.0 ** -7
    # exact midpoint ties to even (1.0)
    assert oracle.bf16_to_f64(oracle.f64_to_bf16([1.0 + 2.0 ** -8]))[0] == 1.0
