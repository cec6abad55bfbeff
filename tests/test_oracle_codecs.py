"""Pins for the oracle's block quantizers, packing and dequantization.

BeeLlama v0.4.0 news, section 新增标准 KV cache 类型 (q8_0, q6_0/q6_1, q4_0,
q3_0/q3_1, q2_0/q2_1); the tiny workload's q4_0 definition (d = max|x|/7, codes
round(x/d) clamped to [-8, 7]); KV-COBRA explainer, section Jargon, "Scalar
quantization" (2^b levels, each extra bit cuts the rounding error ~4x).
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import F16, Q8_0, Q6_0, Q5_0, Q4_0, Q3_0, Q2_0, Q8_1, Q6_1, Q5_1, Q4_1, Q3_1, Q2_1, RANK

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "codec_examples.json")))
SYM = [Q8_0, Q6_0, Q5_0, Q4_0, Q3_0, Q2_0]
ASYM = [Q8_1, Q6_1, Q5_1, Q4_1, Q3_1, Q2_1]
BITS = oracle.CODEC_BITS


def _scales_f32(codec, scales):
    s = oracle.f16_to_f32(scales)
    if codec in ASYM:
        return s[:, 0::2], s[:, 1::2]
    return s, None


def test_row_bytes():
    expect = {F16: (256, 0), Q8_0: (128, 8), Q6_0: (96, 8), Q5_0: (80, 8), Q4_0: (64, 8), Q3_0: (48, 8),
              Q2_0: (32, 8), Q8_1: (128, 16), Q6_1: (96, 16), Q5_1: (80, 16), Q4_1: (64, 16), Q3_1: (48, 16),
              Q2_1: (32, 16)}
    for c, v in expect.items():
        assert oracle.row_bytes(c) == v


def test_cobra_worked_example_bit_budget():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cobra_budget.json")))
    total = 0
    for s in g["settings"]:
        cb, sb = oracle.row_bytes(RANK, s["rank"], s["bits"])
        assert cb * 8 == s["bits_per_token"]
    cbA, _ = oracle.row_bytes(RANK, 16, 4)
    cbB, _ = oracle.row_bytes(RANK, 96, 2)
    assert (cbA + cbB) * 8 == g["pair_total_bits"] == 2 * g["head_dim"] * g["bpd"]


def test_q4_0_worked_block():
    ex = GOLD["q4_0_block"]
    x = np.zeros(128, np.float32)
    x[:8] = ex["x_first8"]
    codes, scales = oracle.quantize_rows(Q4_0, x)
    assert hex(scales[0, 0]) == ex["expected_scale_f16_hex"]
    u = oracle.unpack_codes(codes[0], 128, 4).astype(int)
    assert list(u[:8] - 8) == ex["expected_codes_first8"]
    assert (u[8:32] == 8).all()
    ex2 = GOLD["q4_0_clamp"]
    x = np.zeros(128, np.float32)
    x[:2] = ex2["x_first2"]
    codes, _ = oracle.quantize_rows(Q4_0, x)
    u = oracle.unpack_codes(codes[0], 128, 4).astype(int)
    assert list(u[:2] - 8) == ex2["expected_codes_first2"]


@pytest.mark.parametrize("name,bits", [("pack_q4", 4), ("pack_q2", 2), ("pack_q1", 1)])
def test_packing_golden(name, bits):
    ex = GOLD[name]
    u = np.array(ex["u"], np.uint8)
    assert list(oracle.pack_codes(u, bits)) == ex["bytes"]
    assert np.array_equal(oracle.unpack_codes(np.array(ex["bytes"], np.uint8), len(u), bits), u)


def test_packing_golden_planes():
    for name, bits, key in (("pack_q6", 6, "u_first4"), ("pack_q3", 3, "u_first8"), ("pack_q5", 5, "u_first8")):
        ex = GOLD[name]
        u = np.zeros(ex["n"], np.uint8)
        u[: len(ex[key])] = ex[key]
        assert list(oracle.pack_codes(u, bits)) == ex["bytes"]
        assert np.array_equal(oracle.unpack_codes(np.array(ex["bytes"], np.uint8), ex["n"], bits), u)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 8])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    for n in (16, 32, 96, 128):
        u = rng.integers(0, 1 << bits, n).astype(np.uint8)
        assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(u, bits), n, bits), u)


def _random_rows(seed, n=2000):
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((n, 128)) * rng.uniform(0.01, 40.0, (n, 1))
    base[::7] += rng.uniform(-50, 50, (len(base[::7]), 1))            # offset blocks
    base[::11, 3] *= 30                                               # outliers
    return base.astype(np.float32)


@pytest.mark.parametrize("codec", SYM + ASYM)
def test_error_bound(codec):
    y = _random_rows(codec)
    codes, scales = oracle.quantize_rows(codec, y)
    yhat = oracle.dequantize_rows(codec, codes, scales)
    d, _ = _scales_f32(codec, scales)
    dcol = np.repeat(d, 32, axis=1)
    err = np.abs(yhat.astype(np.float64) - y.astype(np.float64))
    bound = dcol.astype(np.float64) * (0.5 + 2.0 ** -10) + np.abs(y) * 2.0 ** -22
    assert (err <= bound).all()


@pytest.mark.parametrize("codec", SYM)
def test_symmetric_grid_roundtrip(codec):
    """x = k d with fp16 d and integer k in [-qmax, qmax], max|k| = qmax -> exact."""
    b = BITS[codec]
    qmax = (1 << (b - 1)) - 1
    rng = np.random.default_rng(100 + codec)
    for _ in range(200):
        d = np.float32(np.float16(rng.uniform(1e-3, 100)))
        k = rng.integers(-qmax, qmax + 1, 128)
        k[rng.integers(0, 32, 4) + 32 * np.arange(4)] = qmax * rng.choice([-1, 1], 4)
        x = (k * d).astype(np.float32)
        codes, scales = oracle.quantize_rows(codec, x)
        assert np.array_equal(oracle.f16_to_f32(scales[0]), np.full(4, d, np.float32))
        assert np.array_equal(oracle.dequantize_rows(codec, codes, scales)[0], x)


@pytest.mark.parametrize("codec", ASYM)
def test_asymmetric_grid_roundtrip(codec):
    """x = m + u d with fp16 m, d, integer u in [0, 2^b-1] hitting both ends -> exact."""
    b = BITS[codec]
    umax = (1 << b) - 1
    rng = np.random.default_rng(200 + codec)
    ok = 0
    for _ in range(300):
        d = np.float32(np.float16(2.0 ** rng.integers(-6, 4)))        # power of two: (max-m)/umax exact
        m = np.float32(np.float16(rng.integers(-64, 64) * d))
        u = rng.integers(0, umax + 1, 128)
        u[::32] = 0
        u[1::32] = umax
        x = (m + u * d).astype(np.float32)
        if not np.array_equal(x.astype(np.float64), m + u * np.float64(d)):
            continue
        codes, scales = oracle.quantize_rows(codec, x)
        assert np.array_equal(oracle.dequantize_rows(codec, codes, scales)[0], x)
        ok += 1
    assert ok > 100


@pytest.mark.parametrize("codec", SYM + ASYM)
def test_zero_block(codec):
    x = np.zeros((1, 128), np.float32)
    x[0, 64:] = np.linspace(-1, 1, 64)
    codes, scales = oracle.quantize_rows(codec, x)
    y = oracle.dequantize_rows(codec, codes, scales)
    assert (y[0, :64] == 0).all()
    d, m = _scales_f32(codec, scales)
    assert d[0, 0] == 0 and d[0, 1] == 0


@pytest.mark.parametrize("codec", SYM + ASYM)
def test_codes_monotone(codec):
    x = np.sort(np.random.default_rng(5).standard_normal(32)).astype(np.float32)
    row = np.tile(x, 4)
    codes, _ = oracle.quantize_rows(codec, row)
    u = oracle.unpack_codes(codes[0], 128, BITS[codec]).astype(int)
    assert (np.diff(u[:32]) >= 0).all()


def test_mse_falls_about_4x_per_bit_symmetric():
    """Each extra bit cuts the rounding error by about 4x (KV-COBRA, Jargon)."""
    y = np.random.default_rng(9).uniform(-1, 1, (4000, 128)).astype(np.float32)
    mse = {}
    for c in SYM:
        codes, scales = oracle.quantize_rows(c, y)
        mse[BITS[c]] = np.mean((oracle.dequantize_rows(c, codes, scales) - y) ** 2)
    assert 3.0 < (mse[4] / mse[6]) ** 0.5 < 6.5          # per-bit factor over a 2-bit step
    assert 3.0 < (mse[6] / mse[8]) ** 0.5 < 6.5
    assert 3.0 < mse[4] / mse[5] < 6.5 and 3.0 < mse[5] / mse[6] < 6.5
    assert mse[2] > mse[3] > mse[4] > mse[5] > mse[6] > mse[8]


@pytest.mark.parametrize("r", [16, 32, 64, 96, 128])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_rank_midrise_bound_and_levels(r, b):
    rng = np.random.default_rng(r * 10 + b)
    z = (rng.standard_normal((500, r)) * rng.uniform(0.01, 20, (500, 1))).astype(np.float32)
    codes, scales = oracle.quantize_rows(RANK, z, r=r, b=b)
    zh = oracle.dequantize_rows(RANK, codes, scales, r=r, b=b)
    blk = min(32, r)
    d = np.repeat(oracle.f16_to_f32(scales), blk, axis=1).astype(np.float64)
    err = np.abs(zh.astype(np.float64) - z)
    assert (err <= d * (0.5 + 2.0 ** -9) + 1e-30).all()
    # every reconstructed value is an odd multiple of d/2 within +-(2^b - 1) d/2
    lev = zh.astype(np.float64) / (0.5 * d)
    assert np.allclose(lev, np.round(lev)) and (np.abs(np.round(lev)) % 2 == 1).all()
    assert np.abs(lev).max() <= (1 << b) - 1 + 1e-9


def test_rank_mse_about_4x_per_bit():
    z = np.random.default_rng(12).uniform(-1, 1, (4000, 128)).astype(np.float32)
    mse = []
    for b in (1, 2, 3, 4):
        codes, scales = oracle.quantize_rows(RANK, z, r=128, b=b)
        mse.append(np.mean((oracle.dequantize_rows(RANK, codes, scales, r=128, b=b) - z) ** 2))
    for b in (1, 2):                               # b -> b+1 for b >= 2 (and 3 -> 4)
        ratio = mse[b] / mse[b + 1]
        assert 3.5 < ratio < 6.0, (b, ratio)


def test_rank_one_bit_is_sign_times_amax():
    z = np.random.default_rng(13).standard_normal((10, 32)).astype(np.float32)
    codes, scales = oracle.quantize_rows(RANK, z, r=32, b=1)
    zh = oracle.dequantize_rows(RANK, codes, scales, r=32, b=1)
    amax = np.float32(np.float16(np.abs(z).max(axis=1) / 0.5)) * 0.5
    assert np.array_equal(zh, np.where(z >= 0, 1.0, -1.0) * amax[:, None])


def test_f16_codec_is_identity_on_fp16_values():
    x = np.random.default_rng(14).standard_normal((50, 128)).astype(np.float16).astype(np.float32)
    codes, scales = oracle.quantize_rows(F16, x)
    assert np.array_equal(codes.view(np.uint16), x.astype(np.float16).view(np.uint16))
    assert np.array_equal(oracle.dequantize_rows(F16, codes, scales), x)


@pytest.mark.parametrize("codec", ASYM)
def test_asymmetric_scale_is_order_independent_with_signed_zeros(codec):
    """R5: the block minimum and maximum follow IEEE-754 minimum/maximum (-0 < +0),
    so permuting a block never changes the stored scale or minimum bits: a block
    whose smallest value is zero stores m = -0 (0x8000) exactly when it holds a -0."""
    rng = np.random.default_rng(300 + codec)
    for trial in range(60):
        x = np.zeros(32, np.float32)
        x[rng.integers(0, 32, 5)] = rng.uniform(0.5, 3, 5).astype(np.float32)
        has_neg_zero = trial % 2 == 0
        if has_neg_zero:
            x[rng.integers(0, 32, 3)] = np.float32(-0.0)
        row = np.tile(x, 4)
        ref = oracle.quantize_rows(codec, row)[1]
        expect_m = 0x8000 if (np.signbit(x) & (x == 0)).any() else 0x0000
        assert ref[0, 1] == expect_m
        for _ in range(4):
            perm = np.concatenate([rng.permutation(32) + 32 * b for b in range(4)])
            assert np.array_equal(oracle.quantize_rows(codec, row[perm])[1], ref)
