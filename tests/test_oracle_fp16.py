"""Pins for the oracle's hand-written binary16 conversions.

RN is compared against numpy's float32 -> float16 cast (an independent, correctly
rounded library routine) over every float32 bit pattern whose exponent can land
in or next to the binary16 range, plus samples elsewhere.  RD is checked against
its definition: the largest binary16 value not above x, found by binary search
in the sorted list of all finite binary16 values.
"""
import numpy as np
import pytest

import oracle


def test_f16_to_f32_exhaustive():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


@pytest.mark.parametrize("sign", [0, 1])
def test_f16_rn_exhaustive_near_range(sign):
    # biased fp32 exponents 100..143 cover 2^-27 .. 2^17: every binary16 normal,
    # subnormal, the underflow-to-zero edge and the overflow-to-inf edge.
    chunk = 1 << 23
    for e in range(100, 144):
        bits = (np.uint32(sign << 31) | np.uint32(e << 23)) + np.arange(chunk, dtype=np.uint32)
        x = bits.view(np.float32)
        ours = oracle.f16_rn(x)
        with np.errstate(over="ignore"):
            ref = x.astype(np.float16).view(np.uint16)
        bad = np.nonzero(ours != ref)[0]
        assert bad.size == 0, (e, hex(bits[bad[0]]), hex(ours[bad[0]]), hex(ref[bad[0]]))


def test_f16_rn_samples_and_specials():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[~np.isnan(x)]
    specials = np.array([0.0, -0.0, np.inf, -np.inf, 65504.0, 65519.99, 65520.0, -65520.0,
                         2.0 ** -24, 2.0 ** -25, 1.5 * 2.0 ** -25, 2.0 ** -14, 1e-40, -1e-40], np.float32)
    x = np.concatenate([x, specials])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.f16_rn(x), ref)


def test_f16_rd_definition():
    allh = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = allh.view(np.float16).astype(np.float64)
    finite = np.isfinite(vals)
    sorted_vals = np.unique(vals[finite])                       # -65504 .. 65504, -0 and +0 merged
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(2_000_000).astype(np.float32) * 10.0,
        (rng.standard_normal(500_000) * 1e-5).astype(np.float32),
        (rng.uniform(-65504, 65504, 500_000)).astype(np.float32),
        sorted_vals.astype(np.float32),
        np.nextafter(sorted_vals.astype(np.float32), np.float32(np.inf)),
        np.nextafter(sorted_vals.astype(np.float32), np.float32(-np.inf)),
    ])
    x = x[(x >= -65504) & (x <= 65504)]
    ours = oracle.f16_to_f32(oracle.f16_rd(x)).astype(np.float64)
    idx = np.searchsorted(sorted_vals, x.astype(np.float64), side="right") - 1
    expect = sorted_vals[idx]
    assert np.array_equal(ours, expect)
    # beyond the range: round-down of a large positive value is the largest finite value
    assert oracle.f16_to_f32(oracle.f16_rd(np.array([1e6], np.float32)))[0] == 65504.0
    assert np.isneginf(oracle.f16_to_f32(oracle.f16_rd(np.array([-1e6], np.float32)))[0])
