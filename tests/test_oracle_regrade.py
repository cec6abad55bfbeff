"""Oracle VBR regrade ("Introducing a new KV format: VBR (Variable Bit Rate)",
first post: the cache is requantized layer by layer as the session grows).

Pins: a symmetric (_0) row regraded to its own codec is unchanged (the quantizer
reproduces its own grid points exactly: the largest magnitude sits on +-qmax);
regrading a row moves each value by at most half a step of the new codec from the
old reconstruction (this also covers the _1 codecs regraded to themselves, whose
minimum code need not be 0, so their scale can move); an F16 row regraded to a
codec is exactly what appending it with that codec stores."""
import numpy as np
import pytest

import oracle
from oracle import F16, Q8_0, Q6_0, Q5_0, Q4_0, Q3_0, Q2_0, Q8_1, Q6_1, Q5_1, Q4_1, Q3_1, Q2_1, ROT_HADAMARD



def _rows(seed, n=400):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((n, 128)) * rng.uniform(0.01, 20, (n, 1))
    y[::7] += rng.uniform(-5, 5, (len(y[::7]), 1))
    return y.astype(np.float32)


@pytest.mark.parametrize("codec", [Q8_0, Q6_0, Q5_0, Q4_0, Q3_0, Q2_0])
def test_regrade_to_the_same_codec_is_the_identity(codec):
    c, s = oracle.quantize_rows(codec, _rows(codec))
    c2, s2 = oracle.regrade_rows(codec, codec, ROT_HADAMARD, c, s)
    assert np.array_equal(c2, c)
    assert np.array_equal(s2, s)


@pytest.mark.parametrize("old,new", [(Q8_0, Q4_0), (Q8_0, Q6_0), (Q6_0, Q4_1), (Q4_1, Q2_1), (Q8_0, Q2_0),
                                     (Q5_1, Q3_1), (Q4_0, Q3_0), (Q8_1, Q8_1), (Q4_1, Q4_1), (Q2_1, Q2_1)])
def test_regrade_moves_values_by_at_most_half_a_new_step(old, new):
    c, s = oracle.quantize_rows(old, _rows(10 * old + new))
    y_old = oracle.dequantize_rows(old, c, s).astype(np.float64).reshape(-1, 4, 32)
    c2, s2 = oracle.regrade_rows(old, new, ROT_HADAMARD, c, s)
    y_new = oracle.dequantize_rows(new, c2, s2).astype(np.float64).reshape(-1, 4, 32)
    asym = new in (Q8_1, Q6_1, Q5_1, Q4_1, Q3_1, Q2_1)
    d = oracle.f16_to_f32(s2.reshape(-1, 4, 2)[..., 0] if asym else s2.reshape(-1, 4)).astype(np.float64)
    err = np.abs(y_new - y_old).max(axis=-1)
    assert (err <= d * (0.5 + 2.0 ** -10) + 1e-30).all()


@pytest.mark.parametrize("new", [Q8_0, Q4_0, Q2_1])
def test_regrade_of_f16_rows_is_the_append_encoding(new):
    rng = np.random.default_rng(new)
    raw = oracle.f16_rn(rng.standard_normal((300, 128)).astype(np.float32) * 3)
    c16, s16 = oracle.quantize_rows(F16, oracle.f16_to_f32(raw))
    assert np.array_equal(c16.view(np.uint16), raw)               # F16 rows store the raw values
    c, s = oracle.regrade_rows(F16, new, ROT_HADAMARD, c16, s16)
    ce, se = oracle.encode_rows(new, ROT_HADAMARD, raw)
    assert np.array_equal(c, ce)
    assert np.array_equal(s, se)
