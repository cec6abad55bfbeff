"""Pins for the oracle's Hadamard rotation, variance normalisation and fused projection.

KV-COBRA explainer, section "Jargon" (Hadamard rotation: a fixed +-1 orthogonal
transform that evens out channel variances) and section "The news" (the rotation
is fused into the per-head projection); BeeLlama v0.4.0 news, section KVarN
(variance-normalised quantization).
"""
from decimal import Decimal, getcontext

import numpy as np

import oracle
from quantized_kv_cache_15_b200 import workloads as W


def test_hadamard_is_sylvester_and_orthogonal():
    H = oracle.hadamard_matrix(128).astype(np.int64)
    # closed form of the Sylvester matrix: (-1)^popcount(i & j)
    i = np.arange(128)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    assert np.array_equal(H, np.where(pc % 2 == 0, 1, -1))
    assert np.array_equal(H @ H.T, 128 * np.eye(128, dtype=np.int64))
    H4 = oracle.hadamard_matrix(4).astype(np.int64)
    assert np.array_equal(H4, [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]])


def test_c_is_nearest_float_to_inverse_sqrt128():
    getcontext().prec = 50
    c = oracle.hadamard_c()
    true = Decimal(1) / Decimal(128).sqrt()
    cbits = np.float32(c).view(np.uint32)
    lo = Decimal(float(np.uint32(cbits - 1).view(np.float32)))
    hi = Decimal(float(np.uint32(cbits + 1).view(np.float32)))
    d = abs(Decimal(float(c)) - true)
    assert d < abs(lo - true) and d < abs(hi - true)
    assert hex(cbits) == "0x3db504f3"


def test_rotation_preserves_norm_and_is_involution():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 128))
    y = oracle.rotate_dense(x)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    assert np.allclose(oracle.rotate_dense(y), x, rtol=0, atol=1e-12)


def test_spec_fwht_matches_dense_rotation():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((256, 128)) * rng.uniform(0.1, 50, (1, 128))).astype(np.float32)
    y32 = oracle.fwht_spec(x).astype(np.float64)
    yd = oracle.rotate_dense(x.astype(np.float64))
    err = np.abs(y32 - yd).max(axis=1) / np.linalg.norm(x.astype(np.float64), axis=1)
    assert err.max() < 1e-6
    # basis vectors go to a column of H / sqrt(128): the FWHT is the Sylvester transform
    e = np.eye(128, dtype=np.float32)[:8]
    H = oracle.hadamard_matrix(128)
    assert np.allclose(oracle.fwht_spec(e), H[:, :8].T / np.sqrt(128.0), atol=1e-7)


def test_rotation_flattens_outlier_channel_variance():
    w = W.make_workload(1)
    k = w.rows("K", 0, 0, 0, 1024)[:, 0, :].numpy().view(np.uint16)
    x = oracle.f16_to_f32(k)
    before = x.var(axis=0)
    after = oracle.fwht_spec(x).var(axis=0)
    assert before.max() / before.min() > 200.0         # 4 channels x20 in std -> ~400 in variance
    assert after.max() / after.min() < 2.0


def test_varnorm_inv_rms_closed_form():
    rng = np.random.default_rng(3)
    a = np.float16(rng.uniform(0.01, 30, 128)).astype(np.float32)
    signs = rng.choice([-1.0, 1.0], size=(512, 128)).astype(np.float32)
    x = (signs * a[None, :]).astype(np.float16)
    x[:, 5] = 0.0                                          # degenerate channel -> 1
    inv = oracle.varnorm_inv_rms(x.view(np.uint16))
    expect = (1.0 / a.astype(np.float64)).astype(np.float32)
    expect[5] = 1.0
    assert np.array_equal(inv, expect)


def test_fused_projection_is_orthonormal_and_reduces_to_hadamard():
    rng = np.random.default_rng(4)
    for r in (16, 32, 64, 96, 128):
        P, _ = np.linalg.qr(rng.standard_normal((128, r)))
        M = oracle.fuse_projection(P).astype(np.float64)
        assert np.abs(M @ M.T - np.eye(r)).max() < 1e-6
    # P = I (r = 128) gives the plain rotation
    M = oracle.fuse_projection(np.eye(128))
    H = oracle.hadamard_matrix(128)
    assert np.array_equal(M, (H / np.sqrt(128.0)).astype(np.float32))
    # r = 96: block-diagonal H_32 / sqrt(32) acting on the first 96 coordinates
    M = oracle.fuse_projection(np.eye(128)[:, :96]).astype(np.float64)
    H32 = oracle.hadamard_matrix(32) / np.sqrt(32.0)
    expect = np.zeros((96, 128))
    for b in range(3):
        expect[32 * b:32 * b + 32, 32 * b:32 * b + 32] = H32
    assert np.allclose(M, expect, atol=1e-7)


def test_projection_keeps_rank_fraction_of_isotropic_variance():
    """KV-COBRA explainer, 'Where the bits actually go': an isotropic head projected
    to rank 32 keeps 32 of 128 directions and loses 75% of its variance; rank 96
    loses 25%."""
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cobra_budget.json")))
    rng = np.random.default_rng(5)
    x = rng.standard_normal((20000, 128))
    for item in g["isotropic_lost_variance"]:
        r = item["rank"]
        P, _ = np.linalg.qr(rng.standard_normal((128, r)))
        M = oracle.fuse_projection(P).astype(np.float64)
        kept = (np.square(x @ M.T).sum()) / np.square(x).sum()
        assert abs((1.0 - kept) - item["lost"]) < 0.01
