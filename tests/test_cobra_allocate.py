"""The library's KV-COBRA allocator (host code behind the C ABI) against the
oracle's: identical allocations; the page's worked example; calibration time.
Runs without a GPU."""
import json
import os
import time

import numpy as np
import pytest

import oracle
from quantized_kv_cache_15_b200 import kvq

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cobra_budget.json")))


@pytest.fixture(scope="module")
def eps():
    z = np.random.default_rng(0).standard_normal((20000, 128)).astype(np.float32)
    out = []
    for b in (1, 2, 3, 4):
        c, s = oracle.quantize_rows(oracle.RANK, z, r=128, b=b)
        zh = oracle.dequantize_rows(oracle.RANK, c, s, r=128, b=b)
        out.append(float(np.mean((zh - z) ** 2) / np.mean(z ** 2)))
    return np.array(out)


def test_worked_example(eps):
    ex = G["allocation_example"]
    top, share = ex["head_A"]["top"], ex["head_A"]["top_share"]
    A = np.array([share / top] * top + [(1 - share) / (128 - top)] * (128 - top))
    B = np.full(128, 1.0 / 128)
    r, b, used = kvq.cobra_allocate(np.stack([A, B]), G["bpd"], eps)
    assert [(int(r[i]), int(b[i])) for i in range(2)] == [(e["rank"], e["bits"]) for e in ex["expected"]]
    assert used == ex["total_bits"]


@pytest.mark.parametrize("bpd", [0.5, 1.0, 2.0, 4.0])
def test_matches_oracle(eps, bpd):
    rng = np.random.default_rng(int(bpd * 10))
    lam = np.sort(rng.gamma(rng.uniform(0.05, 2.0, (256, 1)), size=(256, 128)), axis=1)[:, ::-1]
    lam /= lam.sum(axis=1, keepdims=True)
    r, b, used = kvq.cobra_allocate(lam, bpd, eps)
    ro, bo, uo = oracle.cobra_allocate(lam, bpd, eps)
    assert np.array_equal(r, ro) and np.array_equal(b, bo) and used == uo
    assert used <= int(bpd * 128 * 256 + 0.5)


def test_calibration_time_for_256_heads(eps):
    """The page reports the whole calibration under 200 ms; the allocation for the
    256 kv heads of a LLaMA-3.1-8B-shaped model is a small part of it."""
    lam = np.sort(np.random.default_rng(3).gamma(0.3, size=(256, 128)), axis=1)[:, ::-1]
    t0 = time.perf_counter()
    kvq.cobra_allocate(lam, 1.0, eps)
    assert time.perf_counter() - t0 < 0.2


def test_rejects_bad_input(eps):
    lam = np.full((2, 128), 1.0 / 128)
    with pytest.raises(kvq.KVQError):
        kvq.cobra_allocate(lam[:, ::-1] * np.arange(128)[None, :], 1.0, eps)   # not sorted
    with pytest.raises(kvq.KVQError):
        kvq.cobra_allocate(lam, 0.05, eps)                                     # below 16 bits per head
