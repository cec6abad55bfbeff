"""Pins for the oracle's KV-COBRA rank/bit allocation.

KV-COBRA explainer, section "The news": C1 picks, inside a head, the rank and bit
width where dropping directions (their variance is lost outright) and thinner
bits (rounding noise, ~4x smaller per extra bit) balance; C2 moves budget across
heads, a bit going where it removes the most error ("water-filling").  Section
"Where the bits actually go" gives a worked two-head example, used here as the
golden case.  The rounding-noise factors are measured from the oracle's own
b-bit rank quantizer on Gaussian coordinates.
"""
import json
import os

import numpy as np
import pytest

import oracle

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


def _heads():
    ex = G["allocation_example"]["head_A"]
    top, share = ex["top"], ex["top_share"]
    A = np.array([share / top] * top + [(1 - share) / (128 - top)] * (128 - top))
    B = np.full(128, 1.0 / 128)
    return A, B


def test_rounding_noise_falls_about_4x_per_bit(eps):
    assert 3.0 < eps[1] / eps[2] < 7.0 and 3.0 < eps[2] / eps[3] < 7.0


def test_worked_example_allocation(eps):
    A, B = _heads()
    r, b, used = oracle.cobra_allocate(np.stack([A, B]), G["bpd"], eps)
    exp = G["allocation_example"]["expected"]
    assert [(int(r[i]), int(b[i])) for i in range(2)] == [(e["rank"], e["bits"]) for e in exp]
    assert used == G["allocation_example"]["total_bits"] == G["pair_total_bits"]


def test_worked_example_uniform_setting_loses_75_percent_of_head_b(eps):
    _, B = _heads()
    # lost variance alone is 96/128; the error model adds the rounding noise on top
    assert oracle.cobra_error(B, 32, 4, np.zeros(4)) == pytest.approx(0.75)
    assert oracle.cobra_error(B, 96, 2, np.zeros(4)) == pytest.approx(0.25)
    assert oracle.cobra_error(B, 96, 2, eps) < oracle.cobra_error(B, 32, 4, eps)


def test_c1_is_exhaustive_minimum(eps):
    rng = np.random.default_rng(1)
    for _ in range(50):
        lam = np.sort(rng.gamma(0.3, size=128))[::-1]
        lam /= lam.sum()
        budget = int(rng.integers(16, 513))
        best = oracle.cobra_best(lam, budget, eps)
        cands = [(oracle.cobra_error(lam, r, b, eps), r * b, r, b) for r in (16, 32, 64, 96, 128)
                 for b in (1, 2, 3, 4) if r * b <= budget]
        e, bits, r, b = min(cands)
        assert best == (r, b)


def test_c2_respects_budget_and_is_locally_optimal(eps):
    rng = np.random.default_rng(2)
    lam = np.sort(rng.gamma(0.3, size=(64, 128)), axis=1)[:, ::-1]
    lam /= lam.sum(axis=1, keepdims=True)
    r, b, used = oracle.cobra_allocate(lam, 1.0, eps)
    assert used == int((r * b).sum()) <= 64 * 128
    # every head's setting is C1-optimal for the bits it received
    for h in range(64):
        e = oracle.cobra_error(lam[h], int(r[h]), int(b[h]), eps)
        rb = oracle.cobra_best(lam[h], int(r[h] * b[h]), eps)
        assert oracle.cobra_error(lam[h], rb[0], rb[1], eps) >= e - 1e-12
    # concentrated heads get fewer bits than diffuse ones on average
    top16 = lam[:, :16].sum(axis=1)
    conc, diff = top16 > np.median(top16), top16 <= np.median(top16)
    assert (r * b)[conc].mean() < (r * b)[diff].mean()
