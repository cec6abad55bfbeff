"""The seeded input generator (quantized_kv_cache_15_b200.workloads): its normal
values follow N(0,1) -- the distribution the workloads name for K, V and the
queries -- and are a pure function of (stream key, element index), so any chunk
of rows can be regenerated on either side.  (Device independence of the bits is
checked on the GPU in test_gpu_a_workloads.py.)"""
from statistics import NormalDist

import numpy as np

from quantized_kv_cache_15_b200 import workloads as W

N = 4_000_000


def test_normal_values_match_the_standard_normal():
    x = W.gauss(20240, 0, N, "cpu").double().numpy()
    se = 1.0 / np.sqrt(N)
    assert abs(x.mean()) < 5 * se
    assert abs(x.var() - 1.0) < 5 * np.sqrt(2.0) * se
    nd = NormalDist()
    for q in (0.001, 0.01, 0.1, 0.3, 0.5, 0.7, 0.9, 0.99, 0.999):
        # quantile standard error sqrt(q(1-q)/N) / phi(z_q), five of them
        z = nd.inv_cdf(q)
        tol = 5 * np.sqrt(q * (1 - q) / N) / nd.pdf(z)
        assert abs(np.quantile(x, q) - z) < tol, (q, np.quantile(x, q), z)
    # tails: mass beyond 3 sigma within 5 standard errors, values reach past 4.5 sigma
    p3 = 2 * nd.cdf(-3.0)
    assert abs((np.abs(x) > 3).mean() - p3) < 5 * np.sqrt(p3 / N)
    assert np.abs(x).max() > 4.5


def test_values_depend_only_on_key_and_index():
    a = W.gauss(7, 1000, 5000, "cpu")
    b = W.gauss(7, 3000, 1000, "cpu")
    assert np.array_equal(a[2000:3000].numpy(), b.numpy())
    assert not np.array_equal(W.gauss(8, 1000, 5000, "cpu").numpy(), a.numpy())


def test_quantile_table_is_monotone_and_symmetric():
    t = W.normal_quantiles("cpu").double().numpy()
    assert t.shape == (65537,)
    assert np.all(np.diff(t) > 0)
    assert np.allclose(t, -t[::-1], atol=1e-6)
    assert t[32768] == 0.0
