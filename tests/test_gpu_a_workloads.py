"""The seeded input generators give the same bits on CPU and CUDA, so the oracle
can regenerate any slice of what the GPU path was fed."""
import pytest
import torch

from quantized_kv_cache_15_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_generators_device_independent(cfg):
    w = W.make_workload(cfg, "small")
    for kind in "KV":
        for (l, s, t0, t1) in ((0, 0, 0, 300), (w.n_layers - 1, w.batch - 1, 77, 333)):
            a = w.rows(kind, l, s, t0, t1, "cpu")
            b = w.rows(kind, l, s, t0, t1, "cuda").cpu()
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), (cfg, kind, l, s)
    qa = w.queries(0, 0, 3, "cpu")
    qb = w.queries(0, 0, 3, "cuda").cpu()
    assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
    ca = w.calib_rows("K", 0, 512, "cpu")
    cb = w.calib_rows("K", 0, 512, "cuda").cpu()
    assert torch.equal(ca.view(torch.int16), cb.view(torch.int16))
