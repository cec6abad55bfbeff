"""kvq_decode_attention_noalloc: decode attention for callers that cannot allocate.

Some callers cannot hand the library a workspace (allocator-free runtimes,
hosts whose pool owns all device memory, loops that must never call cudaMalloc).
This entry point uses a fixed scratch array inside the library instead.  It must
give the same result as kvq_decode_attention (same tolerance as the parity
tests), call after call: the array keeps the previous call's contents, so the
second call checks that nothing stale leaks in.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode_twice():
    w = W.make_workload(3, "small")           # tail, mixed codecs, several splits per sequence
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=700)
    for step in range(2):
        for layer in range(w.n_layers):
            q = torch.stack([w.queries(layer, 0, step, "cuda")])
            ref = torch.empty((1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
            got = torch.full_like(ref, float("nan"))
            ws = plan.new_workspace(1)
            plan.decode(layer, [0], q, ref, ws)
            plan.decode_noalloc(layer, [0], q, got)
            torch.cuda.synchronize()
            err = H.rel_err_rows(got.cpu().numpy()[0], ref.cpu().numpy()[0])
            assert err.max() <= H.TOL, (step, layer, err.max())
    plan.check_device_error()


def test_noalloc_rejects_batches_beyond_the_scratch_limit():
    w = W.make_workload(5, "small")
    plan = H.make_plan(w)
    need = plan.workspace_bytes(200)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((200, w.n_q_heads, 128), dtype=torch.float16, device="cuda")
    out = torch.empty((200, w.n_q_heads, 128), device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        plan.decode_noalloc(0, [0] * 200, q, out)
    assert e.value.status == 3
