"""kvq_decode_attention_noalloc: decode attention for callers that cannot allocate.

Some callers cannot hand the library a workspace: runtimes without a device
allocator, hosts whose memory pool owns all device memory and cannot lend a slice
to a library, and loops that must never call cudaMalloc (it can synchronise the
device).  This entry point uses a fixed scratch array inside the library instead.
Its output must match the CPU oracle within the tolerance of the other parity
tests (2e-3 per row), call after call: the array keeps the previous call's
contents, so the second call checks that nothing stale leaks in.  It must also
leave the device's free memory and torch's allocations unchanged.  This file is
collected last.
"""
import gc

import pytest
import torch

from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [3, 4])
def test_noalloc_decode_matches_the_oracle_twice(cfg):
    """Workload 3 (tail, mixed codecs, several splits) and workload 4 (per-head
    projection: the projected queries also live in the scratch array)."""
    w = W.make_workload(cfg, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=700)
    seqs = list(range(w.batch))
    # warm-up call: the first call on a device looks the array's address up
    q0 = torch.stack([w.queries(0, s, 9, "cuda") for s in seqs])
    o0 = torch.empty((len(seqs), w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    plan.decode_noalloc(0, seqs, q0, o0)
    torch.cuda.synchronize()
    qs = {(step, l): torch.stack([w.queries(l, s, step, "cuda") for s in seqs])
          for step in range(2) for l in range(w.n_layers)}
    outs = {k: torch.full((len(seqs), w.n_q_heads, 128), float("nan"), device="cuda") for k in qs}
    # objects of earlier tests that the collector frees in the middle of the calls
    # would change the device's free memory: collect them first, then hold it off
    gc.collect()
    torch.cuda.synchronize()
    gc.disable()
    try:
        alloc0 = torch.cuda.memory_allocated()
        free0, _ = torch.cuda.mem_get_info()
        for step in range(2):
            for l in range(w.n_layers):
                plan.decode_noalloc(l, seqs, qs[(step, l)], outs[(step, l)])
        torch.cuda.synchronize()
        alloc1 = torch.cuda.memory_allocated()
        free1, _ = torch.cuda.mem_get_info()
    finally:
        gc.enable()
    assert alloc1 == alloc0
    assert free1 == free0
    plan.check_device_error()
    for (step, l), out in outs.items():
        got = out.cpu().numpy()
        q = qs[(step, l)].cpu()
        for i, s in enumerate(seqs):
            for h in range(w.n_kv_heads):
                ref = H.oracle_decode(w, l, s, h, H.f16_bits(q[i, h * w.G:(h + 1) * w.G]))
                err = H.rel_err_rows(got[i, h * w.G:(h + 1) * w.G], ref).max()
                assert err <= H.TOL, (cfg, step, l, s, h, err)


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


def test_noalloc_checks_arguments_before_enqueueing():
    """Bad arguments come back as argument errors: the entry point validates the
    whole call before it resets the scratch array's merge counters."""
    w = W.make_workload(3, "small")
    plan = H.make_plan(w)
    q = torch.zeros((1, w.n_q_heads, 128), dtype=torch.float16, device="cuda")
    out = torch.empty((1, w.n_q_heads, 128), device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        plan.decode_noalloc(w.n_layers, [0], q, out)    # layer out of range
    assert e.value.status == 1
    with pytest.raises(kvq.KVQError) as e:
        plan.decode_noalloc(0, [w.batch], q, out)       # sequence out of range
    assert e.value.status == 1
