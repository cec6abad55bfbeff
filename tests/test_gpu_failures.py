"""Failure paths, made on the host or with bounded device waits (no GPU fault).

- An injected allocation failure makes kvq_plan_create return KVQ_ERR_OOM and no
  plan; the next creation, without the injection, succeeds.
- A decode launch whose producers skip their last tile (test-only injection) has
  a consumer whose bounded wait runs out after a short limit: the launch
  completes, kvq_check_device_error reports KVQ_ERR_TIMEOUT, and the context is
  still usable (the next, normal decode matches the oracle).
"""
import ctypes
import os

import pytest
import torch

from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def test_injected_allocation_failure_gives_oom_and_no_plan():
    w = W.make_workload(1)
    os.environ["KVQ_TEST_FAIL_ALLOC"] = "1"
    try:
        with pytest.raises(kvq.KVQError) as e:
            H.make_plan(w)
        assert e.value.status == 4                      # KVQ_ERR_OOM
        # the C entry point leaves the output handle null
        lib = kvq.lib()
        desc = kvq._Desc()
        kc = (ctypes.c_int * 2)(kvq.Q4_0, kvq.Q4_0)
        desc.n_layers, desc.n_q_heads, desc.n_kv_heads, desc.head_dim = 1, 8, 2, 128
        desc.max_seqs, desc.max_tokens_per_seq = 1, 1024
        desc.k_codec = ctypes.cast(kc, kvq._IP)
        desc.v_codec = ctypes.cast(kc, kvq._IP)
        desc.rot = kvq.ROT_HADAMARD
        h = ctypes.c_void_p(1234)
        assert lib.kvq_plan_create(ctypes.byref(desc), ctypes.byref(h)) == 4
        assert not h.value
    finally:
        del os.environ["KVQ_TEST_FAIL_ALLOC"]
    plan = H.make_plan(w)                               # works again
    assert plan.cache_bytes() > 0


def test_bounded_wait_runs_out_and_reports_timeout():
    w = W.make_workload(1, "full")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=512)
    q = w.queries(0, 0, 0, "cuda").unsqueeze(0)
    out = torch.empty((1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    ws = plan.new_workspace(1)
    plan.debug_set_decode_split(4)                      # several CTAs, each with tiles
    plan.debug_fault_injection(wait_limit_ns=1_000_000, drop_last_tile=True)
    plan.decode(0, [0], q, out, ws)
    with pytest.raises(kvq.KVQError) as e:
        plan.check_device_error()
    assert e.value.status == 7                          # KVQ_ERR_TIMEOUT
    # back to normal: the same context serves a correct decode
    plan.debug_fault_injection(wait_limit_ns=2_000_000_000, drop_last_tile=False)
    plan.debug_set_decode_split(0)
    ws.zero_()
    plan.decode(0, [0], q, out, ws)
    torch.cuda.synchronize()
    plan.check_device_error()
    got = out.cpu().numpy()[0]
    qb = H.f16_bits(q[0])
    for h in range(w.n_kv_heads):
        ref = H.oracle_decode(w, 0, 0, h, qb[h * w.G:(h + 1) * w.G])
        assert H.rel_err_rows(got[h * w.G:(h + 1) * w.G], ref).max() <= H.TOL


def test_fault_injection_rejects_bad_settings():
    w = W.make_workload(1)
    plan = H.make_plan(w)
    for args in ((10, False), (3_000_000_000, False)):
        with pytest.raises(kvq.KVQError):
            plan.debug_fault_injection(*args)
    with pytest.raises(kvq.KVQError):
        plan.debug_set_decode_split(-1)
