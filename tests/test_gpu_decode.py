"""Decode attention through the C ABI against the oracle.

Forum thread on KV compression (attention paragraph): dot the query with every
prior key, softmax, weighted average of the values.  The oracle attends in fp64
over the dequantized cache in the original basis; the GPU works in the stored
basis in fp32.  Bar: max_j |o - o*| <= 2e-3 * max_j |o*| per (sequence, query
head) row (R16).
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _decode(plan, w, layer, seqs, step=0):
    q = torch.stack([w.queries(layer, s, step, "cuda") for s in seqs])
    out = torch.empty((len(seqs), w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    ws = plan.new_workspace(len(seqs))
    plan.decode(layer, seqs, q, out, ws)
    torch.cuda.synchronize()
    return q, out.cpu().numpy()


def _check(plan, w, layers=None, seqs=None, step=0, tol=H.TOL):
    seqs = list(range(w.batch)) if seqs is None else seqs
    layers = range(w.n_layers) if layers is None else layers
    worst = 0.0
    for l in layers:
        q, out = _decode(plan, w, l, seqs, step)
        for i, s in enumerate(seqs):
            for h in range(w.n_kv_heads):
                qh = H.f16_bits(q[i, h * w.G:(h + 1) * w.G])
                ref = H.oracle_decode(w, l, s, h, qh)
                err = H.rel_err_rows(out[i, h * w.G:(h + 1) * w.G], ref)
                worst = max(worst, float(err.max()))
                assert err.max() <= tol, (l, s, h, err.max())
    return worst


def test_tiny_workload_full_size():
    w = W.make_workload(1, "full")
    plan = H.make_plan(w)
    H.fill(plan, w)
    _check(plan, w)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_workloads_small(cfg):
    w = W.make_workload(cfg, "small")       # the workload's own rows, nothing substituted
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    _check(plan, w)


def test_tail_covering_context_equals_f16_cache():
    """A tail that covers the whole context gives F16 attention: the same raw rows,
    read from 16-row tail pages instead of 64-row F16 pages, so only the order of
    the fp32 softmax merges differs (the oracle checks the bit-for-bit form)."""
    a = W.make_workload(1, "full", ctx=[768], tail=1024, k_codec=[[W.Q2_0] * 2], v_codec=[[W.Q2_0] * 2])
    b = W.make_workload(1, "full", ctx=[768], tail=0, k_codec=[[W.F16] * 2], v_codec=[[W.F16] * 2])
    pa, pb = H.make_plan(a), H.make_plan(b)
    H.fill(pa, a, chunk=100)
    H.fill(pb, b, chunk=100)
    _, oa = _decode(pa, a, 0, [0])
    _, ob = _decode(pb, b, 0, [0])
    assert H.rel_err_rows(oa[0], ob[0]).max() < 1e-6
    _check(pa, a)


def test_split_count_invariance():
    w = W.make_workload(3, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    outs = []
    for pps in (1, 3, 1000):
        plan.debug_set_decode_split(pps)
        outs.append(_decode(plan, w, 2, [0])[1])
    plan.debug_set_decode_split(0)
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 1e-5 * np.abs(outs[0]).max()


def test_lengths_edge_cases():
    """Empty context (zeros), a single token, lengths around page and tail edges."""
    w = W.make_workload(5, "small", ctx=[0, 1, 63, 64, 65, 129])
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=50)
    q, out = _decode(plan, w, 0, list(range(6)))
    assert np.abs(out[0]).max() == 0.0
    _check(plan, w, seqs=[1, 2, 3, 4, 5])


def test_decode_reports_bad_arguments():
    w = W.make_workload(1)
    plan = H.make_plan(w)
    q = torch.zeros((1, 8, 128), dtype=torch.float16, device="cuda")
    out = torch.empty((1, 8, 128), device="cuda")
    ws = plan.new_workspace(1)
    with pytest.raises(kvq.KVQError):
        plan.decode(1, [0], q, out, ws)
    with pytest.raises(kvq.KVQError):
        plan.decode(0, [7], q, out, ws)


ALL_CODECS = [W.Q8_0, W.Q6_0, W.Q5_0, W.Q4_0, W.Q3_0, W.Q2_0, W.Q8_1, W.Q6_1, W.Q5_1, W.Q4_1, W.Q3_1, W.Q2_1, W.F16]


@pytest.mark.parametrize("kc", ALL_CODECS)
def test_every_codec_as_key_and_value(kc):
    """Every block codec on the key side (integer dot products) and on the value side
    (packed fp32 accumulation), with a tail, GQA 4, ragged lengths."""
    vc = ALL_CODECS[(ALL_CODECS.index(kc) + 5) % len(ALL_CODECS)]
    w = W.make_workload(1, "full", ctx=[700, 131], tail=64, n_q_heads=8, n_kv_heads=2,
                        k_codec=[[kc, vc]], v_codec=[[vc, kc]])
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=250)
    _check(plan, w)


def test_one_workspace_serves_calls_of_any_smaller_size():
    """The merge counters sit at a fixed place in the workspace, so one zeroed
    workspace serves a mix of batch sizes (here 6, 2, 5, 6 sequences)."""
    w = W.make_workload(5, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    ws = plan.new_workspace(w.batch)
    for seqs in (list(range(w.batch)), [4, 1], [0, 2, 3, 4, 5], list(range(w.batch))):
        q = torch.stack([w.queries(0, s, 0, "cuda") for s in seqs])
        out = torch.empty((len(seqs), w.n_q_heads, 128), dtype=torch.float32, device="cuda")
        plan.decode(0, seqs, q, out, ws)
        torch.cuda.synchronize()
        out = out.cpu().numpy()
        for i, s in enumerate(seqs):
            for h in range(w.n_kv_heads):
                ref = H.oracle_decode(w, 0, s, h, H.f16_bits(q[i, h * w.G:(h + 1) * w.G]))
                assert H.rel_err_rows(out[i, h * w.G:(h + 1) * w.G], ref).max() <= H.TOL, (seqs, s, h)
