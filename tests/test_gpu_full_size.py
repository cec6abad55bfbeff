"""Parity at the workloads' full sizes, on sampled outputs.

The cache is filled through the C ABI exactly as bench.py fills it; every layer is
decoded; the oracle then recomputes sampled (sequence, layer, kv head) outputs
from the regenerated fp16 history (the inputs are device independent).  Sampled
packed rows are also compared bit for bit.  Bar: R16, 2e-3 per row.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _decode_all(plan, w, layers, seqs, step=0):
    outs = {}
    ws = plan.new_workspace(len(seqs))
    for l in layers:
        q = torch.stack([w.queries(l, s, step, "cuda") for s in seqs])
        out = torch.empty((len(seqs), w.n_q_heads, 128), dtype=torch.float32, device="cuda")
        plan.decode(l, seqs, q, out, ws)
        outs[l] = (q.cpu(), out)
    torch.cuda.synchronize()
    plan.check_device_error()
    return {l: (q, o.cpu().numpy()) for l, (q, o) in outs.items()}


def _check_samples(w, outs, samples, seqs):
    worst = 0.0
    for (l, si, h) in samples:
        q, out = outs[l]
        qh = H.f16_bits(q[si, h * w.G:(h + 1) * w.G])
        ref = H.oracle_decode(w, l, seqs[si], h, qh)
        err = H.rel_err_rows(out[si, h * w.G:(h + 1) * w.G], ref)
        worst = max(worst, float(err.max()))
        assert err.max() <= H.TOL, (l, seqs[si], h, err.max())
    return worst


def test_llama8b_shape_full():
    """32 layers x 32k, K q8_0 / V q4_0 (the bench workload)."""
    w = W.make_workload(2, "full")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=4096)
    outs = _decode_all(plan, w, range(w.n_layers), [0])
    _check_samples(w, outs, [(0, 0, 0), (13, 0, 5), (31, 0, 7)], [0])


def test_vbr_mix_full():
    """64 layers x 64k, tail 1024, every codec band of the VBR map."""
    w = W.make_workload(3, "full")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=8192)
    layers = [0, 7, 20, 40, 63]                        # F16, F16/q8_0, q8_0/q6_0, q6_0/q4_1, q4_1/q2_1
    outs = _decode_all(plan, w, layers, [0])
    _check_samples(w, outs, [(l, 0, l % 4) for l in layers], [0])


def test_cobra_rank_bits_full():
    """256 heads with per-head (r, b), 128k tokens, tcgen05 projection."""
    w = W.make_workload(4, "full")
    samples = [(0, 0, 0), (0, 0, 5), (17, 0, 3), (31, 0, 6)]
    H.make_projection_unambiguous(w, samples)
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=8192)
    layers = [0, 17, 31]
    outs = _decode_all(plan, w, layers, [0])
    _check_samples(w, outs, samples, [0])


def test_batched_kvarn_full():
    """64 ragged sequences, varnorm + H + q4_0, tail 256, then a 2048-token chunk
    appended to 8 sequences (the bench's serving step) before decoding."""
    w = W.make_workload(5, "full")
    plan = H.make_plan(w, extra_tokens=2048)
    H.fill(plan, w, chunk=8192)
    grown = list(range(0, 64, 8))
    for l in range(w.n_layers):
        ks = [w.rows("K", l, s, w.ctx[s], w.ctx[s] + 2048, "cuda") for s in grown]
        vs = [w.rows("V", l, s, w.ctx[s], w.ctx[s] + 2048, "cuda") for s in grown]
        plan.append(l, grown, [2048] * len(grown), torch.cat(ks), torch.cat(vs))
    for s in grown:
        w.ctx[s] += 2048
    seqs = list(range(64))
    layers = [0, 31]
    outs = _decode_all(plan, w, layers, seqs)
    samples = [(0, 0, 0), (0, 8, 3), (31, 17, 7), (31, 40, 2)]
    _check_samples(w, outs, samples, seqs)
