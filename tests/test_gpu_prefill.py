"""Chunked-prefill attention over the quantized cache through the C ABI against the
oracle (forum thread on KV compression, attention paragraph; BeeLlama v0.4.0 news,
§KV cache 精度尾部 for the raw tail rows).

The last n_q tokens of a sequence attend causally: query i at position
len - n_q + i sees positions 0 .. len - n_q + i, i.e. a prefix of the quantized
rows and, once past them, a cyclic run of tail slots.  Each query is checked
against oracle attention over exactly that prefix of the oracle's own encoding
(rows older than the tail quantized, the rest raw), at the decode parity bar.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _prefill(plan, w, layer, seq, n_q):
    q = torch.stack([w.queries(layer, seq, i, "cuda") for i in range(n_q)]).contiguous()
    out = torch.empty((n_q, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    ws = plan.new_workspace(min(n_q, 256))
    plan.prefill(layer, seq, q, out, ws)
    torch.cuda.synchronize()
    return q, out.cpu().numpy()


def _check(plan, w, layer, seq, n_q, sample):
    n = w.ctx[seq]
    nq_all = max(0, n - w.tail)
    q, out = _prefill(plan, w, layer, seq, n_q)
    worst = 0.0
    for h in range(w.n_kv_heads):
        args = H.head_params(w, layer, h)
        K = H.f16_bits(w.rows("K", layer, seq, 0, n)[:, h, :])
        V = H.f16_bits(w.rows("V", layer, seq, 0, n)[:, h, :])
        ck, sk = oracle.encode_rows(args["k_codec"], w.rot, K[:nq_all], inv_s=args.get("inv_s_k"))
        cv, sv = oracle.encode_rows(args["v_codec"], w.rot, V[:nq_all], inv_s=args.get("inv_s_v"))
        for i in sample:
            lim = n - n_q + i + 1
            nqv = min(lim, nq_all)
            ref = oracle.decode_packed(ck[:nqv], sk[:nqv], cv[:nqv], sv[:nqv], K[nq_all:lim], V[nq_all:lim],
                                       H.f16_bits(q[i, h * w.G:(h + 1) * w.G]), args["k_codec"], args["v_codec"],
                                       w.rot, inv_s_k=args.get("inv_s_k"), inv_s_v=args.get("inv_s_v"))
            err = H.rel_err_rows(out[i, h * w.G:(h + 1) * w.G], ref)
            worst = max(worst, float(err.max()))
            assert err.max() <= H.TOL, (layer, seq, h, i, lim, err.max())
    return q, out, worst


@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_prefill_queries_match_oracle(cfg):
    w = W.make_workload(cfg, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    seq = int(np.argmax(w.ctx))
    n = w.ctx[seq]
    n_q = min(n, 300)                      # more than one launch of 256 queries
    # every query whose visible tail run changes tile, plus a stride through the rest
    sample = sorted(set(range(0, n_q, 9)) | set(range(max(0, n_q - 70), n_q)) | {0, n_q - 1})
    _check(plan, w, w.n_layers - 1, seq, n_q, sample)


def test_last_prefill_query_is_the_decode_query():
    w = W.make_workload(5, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    seq, layer, n_q = 0, 1, 40
    q, out = _prefill(plan, w, layer, seq, n_q)
    ref = torch.empty((1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    plan.decode(layer, [seq], q[n_q - 1:n_q].contiguous(), ref, plan.new_workspace(1))
    torch.cuda.synchronize()
    assert H.rel_err_rows(out[n_q - 1], ref.cpu().numpy()[0]).max() < 1e-5


def test_prefill_rejects_more_queries_than_tokens():
    w = W.make_workload(1, "small")
    plan = H.make_plan(w)
    H.fill(plan, w)
    n = w.ctx[0]
    q = torch.zeros((n + 1, w.n_q_heads, 128), dtype=torch.float16, device="cuda")
    out = torch.empty((n + 1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KVQError):
        plan.prefill(0, 0, q, out, plan.new_workspace(256))
