"""Chunked-prefill attention over the quantized cache through the C ABI against the
oracle (forum thread on KV compression, attention paragraph; BeeLlama v0.4.0 news,
§KV cache 精度尾部 for the raw tail rows).

The last n_q tokens of a sequence attend causally: query i at position
len - n_q + i sees positions 0 .. len - n_q + i, i.e. a prefix of the quantized
rows and, once past them, a run of tail slots.  Each query is checked against
oracle attention over exactly that prefix of the oracle's own encoding (rows
older than the tail quantized, the rest raw), at the decode parity bar.

Layers of block codecs run on the tensor-core kernel (128 / G queries per CTA,
fp16 operand images); F16 pages and the rank codec, and every layer when the
test-only path switch asks for it, run each query through the decode kernel.
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
    out = torch.full((n_q, w.n_q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = plan.new_workspace(min(n_q, 256))
    plan.prefill(layer, seq, q, out, ws)
    torch.cuda.synchronize()
    plan.check_device_error()
    return q, out.cpu().numpy()


def _check(plan, w, layer, seq, n_q, sample):
    n = w.ctx[seq]
    nq_all = max(0, n - w.tail)
    q, out = _prefill(plan, w, layer, seq, n_q)
    assert np.isfinite(out).all()
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


def _sample(n_q, qb):
    """Every query of the first and last blocks, the block edges, and a stride."""
    s = set(range(0, min(n_q, qb))) | set(range(max(0, n_q - qb - 3), n_q)) | set(range(0, n_q, 7))
    s |= {b * qb + d for b in range(n_q // qb + 1) for d in (-1, 0) if 0 <= b * qb + d < n_q}
    return sorted(s)


@pytest.mark.parametrize("cfg,layer", [(1, 0), (2, 1), (3, 2), (3, 3), (3, 4), (5, 1), (3, 0), (3, 1)])
def test_prefill_queries_match_oracle(cfg, layer):
    """Block-codec layers (tensor cores): q4_0 without a tail (1), q8_0/q4_0 (2),
    q8_0/q6_0, q6_0/q4_1 and q4_1/q2_1 with a tail at GQA 6 (3), KVarN q4_0 with a
    tail (5); F16 layers of the VBR mix take the decode kernel (3: layers 0, 1)."""
    w = W.make_workload(cfg, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    seq = int(np.argmax(w.ctx))
    n = w.ctx[seq]
    n_q = min(n, 300)                      # several query blocks, the last one partial
    _check(plan, w, layer, seq, n_q, _sample(n_q, 128 // w.G))


ALL_BLOCK = [W.Q8_0, W.Q6_0, W.Q5_0, W.Q4_0, W.Q3_0, W.Q2_0, W.Q8_1, W.Q6_1, W.Q5_1, W.Q4_1, W.Q3_1, W.Q2_1]


@pytest.mark.parametrize("kc", ALL_BLOCK)
def test_every_block_codec_as_key_and_value(kc):
    """Each block codec as keys and (for the other kv head) as values on the
    tensor-core path, with a tail, GQA 4 and a query block crossing into the tail."""
    vc = ALL_BLOCK[(ALL_BLOCK.index(kc) + 5) % len(ALL_BLOCK)]
    w = W.make_workload(1, "full", ctx=[700], tail=64, n_q_heads=8, n_kv_heads=2,
                        k_codec=[[kc, vc]], v_codec=[[vc, kc]])
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=250)
    n_q = 150
    _check(plan, w, 0, 0, n_q, _sample(n_q, 32))


def test_prefill_of_the_whole_sequence():
    """n_q = len: the first query sees only position 0, the last one everything;
    one CTA per 32 positions and kv head, every tile on the causal diagonal once."""
    w = W.make_workload(5, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    seq = 1                                 # 1059 tokens: 16 quantized pages, a 64-token tail
    n = w.ctx[seq]
    _check(plan, w, 1, seq, n, _sample(n, 32))


def test_decode_kernel_path_matches_oracle_and_decode():
    """The test-only switch sends every query through the decode kernel: parity with
    the oracle, and its last query equals the decode call to rounding."""
    w = W.make_workload(5, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    plan.debug_set_prefill_path(1)
    seq, layer, n_q = 3, 1, 70
    q, out, _ = _check(plan, w, layer, seq, n_q, _sample(n_q, 32))
    ref = torch.empty((1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    plan.decode(layer, [seq], q[n_q - 1:n_q].contiguous(), ref, plan.new_workspace(1))
    torch.cuda.synchronize()
    assert H.rel_err_rows(out[n_q - 1], ref.cpu().numpy()[0]).max() < 1e-5
    with pytest.raises(kvq.KVQError):
        plan.debug_set_prefill_path(2)


def test_tensor_core_prefill_last_query_agrees_with_decode():
    """The tensor-core prefill's last query and the decode call compute the same
    attention with different roundings (fp16 operand images against integer dot
    products): they agree within the parity bar."""
    w = W.make_workload(5, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=640)
    seq, layer, n_q = 0, 1, 40
    q, out = _prefill(plan, w, layer, seq, n_q)
    ref = torch.empty((1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    plan.decode(layer, [seq], q[n_q - 1:n_q].contiguous(), ref, plan.new_workspace(1))
    torch.cuda.synchronize()
    assert H.rel_err_rows(out[n_q - 1], ref.cpu().numpy()[0]).max() <= H.TOL


def test_prefill_rejects_more_queries_than_tokens():
    w = W.make_workload(1, "small")
    plan = H.make_plan(w)
    H.fill(plan, w)
    n = w.ctx[0]
    q = torch.zeros((n + 1, w.n_q_heads, 128), dtype=torch.float16, device="cuda")
    out = torch.empty((n + 1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KVQError):
        plan.prefill(0, 0, q, out, plan.new_workspace(256))


def test_prefill_at_bench_scale_sampled():
    """The bench's prefill call at scale: 2048 queries at the end of one long
    KVarN q4_0 sequence (the batch workload's recipe, 256-token tail), every query
    block of 32 positions on the tensor cores; sampled queries (the first and last
    blocks' edges and a stride) against the oracle."""
    w = W.make_workload(5, "full", ctx=[24576])
    w.n_layers = 1
    w.k_codec, w.v_codec = w.k_codec[:1], w.v_codec[:1]
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=2048)
    n_q = 2048
    sample = sorted({0, 1, 31, 32, 1023, 1024, 2015, 2016, 2046, 2047} | set(range(5, n_q, 97)))
    _, _, worst = _check(plan, w, 0, 0, n_q, sample)
    assert worst <= H.TOL
