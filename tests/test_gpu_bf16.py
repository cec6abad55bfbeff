"""BF16 plans through the C ABI against the oracle (BeeLlama v0.4.0 news, §KV cache
精度尾部: the newest tokens may be kept in BF16 or F16).

bf16 K/V rows are appended (chunks through the four-threads-per-row kernel, single
tokens through the warp-per-row kernel), quantized bit-exactly like the oracle's
bf16 path, and kept raw in a bf16 tail; decode with bf16 queries matches the
oracle within the parity bar.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _rows(w, kind, l, s, t0, t1):
    return w.rows(kind, l, s, t0, t1, "cuda").to(torch.bfloat16)


def _plan(w, inv=None):
    kwargs = {}
    if w.rot == W.ROT_VARNORM_HADAMARD:
        kwargs["inv_rms"] = H.gpu_inv_rms(w) if inv is None else inv
    plan = kvq.Plan(w.n_layers, w.n_q_heads, w.n_kv_heads, max_seqs=w.batch, max_tokens_per_seq=max(w.ctx),
                    k_codec=np.array(w.k_codec, np.int32), v_codec=np.array(w.v_codec, np.int32), rot=w.rot,
                    tail_tokens=w.tail, kv_dtype=kvq.KV_BF16, **kwargs)
    plan.allocate_cache()
    return plan


def _fill(plan, w, chunk):
    for l in range(w.n_layers):
        for s in range(w.batch):
            t = 0
            while t < w.ctx[s]:
                n = min(chunk, w.ctx[s] - t)
                plan.append(l, [s], [n], _rows(w, "K", l, s, t, t + n), _rows(w, "V", l, s, t, t + n))
                t += n
    torch.cuda.synchronize()


def _read(plan, w, layer, seq, kv, nq):
    cbs = [plan.row_bytes(layer, h, kv) for h in range(w.n_kv_heads)]
    codes = torch.zeros(max(sum(c for c, _ in cbs) * nq, 1), dtype=torch.uint8, device="cuda")
    scales = torch.zeros(max(sum(s for _, s in cbs) * nq, 2), dtype=torch.uint8, device="cuda")
    plan.read_rows(layer, seq, 0, nq, kv, codes, scales)
    torch.cuda.synchronize()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    out, co, so = [], 0, 0
    for cb, sb in cbs:
        out.append((codes[co:co + cb * nq].reshape(nq, cb), scales[so:so + sb * nq].reshape(nq, sb).copy().view(np.uint16)))
        co += cb * nq
        so += sb * nq
    return out


@pytest.mark.parametrize("cfg", [2, 5])
def test_bf16_rows_quantize_bit_exact_and_tail_stays_raw(cfg):
    w = W.make_workload(cfg, "small")
    plan = _plan(w)
    _fill(plan, w, chunk=700)
    for s in range(min(w.batch, 3)):
        n = w.ctx[s]
        nq = max(0, n - w.tail)
        for l in range(w.n_layers):
            for kv, kind in enumerate("KV"):
                hist = _bits(_rows(w, kind, l, s, 0, n))
                if nq:
                    rows = _read(plan, w, l, s, kv, nq)
                    for h in range(w.n_kv_heads):
                        args = H.head_params(w, l, h)
                        codec = args["k_codec"] if kv == 0 else args["v_codec"]
                        inv = args.get("inv_s_k" if kv == 0 else "inv_s_v")
                        oc, os_ = oracle.encode_rows(codec, w.rot, hist[:nq, h, :], inv_s=inv, bf16=True)
                        assert np.array_equal(rows[h][0], oc), (cfg, s, l, kind, h)
                        assert np.array_equal(rows[h][1], os_), (cfg, s, l, kind, h)
            if w.tail and n > nq:
                k = torch.empty((n, w.n_kv_heads, 128), device="cuda")
                v = torch.empty_like(k)
                plan.dequantize(l, s, 0, n, k, v)
                torch.cuda.synchronize()
                for t, kind in ((k, "K"), (v, "V")):
                    raw = _rows(w, kind, l, s, nq, n).float().cpu().numpy()
                    assert np.array_equal(t[nq:].cpu().numpy(), raw)


@pytest.mark.parametrize("cfg", [2, 5])
def test_bf16_decode_matches_oracle(cfg):
    w = W.make_workload(cfg, "small")
    plan = _plan(w)
    _fill(plan, w, chunk=640)
    seqs = list(range(w.batch))
    q = torch.stack([w.queries(0, s, 0, "cuda") for s in seqs]).to(torch.bfloat16)
    for l in range(w.n_layers):
        out = torch.empty((len(seqs), w.n_q_heads, 128), dtype=torch.float32, device="cuda")
        plan.decode(l, seqs, q, out, plan.new_workspace(len(seqs)))
        torch.cuda.synchronize()
        out = out.cpu().numpy()
        for i, s in enumerate(seqs):
            K = _bits(_rows(w, "K", l, s, 0, w.ctx[s]))
            V = _bits(_rows(w, "V", l, s, 0, w.ctx[s]))
            for h in range(w.n_kv_heads):
                ref = oracle.decode_head(K[:, h, :], V[:, h, :], _bits(q[i, h * w.G:(h + 1) * w.G]),
                                         bf16=True, **H.head_params(w, l, h))
                err = H.rel_err_rows(out[i, h * w.G:(h + 1) * w.G], ref)
                assert err.max() <= H.TOL, (cfg, l, s, h, err.max())


def test_bf16_single_tokens_and_chunks_build_the_same_cache():
    w = W.make_workload(5, "small")
    inv = H.gpu_inv_rms(w)
    a, b = _plan(w, inv), _plan(w, inv)
    _fill(a, w, chunk=10_000)
    _fill(b, w, chunk=1)
    for l in range(w.n_layers):
        for s in range(w.batch):
            n = w.ctx[s]
            ka = torch.empty((n, w.n_kv_heads, 128), device="cuda"); kb = torch.empty_like(ka)
            va = torch.empty_like(ka); vb = torch.empty_like(ka)
            a.dequantize(l, s, 0, n, ka, va)
            b.dequantize(l, s, 0, n, kb, vb)
            torch.cuda.synchronize()
            assert torch.equal(ka, kb) and torch.equal(va, vb), (l, s)


def test_bf16_plans_keep_raw_rows_in_the_tail_only():
    with pytest.raises(kvq.KVQError) as e:
        kvq.Plan(1, 8, 2, max_seqs=1, max_tokens_per_seq=128, k_codec=[kvq.F16, kvq.Q4_0],
                 v_codec=[kvq.Q4_0, kvq.Q4_0], rot=kvq.ROT_HADAMARD, kv_dtype=kvq.KV_BF16)
    assert e.value.status == 2


@pytest.mark.parametrize("path", [0, 1])
def test_bf16_prefill_matches_oracle(path):
    """Chunked prefill of a bf16 plan (bf16 queries, bf16 raw tail rows) on the
    tensor-core path (0) and the decode-kernel path (1): sampled causal queries
    against the oracle's bf16 encoding of the rows older than the tail."""
    w = W.make_workload(5, "small")
    plan = _plan(w)
    _fill(plan, w, chunk=640)
    plan.debug_set_prefill_path(path)
    seq, layer = 1, 1
    n = w.ctx[seq]
    nq_all = n - w.tail
    n_q = 150
    q = torch.stack([w.queries(layer, seq, i, "cuda") for i in range(n_q)]).to(torch.bfloat16).contiguous()
    out = torch.empty((n_q, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
    plan.prefill(layer, seq, q, out, plan.new_workspace(min(n_q, 256)))
    torch.cuda.synchronize()
    plan.check_device_error()
    out = out.cpu().numpy()
    K = _bits(_rows(w, "K", layer, seq, 0, n))
    V = _bits(_rows(w, "V", layer, seq, 0, n))
    for h in range(w.n_kv_heads):
        args = H.head_params(w, layer, h)
        ck, sk = oracle.encode_rows(args["k_codec"], w.rot, K[:nq_all, h, :], inv_s=args.get("inv_s_k"), bf16=True)
        cv, sv = oracle.encode_rows(args["v_codec"], w.rot, V[:nq_all, h, :], inv_s=args.get("inv_s_v"), bf16=True)
        for i in sorted({0, 31, 32, 63, 64, 85, 86, 117, 118, 149} | set(range(3, n_q, 11))):
            lim = n - n_q + i + 1
            nqv = min(lim, nq_all)
            ref = oracle.decode_packed(ck[:nqv], sk[:nqv], cv[:nqv], sv[:nqv], K[nq_all:lim, h, :],
                                       V[nq_all:lim, h, :], _bits(q[i, h * w.G:(h + 1) * w.G]), args["k_codec"],
                                       args["v_codec"], w.rot, inv_s_k=args.get("inv_s_k"),
                                       inv_s_v=args.get("inv_s_v"), bf16=True)
            err = H.rel_err_rows(out[i, h * w.G:(h + 1) * w.G], ref)
            assert err.max() <= H.TOL, (path, h, i, err.max())
