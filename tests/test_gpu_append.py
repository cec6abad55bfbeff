"""Append-quantize through the C ABI against the oracle.

Packed rows read back from the paged cache must equal the oracle's encoding of
the same fp16 history bit for bit (Hadamard, variance-normalised and F16
paths); the F16 precision tail keeps exactly the newest T rows raw (BeeLlama
v0.4.0 news, §KV cache 精度尾部); the cache content does not depend on how the
history was chunked into appends.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _read(plan, w, layer, seq, kv, nq):
    cbs = [plan.row_bytes(layer, h, kv) for h in range(w.n_kv_heads)]
    tc = sum(c for c, _ in cbs) * nq
    ts = sum(s for _, s in cbs) * nq
    codes = torch.zeros(max(tc, 1), dtype=torch.uint8, device="cuda")
    scales = torch.zeros(max(ts, 2), dtype=torch.uint8, device="cuda")
    plan.read_rows(layer, seq, 0, nq, kv, codes, scales)
    torch.cuda.synchronize()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    out, co, so = [], 0, 0
    for cb, sb in cbs:
        c = codes[co:co + cb * nq].reshape(nq, cb)
        s = scales[so:so + sb * nq].reshape(nq, sb).copy().view(np.uint16) if sb else np.zeros((nq, 0), np.uint16)
        out.append((c, s))
        co += cb * nq
        so += sb * nq
    return out


@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_packed_rows_bit_exact(cfg):
    w = W.make_workload(cfg, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=700)
    for s in range(min(w.batch, 3)):
        for l in range(w.n_layers):
            nq = max(0, w.ctx[s] - w.tail)
            if nq == 0:
                continue
            for kv, kind in enumerate("KV"):
                rows = _read(plan, w, l, s, kv, nq)
                hist = w.rows(kind, l, s, 0, nq)
                for h in range(w.n_kv_heads):
                    args = H.head_params(w, l, h)
                    codec = args["k_codec"] if kv == 0 else args["v_codec"]
                    inv = args.get("inv_s_k" if kv == 0 else "inv_s_v")
                    oc, os_ = oracle.encode_rows(codec, w.rot, H.f16_bits(hist[:, h, :]), inv_s=inv)
                    gc, gs = rows[h]
                    assert np.array_equal(gc, oc), (cfg, s, l, kv, h)
                    assert np.array_equal(gs, os_), (cfg, s, l, kv, h)


def test_projection_codes_bit_exact():
    """The per-head projection path (KV-COBRA): packed rows read back from the cache
    equal the oracle's encoding of the same fp16 history bit for bit, every row, K and
    V, every head of both layers."""
    w = W.make_workload(4, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=512)
    for l in range(w.n_layers):
        for kv, kind in enumerate("KV"):
            rows = _read(plan, w, l, 0, kv, w.ctx[0])
            hist = w.rows(kind, l, 0, 0, w.ctx[0])
            for h in range(w.n_kv_heads):
                r = w.rank[l][h]
                b = w.k_bits[l][h] if kv == 0 else w.v_bits[l][h]
                M = oracle.fuse_projection(w.proj_basis(l, h))
                x = H.f16_bits(hist[:, h, :])
                oc, os_ = oracle.encode_rows(kvq.RANK, W.ROT_PROJECTION, x, M=M, r=r, b=b)
                gc, gs = rows[h]
                assert np.array_equal(gc, oc), (l, kv, h)
                assert np.array_equal(gs, os_), (l, kv, h)


def test_tail_holds_newest_rows_raw_and_dequantize_matches_oracle():
    w = W.make_workload(3, "small")           # tail 256, mixed codecs
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=333)
    n = w.ctx[0]
    for l in range(w.n_layers):
        k = torch.empty((n, w.n_kv_heads, 128), dtype=torch.float32, device="cuda")
        v = torch.empty_like(k)
        plan.dequantize(l, 0, 0, n, k, v)
        torch.cuda.synchronize()
        k, v = k.cpu().numpy(), v.cpu().numpy()
        for kind, got in (("K", k), ("V", v)):
            hist = w.rows(kind, l, 0, 0, n)
            raw = oracle.f16_to_f32(H.f16_bits(hist)).reshape(n, w.n_kv_heads, 128)
            # newest T rows: exactly the raw fp16 values
            assert np.array_equal(got[n - w.tail:], raw[n - w.tail:])
            for h in range(w.n_kv_heads):
                args = H.head_params(w, l, h)
                codec = args["k_codec"] if kind == "K" else args["v_codec"]
                nq = n - w.tail
                oc, os_ = oracle.encode_rows(codec, w.rot, H.f16_bits(hist[:nq, h, :]))
                ref = oracle.decode_rows_original(codec, w.rot, oc, os_)
                err = np.abs(got[:nq, h, :] - ref).max(axis=1) / np.maximum(np.abs(ref).max(axis=1), 1e-30)
                assert err.max() < 1e-5, (l, h, kind, err.max())


@pytest.mark.parametrize("cfg", [3, 5])
def test_chunking_does_not_change_the_cache(cfg):
    """Token-by-token and 97-token appends run the warp-per-row kernel, whole-
    history appends the four-threads-per-row one: the bytes must not differ
    (mixed per-layer codecs with F16 layers and a tail; KVarN with a tail)."""
    w = W.make_workload(cfg, "small")
    inv = H.gpu_inv_rms(w) if w.rot == W.ROT_VARNORM_HADAMARD else None
    a = H.make_plan(w, inv_rms=inv)
    b = H.make_plan(w, inv_rms=inv)
    H.fill(a, w, chunk=10_000)
    # token by token for the first 300 tokens, then uneven chunks
    for l in range(w.n_layers):
        for s in range(w.batch):
            t = 0
            step = 1
            while t < w.ctx[s]:
                n = min(step if t < 300 else 97, w.ctx[s] - t)
                b.append(l, [s], [n], w.rows("K", l, s, t, t + n, "cuda"), w.rows("V", l, s, t, t + n, "cuda"))
                t += n
    torch.cuda.synchronize()
    for l in range(w.n_layers):
        for s in range(w.batch):
            n = w.ctx[s]
            nq = max(0, n - w.tail)
            for kv in (0, 1):
                if nq:
                    ra, rb = _read(a, w, l, s, kv, nq), _read(b, w, l, s, kv, nq)
                    for (ca, sa), (cb_, sb_) in zip(ra, rb):
                        assert np.array_equal(ca, cb_) and np.array_equal(sa, sb_)
            ka = torch.empty((n, w.n_kv_heads, 128), device="cuda"); kb = torch.empty_like(ka)
            va = torch.empty_like(ka); vb = torch.empty_like(ka)
            a.dequantize(l, s, 0, n, ka, va)
            b.dequantize(l, s, 0, n, kb, vb)
            torch.cuda.synchronize()
            assert torch.equal(ka, kb) and torch.equal(va, vb)


def test_multi_sequence_append_matches_single_sequence_appends():
    w = W.make_workload(5, "small")
    inv = H.gpu_inv_rms(w)
    a = H.make_plan(w, inv_rms=inv)
    b = H.make_plan(w, inv_rms=inv)
    H.fill(a, w, chunk=100_000)
    for l in range(w.n_layers):
        ks = [w.rows("K", l, s, 0, w.ctx[s], "cuda") for s in range(w.batch)]
        vs = [w.rows("V", l, s, 0, w.ctx[s], "cuda") for s in range(w.batch)]
        b.append(l, list(range(w.batch)), w.ctx, torch.cat(ks), torch.cat(vs))
    torch.cuda.synchronize()
    for l in range(w.n_layers):
        for s in range(w.batch):
            n = w.ctx[s]
            ka = torch.empty((n, w.n_kv_heads, 128), device="cuda"); kb = torch.empty_like(ka)
            a.dequantize(l, s, 0, n, ka, None)
            b.dequantize(l, s, 0, n, kb, None)
            torch.cuda.synchronize()
            assert torch.equal(ka, kb)


def test_capacity_and_argument_errors_are_reported():
    w = W.make_workload(1)
    plan = H.make_plan(w)
    k = w.rows("K", 0, 0, 0, 8, "cuda")
    with pytest.raises(kvq.KVQError) as e:
        plan.append(0, [0], [w.ctx[0] + 1], k, k)
    assert e.value.status == 3
    with pytest.raises(kvq.KVQError) as e:
        plan.append(5, [0], [8], k, k)
    assert e.value.status == 1
    with pytest.raises(kvq.KVQError) as e:
        plan.append(0, [0, 0], [4, 4], k, k)
    assert e.value.status == 1
    # pool exhaustion: 2 pages for a sequence that needs 16
    small = H.make_plan(w, max_pages=2)
    kk = w.rows("K", 0, 0, 0, 1024, "cuda")
    with pytest.raises(kvq.KVQError) as e:
        small.append(0, [0], [1024], kk, kk)
    assert e.value.status == 3
    assert small.seq_length(0, 0) == 0
    small.check_device_error()
    plan.check_device_error()
