"""Parity at the workloads' full sizes.

The cache is filled through the C ABI exactly as bench.py fills it and every
checked layer is decoded in the launch configuration the bench times.  The
oracle then recomputes (sequence, layer, kv head) cells from the regenerated
fp16 history: every layer of sequence 0 for the single-sequence workloads, and
32+ cells of the 64-sequence batch.  Sampled runs of packed rows are compared
bit for bit with the oracle's encoding of the same rows.  Bar: R16, 2e-3 per
(sequence, query head) row.

The seeded generators give the same bits on every device
(tests/test_gpu_a_workloads.py), so the history is regenerated on the GPU and
copied to the host; the oracle runs on the host cores, one cell per thread (its
C code runs outside the interpreter lock).
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, os.cpu_count() or 1))


def _decode_all(plan, w, layers, seqs, step=0):
    outs = {}
    ws = plan.new_workspace(len(seqs))
    for l in layers:
        q = torch.stack([w.queries(l, s, step, "cuda") for s in seqs])
        out = torch.empty((len(seqs), w.n_q_heads, 128), dtype=torch.float32, device="cuda")
        plan.decode(l, seqs, q, out, ws)
        outs[l] = (q, out)
    torch.cuda.synchronize()
    plan.check_device_error()
    return {l: (q.cpu(), o.cpu().numpy()) for l, (q, o) in outs.items()}


def _history(w, layer, seq, n):
    """fp16 bits of K and V [n][Hkv][128] of one (layer, sequence), generated on the GPU."""
    k = H.f16_bits(w.rows("K", layer, seq, 0, n, "cuda"))
    v = H.f16_bits(w.rows("V", layer, seq, 0, n, "cuda"))
    return k, v


def _check_cells(w, outs, cells, seqs):
    """Oracle decode of every (layer, index into seqs, kv head) cell; returns the worst
    relative error and asserts the bar per cell."""
    by_ls = {}
    for (l, si, h) in cells:
        by_ls.setdefault((l, si), []).append(h)
    jobs = []
    for (l, si), heads in by_ls.items():
        s = seqs[si]
        K, V = _history(w, l, s, w.ctx[s])
        q, out = outs[l]
        for h in heads:
            qh = H.f16_bits(q[si, h * w.G:(h + 1) * w.G])
            jobs.append(((l, s, h), K[:, h, :].copy(), V[:, h, :].copy(), qh, H.head_params(w, l, h),
                         out[si, h * w.G:(h + 1) * w.G]))

    def run(job):
        cell, K, V, qh, hp, got = job
        ref = oracle.decode_head(K, V, qh, **hp)
        return cell, float(H.rel_err_rows(got, ref).max())

    with ThreadPoolExecutor(max_workers=THREADS) as pool:
        res = list(pool.map(run, jobs))
    bad = [(c, e) for c, e in res if not e <= H.TOL]
    assert not bad, bad[:10]
    return max(e for _, e in res)


def _read_rows(plan, w, layer, seq, kv, t0, t1):
    """Packed rows [t1-t0] of every kv head: list of (codes [n][cb], scales [n][sb/2] uint16)."""
    n = t1 - t0
    cbs = [plan.row_bytes(layer, h, kv) for h in range(w.n_kv_heads)]
    codes = torch.zeros(max(sum(c for c, _ in cbs) * n, 1), dtype=torch.uint8, device="cuda")
    scales = torch.zeros(max(sum(s for _, s in cbs) * n, 2), dtype=torch.uint8, device="cuda")
    plan.read_rows(layer, seq, t0, t1, kv, codes, scales)
    torch.cuda.synchronize()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    out, co, so = [], 0, 0
    for cb, sb in cbs:
        c = codes[co:co + cb * n].reshape(n, cb)
        s = scales[so:so + sb * n].reshape(n, sb).copy().view(np.uint16) if sb else np.zeros((n, 0), np.uint16)
        out.append((c, s))
        co += cb * n
        so += sb * n
    return out


def _check_packed_rows(plan, w, cells, runs=((0, 64), (0.5, 64), (1.0, 64))):
    """Runs of packed rows (start of the quantized range, its middle, its end) of the
    cells' (layer, seq, head), K and V, equal the oracle's encoding bit for bit."""
    checked = 0
    for (l, s, h) in cells:
        nq = max(0, w.ctx[s] - w.tail)
        if nq == 0:
            continue
        K, V = _history(w, l, s, nq)
        hp = H.head_params(w, l, h)
        for frac, n in runs:
            t0 = min(max(0, int(frac * nq) - (n if frac > 0 else 0)), max(0, nq - n))
            t1 = min(nq, t0 + n)
            for kv, X in ((0, K), (1, V)):
                gc, gs = _read_rows(plan, w, l, s, kv, t0, t1)[h]
                x = X[t0:t1, h, :]
                if w.rot == W.ROT_PROJECTION:
                    b = hp["kb"] if kv == 0 else hp["vb"]
                    oc, os_ = oracle.encode_rows(W.RANK, w.rot, x, M=hp["M"], r=hp["r"], b=b)
                else:
                    codec = hp["k_codec"] if kv == 0 else hp["v_codec"]
                    inv = hp.get("inv_s_k" if kv == 0 else "inv_s_v")
                    oc, os_ = oracle.encode_rows(codec, w.rot, x, inv_s=inv)
                assert np.array_equal(gc, oc), (l, s, h, kv, t0)
                assert np.array_equal(gs, os_), (l, s, h, kv, t0)
                checked += t1 - t0
    assert checked > 0


def test_llama8b_shape_full():
    """32 layers x 32k, K q8_0 / V q4_0 (the Llama-3.1-8B-shaped workload): every layer
    of the sequence, two kv heads per layer (all eight heads over four layers)."""
    w = W.make_workload(2, "full")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=4096)
    outs = _decode_all(plan, w, range(w.n_layers), [0])
    cells = [(l, 0, (2 * l + k) % w.n_kv_heads) for l in range(w.n_layers) for k in range(2)]
    _check_cells(w, outs, cells, [0])
    _check_packed_rows(plan, w, [(l, 0, h) for (l, _, h) in cells[::8]])


def test_vbr_mix_full():
    """64 layers x 64k, tail 1024, every codec band of the VBR map: every layer."""
    w = W.make_workload(3, "full")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=8192)
    outs = _decode_all(plan, w, range(w.n_layers), [0])
    cells = [(l, 0, l % w.n_kv_heads) for l in range(w.n_layers)]
    _check_cells(w, outs, cells, [0])
    _check_packed_rows(plan, w, [(l, 0, l % w.n_kv_heads) for l in (0, 7, 20, 40, 63)])


def test_cobra_rank_bits_full():
    """256 heads with per-head (r, b), 128k tokens, per-head projection: every layer,
    on the workload's own rows."""
    w = W.make_workload(4, "full")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=8192)
    outs = _decode_all(plan, w, range(w.n_layers), [0])
    cells = [(l, 0, (3 * l) % w.n_kv_heads) for l in range(w.n_layers)]
    _check_cells(w, outs, cells, [0])
    _check_packed_rows(plan, w, [(l, 0, h) for (l, _, h) in cells[::6]], runs=((0, 64), (1.0, 64)))


def test_batched_kvarn_full():
    """64 ragged sequences, varnorm + H + q4_0, tail 256, then a 2048-token chunk
    appended to 8 sequences (the bench's serving step) before decoding: 40 cells
    over both checked layers, the grown sequences among them."""
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
    layers = [0, 13, 31]
    outs = _decode_all(plan, w, layers, seqs)
    cells = [(layers[i % 3], (5 * i + 3) % 64, i % w.n_kv_heads) for i in range(36)]
    cells += [(31, s, s % w.n_kv_heads) for s in grown[:4]]
    _check_cells(w, outs, cells, seqs)
    _check_packed_rows(plan, w, [(l, seqs[si], h) for (l, si, h) in cells[::9]])
