"""VBR regrade through the C ABI against the oracle ("Introducing a new KV format:
VBR (Variable Bit Rate)", first post: the cache is requantized layer by layer as
the session grows).

Every layer of the VBR-mix workload moves one step down the ladder F16 > q8_0 >
q6_0 > q4_1 > q2_1.  The regraded packed rows must equal the oracle's regrade of
its own packed rows bit for bit; decode over the regraded cache, and over the cache
after more appends (new rows quantized with the new codecs), must match the
oracle within the 2e-3 bar."""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

LADDER = [W.F16, W.Q8_0, W.Q6_0, W.Q4_1, W.Q2_1]


def _down(c):
    return LADDER[min(LADDER.index(c) + 1, len(LADDER) - 1)]


def _read(plan, w, layer, kv, nq):
    cbs = [plan.row_bytes(layer, h, kv) for h in range(w.n_kv_heads)]
    codes = torch.zeros(max(sum(c for c, _ in cbs) * nq, 1), dtype=torch.uint8, device="cuda")
    scales = torch.zeros(max(sum(s for _, s in cbs) * nq, 2), dtype=torch.uint8, device="cuda")
    plan.read_rows(layer, 0, 0, nq, kv, codes, scales)
    torch.cuda.synchronize()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    out, co, so = [], 0, 0
    for cb, sb in cbs:
        out.append((codes[co:co + cb * nq].reshape(nq, cb),
                    scales[so:so + sb * nq].reshape(nq, sb).copy().view(np.uint16) if sb else
                    np.zeros((nq, 0), np.uint16)))
        co += cb * nq
        so += sb * nq
    return out


def _oracle_rows(w, layer, kind, head, old, new, n_old_q, n_new_q):
    """Oracle packed rows of the regraded cache: rows below the old tail regraded,
    rows that left the tail afterwards encoded with the new codec."""
    hist = H.f16_bits(w.rows(kind, layer, 0, 0, n_new_q)[:, head, :])
    inv = H.head_params(w, layer, head).get("inv_s_k" if kind == "K" else "inv_s_v")
    c0, s0 = oracle.encode_rows(old, w.rot, hist[:n_old_q], inv_s=inv)
    c1, s1 = oracle.regrade_rows(old, new, w.rot, c0, s0, inv_s=inv)
    if n_new_q > n_old_q:
        c2, s2 = oracle.encode_rows(new, w.rot, hist[n_old_q:n_new_q], inv_s=inv)
        c1, s1 = np.concatenate([c1, c2]), np.concatenate([s1, s2])
    return c1, s1


def _check_decode(plan, w, new_k, new_v, n, old_codecs, n_old_q):
    ws = plan.new_workspace(1)
    nq = n - w.tail
    for l in range(w.n_layers):
        q = w.queries(l, 0, 5, "cuda").unsqueeze(0).contiguous()
        out = torch.empty((1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
        plan.decode(l, [0], q, out, ws)
        torch.cuda.synchronize()
        out = out.cpu().numpy()[0]
        for h in range(w.n_kv_heads):
            ok, ov = old_codecs[l][h]
            ck, sk = _oracle_rows(w, l, "K", h, ok, new_k[l][h], n_old_q, nq)
            cv, sv = _oracle_rows(w, l, "V", h, ov, new_v[l][h], n_old_q, nq)
            Kt = H.f16_bits(w.rows("K", l, 0, nq, n)[:, h, :])
            Vt = H.f16_bits(w.rows("V", l, 0, nq, n)[:, h, :])
            args = H.head_params(w, l, h)
            qh = H.f16_bits(q[0, h * w.G:(h + 1) * w.G])
            ref = oracle.decode_packed(ck, sk, cv, sv, Kt, Vt, qh, new_k[l][h], new_v[l][h], w.rot,
                                       inv_s_k=args.get("inv_s_k"), inv_s_v=args.get("inv_s_v"))
            err = H.rel_err_rows(out[h * w.G:(h + 1) * w.G], ref)
            assert err.max() <= H.TOL, (l, h, err.max())


@pytest.mark.parametrize("rot", [W.ROT_HADAMARD, W.ROT_VARNORM_HADAMARD])
def test_regrade_one_step_down_the_ladder(rot):
    w = W.make_workload(3, "small")
    w.rot = rot
    plan = H.make_plan(w, extra_tokens=300)
    H.fill(plan, w, chunk=700)
    n = w.ctx[0]
    nq = n - w.tail
    old = [[(w.k_codec[l][h], w.v_codec[l][h]) for h in range(w.n_kv_heads)] for l in range(w.n_layers)]
    new_k = [[_down(c) for c in row] for row in w.k_codec]
    new_v = [[_down(c) for c in row] for row in w.v_codec]
    for l in range(w.n_layers):
        scratch = torch.empty(plan.regrade_bytes(l, new_k[l], new_v[l]), dtype=torch.uint8, device="cuda")
        plan.regrade(l, new_k[l], new_v[l], scratch)
    torch.cuda.synchronize()
    plan.check_device_error()
    # packed rows bit for bit
    for l in range(w.n_layers):
        for kv, kind in enumerate("KV"):
            rows = _read(plan, w, l, kv, nq)
            for h in range(w.n_kv_heads):
                o, nw = old[l][h][kv], (new_k if kv == 0 else new_v)[l][h]
                oc, os_ = _oracle_rows(w, l, kind, h, o, nw, nq, nq)
                gc, gs = rows[h]
                assert np.array_equal(gc, oc), (l, kind, h)
                assert np.array_equal(gs, os_), (l, kind, h)
    _check_decode(plan, w, new_k, new_v, n, old, nq)
    # later appends quantize with the new codecs
    for l in range(w.n_layers):
        plan.append(l, [0], [300], w.rows("K", l, 0, n, n + 300, "cuda"), w.rows("V", l, 0, n, n + 300, "cuda"))
    torch.cuda.synchronize()
    _check_decode(plan, w, new_k, new_v, n + 300, old, nq)


def test_regrade_rejects_growth_and_dequantized_f16():
    w = W.make_workload(3, "small")
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=700)
    with pytest.raises(kvq.KVQError) as e:                      # q4_1 -> q8_0 grows the pages
        plan.regrade_bytes(3, [W.Q8_0] * 4, [W.Q8_0] * 4)
    assert e.value.status == 3
    with pytest.raises(kvq.KVQError):                           # a quantized row cannot become F16
        plan.regrade_bytes(2, [W.F16] * 4, [W.Q6_0] * 4)


def test_vbr_policy_drives_regrades_to_a_budget():
    """An all-F16 cache regraded by the policy step until it fits a budget (or every
    layer reaches the floor); decode then matches the oracle over the same chain of
    regrades."""
    w = W.make_workload(3, "small")
    w.k_codec = [[W.F16] * w.n_kv_heads for _ in range(w.n_layers)]
    w.v_codec = [[W.F16] * w.n_kv_heads for _ in range(w.n_layers)]
    plan = H.make_plan(w)
    H.fill(plan, w, chunk=700)
    start = plan.bytes_in_use()
    tail_bytes = w.batch * w.n_layers * w.n_kv_heads * w.tail * 512
    budget = tail_bytes + (start - tail_bytes) * 45 // 100
    k = [row[:] for row in w.k_codec]
    v = [row[:] for row in w.v_codec]
    history = [[] for _ in range(w.n_layers)]           # (old K, old V, new K, new V) per step
    for _ in range(40):
        layer, nk, nv = kvq.vbr_next(k, v, plan.bytes_in_use(), budget, W.Q2_1)
        if layer < 0:
            break
        scratch = torch.empty(plan.regrade_bytes(layer, nk, nv), dtype=torch.uint8, device="cuda")
        plan.regrade(layer, nk, nv, scratch)
        history[layer].append((k[layer][0], v[layer][0], nk[0], nv[0]))
        k[layer], v[layer] = nk, nv
    torch.cuda.synchronize()
    plan.check_device_error()
    assert plan.bytes_in_use() <= budget
    assert any(history)
    n = w.ctx[0]
    nq = n - w.tail
    ws = plan.new_workspace(1)
    for l in range(w.n_layers):
        q = w.queries(l, 0, 2, "cuda").unsqueeze(0).contiguous()
        out = torch.empty((1, w.n_q_heads, 128), dtype=torch.float32, device="cuda")
        plan.decode(l, [0], q, out, ws)
        torch.cuda.synchronize()
        out = out.cpu().numpy()[0]
        for h in range(w.n_kv_heads):
            packed = []
            for kv, kind in enumerate("KV"):
                hist = H.f16_bits(w.rows(kind, l, 0, 0, nq)[:, h, :])
                c, s = oracle.encode_rows(W.F16, w.rot, hist)
                for step in history[l]:
                    c, s = oracle.regrade_rows(step[kv], step[2 + kv], w.rot, c, s)
                packed += [c, s]
            Kt = H.f16_bits(w.rows("K", l, 0, nq, n)[:, h, :])
            Vt = H.f16_bits(w.rows("V", l, 0, nq, n)[:, h, :])
            qh = H.f16_bits(q[0, h * w.G:(h + 1) * w.G])
            ref = oracle.decode_packed(*packed, Kt, Vt, qh, k[l][h], v[l][h], w.rot)
            err = H.rel_err_rows(out[h * w.G:(h + 1) * w.G], ref)
            assert err.max() <= H.TOL, (l, h, err.max())
