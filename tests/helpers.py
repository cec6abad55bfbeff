"""Test helpers: build a kvq plan for a workload, fill it through the C ABI, and
compute the oracle's expectation for the same seeded inputs.

The product side runs only through quantized_kv_cache_15_b200.kvq (the C ABI);
the expectation side runs only through the oracle package.  Both draw their
inputs from quantized_kv_cache_15_b200.workloads, which holds no arithmetic of
the method.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W

D = 128
TOL = 2e-3          # max_j |o - o*| <= TOL * max_j |o*| per (sequence, query head) row


def f16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_inv_rms(w: W.Workload, layer: int, head: int, kind: str) -> np.ndarray:
    calib = w.calib_rows(kind, layer, 512)[:, head, :]
    return oracle.varnorm_inv_rms(f16_bits(calib))


def gpu_inv_rms(w: W.Workload) -> np.ndarray:
    """[L][Hkv][2][128] via the library's calibration kernel."""
    out = np.zeros((w.n_layers, w.n_kv_heads, 2, D), np.float32)
    for l in range(w.n_layers):
        for kv, kind in enumerate("KV"):
            x = w.calib_rows(kind, l, 512, device="cuda").reshape(512, w.n_kv_heads * D).contiguous()
            inv = torch.empty(w.n_kv_heads * D, dtype=torch.float32, device="cuda")
            kvq.calibrate_varnorm(x, w.n_kv_heads * D, w.n_kv_heads * D, inv)
            out[l, :, kv, :] = inv.cpu().numpy().reshape(w.n_kv_heads, D)
    return out


def make_plan(w: W.Workload, extra_tokens: int = 0, max_pages: int = 0, inv_rms=None) -> kvq.Plan:
    kc = np.array(w.k_codec, np.int32)
    vc = np.array(w.v_codec, np.int32)
    kwargs = {}
    if w.rot == W.ROT_VARNORM_HADAMARD:
        kwargs["inv_rms"] = gpu_inv_rms(w) if inv_rms is None else inv_rms
    if w.rot == W.ROT_PROJECTION:
        kwargs["rank"] = np.array(w.rank, np.int32)
        kwargs["k_bits"] = np.array(w.k_bits, np.int32)
        kwargs["v_bits"] = np.array(w.v_bits, np.int32)
        kwargs["proj_basis"] = [w.proj_basis(l, h) for l in range(w.n_layers) for h in range(w.n_kv_heads)]
    plan = kvq.Plan(w.n_layers, w.n_q_heads, w.n_kv_heads, max_seqs=w.batch,
                    max_tokens_per_seq=max(w.ctx) + extra_tokens, k_codec=kc, v_codec=vc, rot=w.rot,
                    tail_tokens=w.tail, max_pages=max_pages, **kwargs)
    plan.allocate_cache()
    return plan


def fill(plan: kvq.Plan, w: W.Workload, chunk: int = 2048, seqs=None, layers=None):
    """Append every sequence's context, layer by layer, in chunks."""
    seqs = range(w.batch) if seqs is None else seqs
    layers = range(w.n_layers) if layers is None else layers
    for l in layers:
        for s in seqs:
            t = 0
            while t < w.ctx[s]:
                n = min(chunk, w.ctx[s] - t)
                k = w.rows("K", l, s, t, t + n, device="cuda")
                v = w.rows("V", l, s, t, t + n, device="cuda")
                plan.append(l, [s], [n], k, v)
                t += n
    torch.cuda.synchronize()


def head_params(w: W.Workload, layer: int, head: int, inv_rms=None):
    """Codec / transform arguments of one (layer, kv head) for the oracle."""
    kc, vc = w.k_codec[layer][head], w.v_codec[layer][head]
    args = dict(k_codec=kc, v_codec=vc, rot=w.rot, tail=w.tail)
    if w.rot == W.ROT_PROJECTION:
        r = w.rank[layer][head]
        args.update(r=r, kb=w.k_bits[layer][head], vb=w.v_bits[layer][head],
                    M=oracle.fuse_projection(w.proj_basis(layer, head)))
    if w.rot == W.ROT_VARNORM_HADAMARD:
        args.update(inv_s_k=oracle_inv_rms(w, layer, head, "K"), inv_s_v=oracle_inv_rms(w, layer, head, "V"))
    return args


def oracle_decode(w: W.Workload, layer: int, seq: int, head: int, q_f16: np.ndarray, length=None) -> np.ndarray:
    """Oracle output [G][128] for one (layer, seq, kv head); q_f16: uint16 [G][128]."""
    n = w.ctx[seq] if length is None else length
    K = f16_bits(w.rows("K", layer, seq, 0, n)[:, head, :])
    V = f16_bits(w.rows("V", layer, seq, 0, n)[:, head, :])
    return oracle.decode_head(K, V, q_f16, **head_params(w, layer, head))


def rel_err_rows(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per-row relative error max_j |got - ref| / max_j |ref| (rows = last axis)."""
    num = np.abs(got.astype(np.float64) - ref.astype(np.float64)).max(axis=-1)
    den = np.abs(ref.astype(np.float64)).max(axis=-1)
    return num / np.maximum(den, 1e-30)


# ----------------------------------------------------------------------------- projection decisions
# KV-COBRA explainer, §Jargon "Scalar quantization": a block's step is
# d = fp16(max|z| / (2^(b-1) - 1/2)) and a value's level is floor(z / d).  Both are
# integer decisions taken on the projection z = M x.  The kernel forms z on the tensor
# cores (exact fp16 x fp16 products of x and the hi/lo halves of M, fp32 accumulation
# over 256 products); the oracle accumulates in double.  Their difference is bounded
# per value by PROJ_EPS * sum_c |x_c| |M_rc|: with unit roundoff u = 2^-24 and n = 256
# products the probabilistic bound of fp32 summation (Higham and Mary 2019,
# lambda * sqrt(n) * u with lambda = 3) is 2.9e-6; the hi/lo residual of M
# (2^-22 relative) and one ulp of M's own rounding add less than 3e-7.
PROJ_EPS = 3.2e-6


def projection_error_bound(x_f16: np.ndarray, M: np.ndarray) -> np.ndarray:
    """[n][r] bound on |z_kernel - z_oracle| for fp16 rows x [n][128] and M [r][128]."""
    x = oracle.f16_to_f32(x_f16).astype(np.float64)
    return PROJ_EPS * (np.abs(x) @ np.abs(M.astype(np.float64)).T)


def projection_ambiguous_rows(x_f16: np.ndarray, M: np.ndarray, r: int, b: int) -> np.ndarray:
    """Boolean [n]: rows with a block step or a level that the oracle places within
    the projection error bound of a decision boundary (an fp16 rounding midpoint of
    the step, an integer multiple of the step).  Such a row has more than one valid
    encoding; every other row has exactly one."""
    z = oracle.to_stored_basis(kvq.RANK, W.ROT_PROJECTION, x_f16, M=M, r=r)
    _, sc = oracle.quantize_rows(kvq.RANK, z, r=r, b=b)
    eps = projection_error_bound(x_f16, M)
    n = z.shape[0]
    blk = min(r, 32)
    nb = r // blk
    zb = z.astype(np.float64).reshape(n, nb, blk)
    eb = eps.reshape(n, nb, blk)
    L = float((1 << (b - 1)) - 0.5)
    # step decision: fp16 rounding of amax / L (amax moves by at most the largest bound)
    amax = np.abs(zb).max(axis=-1)
    a = (np.float32(1.0) * (amax.astype(np.float32) / np.float32(L))).astype(np.float64)
    hb = oracle.f16_rn(a.astype(np.float32)).astype(np.int64)
    v = oracle.f16_to_f32(hb.astype(np.uint16)).astype(np.float64)
    prev = oracle.f16_to_f32(np.maximum(hb - 1, 0).astype(np.uint16)).astype(np.float64)
    nxt = oracle.f16_to_f32(np.minimum(hb + 1, 0x7BFF).astype(np.uint16)).astype(np.float64)
    dist = np.minimum(np.where(hb > 0, np.abs(a - (prev + v) / 2), np.inf), np.abs(a - (v + nxt) / 2))
    slack = eb.max(axis=-1) / L + a * 2.0 ** -22
    amb = (dist <= slack) & (amax > 0)
    # level decisions: z / d against the integers
    df = oracle.f16_to_f32(sc).astype(np.float64).reshape(n, nb)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = zb / df[..., None]
        near = np.abs(t - np.round(t)) <= eb / df[..., None] + np.abs(t) * 2.0 ** -22
    near &= (df > 0)[..., None]
    amb |= near.any(axis=-1)
    return amb.any(axis=-1)
