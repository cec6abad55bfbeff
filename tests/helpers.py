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
