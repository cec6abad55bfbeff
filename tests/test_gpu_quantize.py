"""GPU quantizer, rotation and calibration against the oracle: bit-exact.

The block quantizers (BeeLlama v0.4.0 news, §新增标准 KV cache 类型; KV-COBRA
explainer, §Jargon) and the staged Hadamard transform are sequences of
correctly rounded fp32 operations in a fixed order, so the GPU's codes, scales
and rotated values must equal the oracle's bit for bit on the same inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

CODECS = [kvq.Q8_0, kvq.Q6_0, kvq.Q5_0, kvq.Q4_0, kvq.Q3_0, kvq.Q2_0, kvq.Q8_1, kvq.Q6_1, kvq.Q5_1, kvq.Q4_1,
          kvq.Q3_1, kvq.Q2_1, kvq.F16]


def _rows(seed, n, width=128):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((n, width)) * rng.uniform(1e-3, 50, (n, 1))
    y[::5] += rng.uniform(-30, 30, (len(y[::5]), 1))
    y[::7, :32] = 0.0                                  # all-zero block
    y[::9] = np.round(y[::9] * 2) / 2                  # many exact ties
    y[3] = 0.0
    y[4, 5] = 1e6                                      # scale clamp at 65504
    y[6, :] = -70000.0                                 # _1 minimum below the fp16 range
    y[8] = np.float32(1e-30)                           # fp16 underflow of the scale
    return y.astype(np.float32)


def _gpu_quantize(codec, y, r=128, b=0, layout=kvq.ROWS_WARP):
    cb, sb = oracle.row_bytes(codec, r, b)
    yd = torch.from_numpy(y).cuda()
    codes = torch.zeros((y.shape[0], cb), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((y.shape[0], max(sb, 2)), dtype=torch.uint8, device="cuda")
    kvq.debug_quantize_f32(codec, r, b, yd, codes, scales, layout)
    torch.cuda.synchronize()
    sc = scales.cpu().numpy()[:, :sb].copy().view(np.uint16) if sb else np.zeros((y.shape[0], 0), np.uint16)
    return codes.cpu().numpy(), sc


@pytest.mark.parametrize("layout", [kvq.ROWS_WARP, kvq.ROWS_QUAD])
@pytest.mark.parametrize("codec", CODECS)
def test_block_quantizer_bit_exact(codec, layout):
    """Both row layouts (a warp per row; four threads per row) against the oracle."""
    y = _rows(codec, 3000)
    if codec == kvq.F16:
        y = y.astype(np.float16).astype(np.float32)
    gc, gs = _gpu_quantize(codec, y, layout=layout)
    oc, os_ = oracle.quantize_rows(codec, y)
    assert np.array_equal(gc, oc)
    assert np.array_equal(gs, os_)


@pytest.mark.parametrize("r", [16, 32, 64, 96, 128])
@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_rank_quantizer_bit_exact(r, b):
    y = _rows(100 * r + b, 1000, width=r)
    gc, gs = _gpu_quantize(kvq.RANK, y, r, b)
    oc, os_ = oracle.quantize_rows(kvq.RANK, y, r=r, b=b)
    assert np.array_equal(gc, oc)
    assert np.array_equal(gs, os_)


@pytest.mark.parametrize("layout", [kvq.ROWS_WARP, kvq.ROWS_QUAD])
@pytest.mark.parametrize("rot", [W.ROT_HADAMARD, W.ROT_VARNORM_HADAMARD])
def test_rotation_bit_exact(rot, layout):
    w = W.make_workload(5 if rot == W.ROT_VARNORM_HADAMARD else 1, "small")
    w.rot = rot
    plan = H.make_plan(w)
    x = w.rows("K", 0, 0, 0, 700)[:, 1, :].contiguous()
    inv = H.gpu_inv_rms(w)[0, 1, 0] if rot == W.ROT_VARNORM_HADAMARD else None
    for kv in (0, 1):
        y = torch.empty((700, 128), dtype=torch.float32, device="cuda")
        plan.debug_rotate(0, 1, kv, x.cuda(), y, layout)
        torch.cuda.synchronize()
        invk = None
        if inv is not None:
            invk = H.gpu_inv_rms(w)[0, 1, kv]
        ref = oracle.to_stored_basis(w.k_codec[0][1], rot, H.f16_bits(x), inv_s=invk)
        assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_projection_bit_exact():
    """z = M_h x as the plan's projection kernel forms it equals the oracle's double
    sum in channel order, rounded to fp32, bit for bit (both K and V, every head, r in
    {16, 32, 64, 96, 128} across the workload's heads)."""
    w = W.make_workload(4, "small")
    plan = H.make_plan(w)
    rs = set()
    for l in range(w.n_layers):
        for h in range(w.n_kv_heads):
            r = w.rank[l][h]
            rs.add(r)
            M = oracle.fuse_projection(w.proj_basis(l, h))
            for kv, kind in enumerate("KV"):
                x = w.rows(kind, l, 0, 0, 300)[:, h, :].contiguous()
                y = torch.empty((300, r), dtype=torch.float32, device="cuda")
                plan.debug_rotate(l, h, kv, x.cuda(), y)
                torch.cuda.synchronize()
                ref = oracle.to_stored_basis(kvq.RANK, W.ROT_PROJECTION, H.f16_bits(x), M=M, r=r)
                assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32)), (l, h, kv, r)
    assert len(rs) >= 3


def test_calibration_bit_exact():
    w = W.make_workload(5, "small")
    g = H.gpu_inv_rms(w)
    for l in range(w.n_layers):
        for h in range(w.n_kv_heads):
            for kv, kind in enumerate("KV"):
                assert np.array_equal(g[l, h, kv], H.oracle_inv_rms(w, l, h, kind))
