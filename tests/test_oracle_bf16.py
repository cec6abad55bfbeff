"""BF16 raw rows in the oracle (BeeLlama v0.4.0 news, §KV cache 精度尾部: the newest
tokens may be kept in BF16 or F16).

Pins: the bf16 -> fp32 widening against torch's conversion on every bit pattern;
the bf16 input path of the encoder against its fp16 input path on values both
formats hold exactly (two independent conversions, one transform and quantizer);
attention over a bf16 tail that covers the whole context against brute-force
softmax attention in numpy.
"""
import numpy as np
import pytest
import torch

import oracle

D = 128


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f16_bits(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(x, np.float32).astype(np.float16).view(np.uint16)


def test_bf16_widening_matches_torch_on_every_pattern():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f32(h)
    ref = torch.from_numpy(h.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


@pytest.mark.parametrize("codec", [oracle.Q8_0, oracle.Q4_0, oracle.Q6_1, oracle.Q3_0, oracle.Q2_1])
@pytest.mark.parametrize("rot", [oracle.ROT_HADAMARD, oracle.ROT_VARNORM_HADAMARD])
def test_bf16_and_fp16_inputs_encode_alike_on_common_values(codec, rot):
    rng = np.random.default_rng(codec * 10 + rot)
    # integers |k| <= 255 times 2^-6: exact in fp16 (11-bit significand) and in bf16 (8-bit)
    x = rng.integers(-255, 256, size=(64, D)).astype(np.float32) * np.float32(2.0 ** -6)
    inv = rng.uniform(0.5, 2.0, D).astype(np.float32) if rot == oracle.ROT_VARNORM_HADAMARD else None
    a = oracle.encode_rows(codec, rot, _bf16_bits(x), inv_s=inv, bf16=True)
    b = oracle.encode_rows(codec, rot, _f16_bits(x), inv_s=inv)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    ya = oracle.to_stored_basis(codec, rot, _bf16_bits(x), inv_s=inv, bf16=True)
    yb = oracle.to_stored_basis(codec, rot, _f16_bits(x), inv_s=inv)
    assert np.array_equal(ya.view(np.uint32), yb.view(np.uint32))


def test_bf16_tail_covering_the_context_is_plain_attention():
    rng = np.random.default_rng(7)
    n, G = 40, 3
    K = _bf16_bits(rng.standard_normal((n, D)))
    V = _bf16_bits(rng.standard_normal((n, D)))
    q = _bf16_bits(rng.standard_normal((G, D)))
    out = oracle.decode_head(K, V, q, oracle.Q4_0, oracle.Q4_0, oracle.ROT_HADAMARD, tail=64, bf16=True)
    Kf, Vf, qf = (oracle.bf16_to_f32(a).astype(np.float64) for a in (K, V, q))
    scale = float(np.float32(1.0 / np.sqrt(D)))
    for g in range(G):
        s = Kf @ qf[g] * scale
        p = np.exp(s - s.max())
        ref = (p @ Vf) / p.sum()
        assert np.abs(out[g] - ref).max() <= 1e-6 * np.abs(ref).max()


def test_bf16_plans_reject_the_projection_path():
    from quantized_kv_cache_15_b200 import kvq
    n = 1
    with pytest.raises(kvq.KVQError) as e:
        kvq.Plan(1, 1, 1, max_seqs=1, max_tokens_per_seq=64, k_codec=[kvq.RANK], v_codec=[kvq.RANK],
                 rot=kvq.ROT_PROJECTION, rank=[16] * n, k_bits=[1] * n, v_bits=[1] * n,
                 proj_basis=[np.eye(D)[:, :16]], kv_dtype=kvq.KV_BF16)
    assert e.value.status == 2
