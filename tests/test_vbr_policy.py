"""VBR policy step (host code; "Introducing a new KV format: VBR (Variable Bit
Rate)": quantize layer by layer as the session grows, within --vbr-vram, above
--vbr-floor).  Ladder F16 > q8_0 > q6_0 > q4_1 > q2_1, V on a rung and K one rung
richer, the deepest layer on the richest rung moves first."""
import pytest

from quantized_kv_cache_15_b200 import kvq
from quantized_kv_cache_15_b200 import workloads as W

LADDER = [W.F16, W.Q8_0, W.Q6_0, W.Q4_1, W.Q2_1]


def _bytes(k, v):
    """Bytes of a toy cache: per layer and head, packed K + V row bytes."""
    rb = {W.F16: 256, W.Q8_0: 136, W.Q6_0: 104, W.Q4_1: 80, W.Q2_1: 48}
    return int(sum(rb[a] + rb[b] for ra, rb_ in zip(k, v) for a, b in zip(ra, rb_)))


def test_within_budget_does_nothing():
    k = [[W.F16] * 2] * 4
    assert kvq.vbr_next(k, k, 100, 100, W.Q2_1)[0] == -1


def test_first_steps_take_the_deepest_layers_one_rung_down():
    k = [[W.F16] * 2 for _ in range(4)]
    v = [[W.F16] * 2 for _ in range(4)]
    layer, nk, nv = kvq.vbr_next(k, v, 2, 1, W.Q2_1)
    assert (layer, nk, nv) == (3, [W.F16] * 2, [W.Q8_0] * 2)
    k[3], v[3] = nk, nv
    layer, nk, nv = kvq.vbr_next(k, v, 2, 1, W.Q2_1)
    assert (layer, nk, nv) == (2, [W.F16] * 2, [W.Q8_0] * 2)


def test_descent_to_a_budget_keeps_k_one_rung_richer_and_respects_the_floor():
    L, H = 6, 2
    k = [[W.F16] * H for _ in range(L)]
    v = [[W.F16] * H for _ in range(L)]
    budget = _bytes(k, v) // 3
    steps = 0
    while True:
        layer, nk, nv = kvq.vbr_next(k, v, _bytes(k, v), budget, W.Q4_1)
        if layer < 0:
            break
        k[layer], v[layer] = nk, nv
        steps += 1
        assert steps < 100
    for l in range(L):
        rv, rk = LADDER.index(v[l][0]), LADDER.index(k[l][0])
        assert rv <= LADDER.index(W.Q4_1)                       # floor
        assert rk == max(0, rv - 1)                             # K one rung richer
    # rungs never increase with depth (deeper layers are never richer)
    rungs = [LADDER.index(v[l][0]) for l in range(L)]
    assert all(a <= b for a, b in zip(rungs, rungs[1:]))
    # either within budget or every layer at the floor
    assert _bytes(k, v) <= budget or all(r == LADDER.index(W.Q4_1) for r in rungs)


def test_every_layer_at_the_floor_stops():
    k = [[W.Q6_0] * 2] * 3
    v = [[W.Q4_1] * 2] * 3
    assert kvq.vbr_next(k, v, 10, 1, W.Q4_1)[0] == -1


def test_codecs_off_the_ladder_are_rejected():
    with pytest.raises(kvq.KVQError):
        kvq.vbr_next([[W.Q4_0] * 2], [[W.Q4_0] * 2], 10, 1, W.Q2_1)
