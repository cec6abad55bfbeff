"""Micro-benchmarks of the CUDA-core pipes and of a streaming read through the
C ABI (kvq_microbench): the ceilings that decode attention on CUDA cores is
measured against.  Prints one line per kind (run with -s to see them):

    ubench <kind> <rate> <unit> (<work> in <ms> ms, <ctas> CTAs)

and checks that each rate is plausible for a B200 (well above what a wrong
launch or an optimised-away loop would give, below the hardware's nominal rate).
"""
import pytest
import torch

from quantized_kv_cache_15_b200 import kvq

pytestmark = pytest.mark.gpu

# nominal B200 ceilings at the 1965 MHz maximum clock: 148 SMs x 128 fp32 lanes
NOMINAL_FMA_PER_S = 148 * 128 * 1.965e9


def _time(kind, iters, ctas, sink, buf=None):
    st = torch.cuda.current_stream()
    kvq.microbench(kind, iters, ctas, sink, buf)                 # warm-up
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    work = kvq.microbench(kind, iters, ctas, sink, buf)
    b.record(st)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    return work, ms


@pytest.mark.parametrize("kind,name,lo", [
    (kvq.UB_FFMA, "ffma", 0.25), (kvq.UB_DP2A, "dp2a", 0.2), (kvq.UB_DP4A, "dp4a", 0.2),
    (kvq.UB_FMA2, "fma.rn.f32x2", 0.2), (kvq.UB_MIX, "dp2a+ffma", 0.2)])
def test_alu_rates(kind, name, lo):
    ctas = 148 * 8
    sink = torch.zeros(ctas * 256, dtype=torch.int64, device="cuda")
    work, ms = _time(kind, 4096, ctas, sink)
    rate = work / (ms / 1e3)
    print(f"ubench {name} {rate / 1e12:.2f} Tmul-add/s ({work:.3e} in {ms:.3f} ms, {ctas} CTAs)")
    assert lo * NOMINAL_FMA_PER_S < rate < 8 * NOMINAL_FMA_PER_S


def test_streaming_read_rate():
    buf = torch.empty(4 << 30, dtype=torch.uint8, device="cuda").fill_(1)   # 4 GiB, far beyond L2
    ctas = 148 * 8
    sink = torch.zeros(ctas * 256, dtype=torch.int64, device="cuda")
    work, ms = _time(kvq.UB_READ, 1, ctas, sink, buf)
    rate = work / (ms / 1e3)
    print(f"ubench read {rate / 1e9:.1f} GB/s ({work:.3e} B in {ms:.3f} ms, {ctas} CTAs)")
    assert 2.0e12 < rate < 9.0e12


def test_microbench_rejects_bad_arguments():
    sink = torch.zeros(256, dtype=torch.int64, device="cuda")
    for args in ((9, 1, 1), (kvq.UB_FFMA, 0, 1), (kvq.UB_FFMA, 1, 0)):
        with pytest.raises(kvq.KVQError):
            kvq.microbench(*args, sink)
    with pytest.raises(kvq.KVQError):
        kvq.microbench(kvq.UB_READ, 1, 1, sink, None)
