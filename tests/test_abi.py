"""The C-ABI library loads and exports every entry point include/kvq.h declares
(no compute calls: this runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def libkvq():
    from quantized_kv_cache_15_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_four_core_entry_points():
    names = declared_functions()
    for n in ("kvq_plan_create", "kvq_append_quantize", "kvq_decode_attention", "kvq_dequantize"):
        assert n in names


def test_every_declared_symbol_is_exported(libkvq):
    missing = [n for n in declared_functions() if not hasattr(libkvq, n)]
    assert not missing, missing


def test_binding_covers_the_header():
    from quantized_kv_cache_15_b200 import kvq
    assert set(declared_functions()) == set(kvq.SIGNATURES)


def test_last_error_is_callable_without_gpu(libkvq):
    libkvq.kvq_last_error.restype = ctypes.c_char_p
    assert libkvq.kvq_last_error() == b""


def test_library_links_no_oracle_and_no_torch():
    """The product library is standalone CUDA: no oracle or PyTorch symbols."""
    import subprocess
    from quantized_kv_cache_15_b200 import build
    path = build.build()
    out = subprocess.run(["nm", "-D", "--undefined-only", path], capture_output=True, text=True).stdout
    assert "orc_" not in out and "torch" not in out and "c10" not in out
    deps = subprocess.run(["ldd", path], capture_output=True, text=True).stdout
    assert "liboracle" not in deps and "libtorch" not in deps


def test_debug_quantize_rejects_bad_row_layouts_before_any_launch(libkvq):
    """Argument checks run on the host: no device is touched."""
    from quantized_kv_cache_15_b200 import kvq
    f = libkvq.kvq_debug_quantize_f32
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    fake = ctypes.c_void_p(16)
    assert f(kvq.RANK, 64, 2, 1, fake, fake, fake, kvq.ROWS_QUAD, None) == 2       # KVQ_ERR_UNSUPPORTED
    assert f(kvq.Q4_0, 128, 0, 1, fake, fake, fake, 7, None) == 1                  # KVQ_ERR_INVALID_ARG


def _prototypes():
    """name -> number of parameters, from the header's function prototypes."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(kvq_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    from quantized_kv_cache_15_b200 import kvq
    protos = _prototypes()
    assert set(protos) == set(kvq.SIGNATURES)
    bad = {n: (protos[n], len(kvq.SIGNATURES[n][1])) for n in protos if protos[n] != len(kvq.SIGNATURES[n][1])}
    assert not bad, bad


def test_host_argument_checks_run_before_any_device_call(libkvq):
    """Descriptor and pointer checks return their status without touching a GPU."""
    from quantized_kv_cache_15_b200 import kvq
    import numpy as np
    with pytest.raises(kvq.KVQError) as e:       # kv_dtype outside kvq_kv_dtype
        kvq.Plan(1, 8, 2, max_seqs=1, max_tokens_per_seq=64, k_codec=[kvq.Q4_0] * 2, v_codec=[kvq.Q4_0] * 2,
                 kv_dtype=5)
    assert e.value.status == 1
    with pytest.raises(kvq.KVQError) as e:       # tail not a multiple of 64
        kvq.Plan(1, 8, 2, max_seqs=1, max_tokens_per_seq=64, k_codec=[kvq.Q4_0] * 2, v_codec=[kvq.Q4_0] * 2,
                 tail_tokens=10)
    assert e.value.status == 1
    f = libkvq.kvq_prefill_attention
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert f(None, 0, 0, 1, None, None, None, 0, None) == 1           # null plan
    assert np.int32(kvq.KV_BF16) == 1
