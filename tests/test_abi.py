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
