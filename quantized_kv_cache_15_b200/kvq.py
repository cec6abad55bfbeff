"""Python binding of the kvq C ABI (ctypes).  Argument marshalling only.

Every operation runs in the CUDA kernels of libkvq.so; there is no CPU or
PyTorch fallback.  Importing this module fails loudly when the library is
missing (build it with ``python -m quantized_kv_cache_15_b200.build``).
Torch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

F16, Q8_0, Q6_0, Q4_0, Q3_0, Q2_0, Q8_1, Q6_1, Q4_1, Q3_1, Q2_1, RANK, Q5_0, Q5_1 = range(14)
ROWS_WARP, ROWS_QUAD = 0, 1          # kvq_row_layout
KV_F16, KV_BF16 = 0, 1                # kvq_kv_dtype
ROT_NONE, ROT_HADAMARD, ROT_VARNORM_HADAMARD, ROT_PROJECTION = range(4)
HEAD_DIM = 128
PAGE_TOKENS = 64
NOALLOC_SCRATCH_BYTES = 16 << 20

STATUS = {0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_UNSUPPORTED", 3: "KVQ_ERR_CAPACITY",
          4: "KVQ_ERR_OOM", 5: "KVQ_ERR_CUDA", 6: "KVQ_ERR_DEVICE", 7: "KVQ_ERR_TIMEOUT", 8: "KVQ_ERR_STATE"}

# name -> (restype, argtypes); mirrors include/kvq.h
_P, _I, _I64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_IP = ctypes.POINTER(ctypes.c_int)
SIGNATURES = {
    "kvq_plan_create": (_I, [_P, ctypes.POINTER(_P)]),
    "kvq_plan_destroy": (None, [_P]),
    "kvq_plan_cache_bytes": (_I, [_P, ctypes.POINTER(_SZ)]),
    "kvq_plan_workspace_bytes": (_I, [_P, _I, ctypes.POINTER(_SZ)]),
    "kvq_cache_bind": (_I, [_P, _P, _SZ]),
    "kvq_append_quantize": (_I, [_P, _I, _I, _IP, _IP, _P, _P, _P]),
    "kvq_decode_attention": (_I, [_P, _I, _I, _IP, _P, _P, _P, _SZ, _P]),
    "kvq_prefill_attention": (_I, [_P, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "kvq_decode_attention_noalloc": (_I, [_P, _I, _I, _IP, _P, _P, _P]),
    "kvq_plan_regrade_bytes": (_I, [_P, _I, _IP, _IP, ctypes.POINTER(ctypes.c_size_t)]),
    "kvq_regrade_layer": (_I, [_P, _I, _IP, _IP, _P, ctypes.c_size_t, _P]),
    "kvq_vbr_next": (_I, [_I, _I, _IP, _IP, ctypes.c_int64, ctypes.c_int64, _I, _IP, _IP, _IP]),
    "kvq_plan_bytes_in_use": (_I, [_P, ctypes.POINTER(ctypes.c_int64)]),
    "kvq_dequantize": (_I, [_P, _I, _I, _I64, _I64, _P, _P, _P]),
    "kvq_row_bytes": (_I, [_P, _I, _I, _I, _IP, _IP]),
    "kvq_read_rows": (_I, [_P, _I, _I, _I64, _I64, _I, _P, _P, _P]),
    "kvq_seq_length": (_I, [_P, _I, _I, ctypes.POINTER(_I64)]),
    "kvq_seq_reset": (_I, [_P, _I]),
    "kvq_calibrate_varnorm": (_I, [_I64, _I, _I64, _P, _P, _P]),
    "kvq_check_device_error": (_I, [_P, _P]),
    "kvq_last_error": (ctypes.c_char_p, []),
    "kvq_launch_count": (_I, [ctypes.POINTER(ctypes.c_uint64)]),
    "kvq_cobra_allocate": (_I, [_I, _P, ctypes.c_double, _P, _IP, _IP, _IP]),
    "kvq_debug_rotate": (_I, [_P, _I, _I, _I, _I, _P, _P, _I, _P]),
    "kvq_debug_quantize_f32": (_I, [_I, _I, _I, _I, _P, _P, _P, _I, _P]),
    "kvq_debug_set_decode_split": (_I, [_P, _I]),
    "kvq_debug_set_prefill_path": (_I, [_P, _I]),
    "kvq_microbench": (_I, [_I, _I, _I, _P, _SZ, _P, ctypes.POINTER(ctypes.c_double), _P]),
    "kvq_debug_fault_injection": (_I, [_P, _I64, _I]),
}


class KVQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class _Desc(ctypes.Structure):
    _fields_ = [("n_layers", _I), ("n_q_heads", _I), ("n_kv_heads", _I), ("head_dim", _I),
                ("max_seqs", _I), ("max_tokens_per_seq", _I64), ("max_pages", _I64), ("tail_tokens", _I),
                ("k_codec", _IP), ("v_codec", _IP), ("rot", _I), ("inv_rms", ctypes.POINTER(ctypes.c_float)),
                ("rank", _IP), ("k_bits", _IP), ("v_bits", _IP), ("proj_basis", ctypes.POINTER(ctypes.c_double)),
                ("softmax_scale", ctypes.c_float), ("kv_dtype", _I)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m quantized_kv_cache_15_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(st: int):
    if st != 0:
        raise KVQError(st, lib().kvq_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ints(v: Sequence[int]):
    a = (ctypes.c_int * len(v))(*[int(x) for x in v])
    return a


class Plan:
    """A kvq plan: layout, codec map and tables of one model's KV cache on one GPU."""

    def __init__(self, n_layers: int, n_q_heads: int, n_kv_heads: int, max_seqs: int, max_tokens_per_seq: int,
                 k_codec, v_codec, rot: int = ROT_HADAMARD, tail_tokens: int = 0, inv_rms=None, rank=None,
                 k_bits=None, v_bits=None, proj_basis=None, softmax_scale: float = 0.0, max_pages: int = 0,
                 kv_dtype: int = KV_F16):
        self.n_layers, self.n_q_heads, self.n_kv_heads = n_layers, n_q_heads, n_kv_heads
        self.kv_dtype = kv_dtype
        self.tail_tokens = tail_tokens
        self.rot = rot
        n = n_layers * n_kv_heads
        kc = np.ascontiguousarray(np.asarray(k_codec, np.int32).reshape(n))
        vc = np.ascontiguousarray(np.asarray(v_codec, np.int32).reshape(n))
        keep = [kc, vc]
        d = _Desc()
        d.n_layers, d.n_q_heads, d.n_kv_heads, d.head_dim = n_layers, n_q_heads, n_kv_heads, HEAD_DIM
        d.max_seqs, d.max_tokens_per_seq, d.max_pages, d.tail_tokens = max_seqs, max_tokens_per_seq, max_pages, tail_tokens
        d.k_codec = kc.ctypes.data_as(_IP)
        d.v_codec = vc.ctypes.data_as(_IP)
        d.rot = rot
        if inv_rms is not None:
            a = np.ascontiguousarray(np.asarray(inv_rms, np.float32).reshape(n * 2 * HEAD_DIM))
            keep.append(a)
            d.inv_rms = a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        for name, arr in (("rank", rank), ("k_bits", k_bits), ("v_bits", v_bits)):
            if arr is not None:
                a = np.ascontiguousarray(np.asarray(arr, np.int32).reshape(n))
                keep.append(a)
                setattr(d, name, a.ctypes.data_as(_IP))
        if proj_basis is not None:
            a = np.ascontiguousarray(np.concatenate([np.asarray(P, np.float64).reshape(-1) for P in proj_basis]))
            keep.append(a)
            d.proj_basis = a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
        d.softmax_scale = softmax_scale
        d.kv_dtype = kv_dtype
        h = ctypes.c_void_p()
        _check(lib().kvq_plan_create(ctypes.byref(d), ctypes.byref(h)))
        self._h = h
        self._cache = None

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.kvq_plan_destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def cache_bytes(self) -> int:
        v = ctypes.c_size_t()
        _check(lib().kvq_plan_cache_bytes(self._h, ctypes.byref(v)))
        return v.value

    def workspace_bytes(self, n_seqs: int) -> int:
        v = ctypes.c_size_t()
        _check(lib().kvq_plan_workspace_bytes(self._h, n_seqs, ctypes.byref(v)))
        return v.value

    def bind(self, cache: torch.Tensor):
        _check(lib().kvq_cache_bind(self._h, _ptr(cache), cache.numel() * cache.element_size()))
        self._cache = cache

    def allocate_cache(self, device="cuda") -> torch.Tensor:
        cache = torch.empty(self.cache_bytes() + 256, dtype=torch.uint8, device=device)
        off = (-cache.data_ptr()) % 256
        view = cache[off:off + self.cache_bytes()]
        self.bind(view)
        self._cache_storage = cache
        return view

    def new_workspace(self, n_seqs: int, device="cuda") -> torch.Tensor:
        return torch.zeros(max(self.workspace_bytes(n_seqs), 16), dtype=torch.uint8, device=device)

    def append(self, layer: int, seq_ids, n_new, k: torch.Tensor, v: torch.Tensor, stream=None):
        _check(lib().kvq_append_quantize(self._h, layer, len(seq_ids), _ints(seq_ids), _ints(n_new),
                                         _ptr(k), _ptr(v), _stream(stream)))

    def decode(self, layer: int, seq_ids, q: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, stream=None):
        _check(lib().kvq_decode_attention(self._h, layer, len(seq_ids), _ints(seq_ids), _ptr(q), _ptr(out),
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream(stream)))

    def decode_noalloc(self, layer: int, seq_ids, q: torch.Tensor, out: torch.Tensor, stream=None):
        """Decode attention using the library's built-in scratch array (no workspace)."""
        _check(lib().kvq_decode_attention_noalloc(self._h, layer, len(seq_ids), _ints(seq_ids), _ptr(q), _ptr(out),
                                                  _stream(stream)))

    def regrade_bytes(self, layer: int, k_codec, v_codec) -> int:
        v = ctypes.c_size_t()
        _check(lib().kvq_plan_regrade_bytes(self._h, layer, _ints(k_codec), _ints(v_codec), ctypes.byref(v)))
        return v.value

    def regrade(self, layer: int, k_codec, v_codec, scratch: torch.Tensor, stream=None):
        """Requantize layer `layer` to new per-kv-head codecs (VBR regrade)."""
        _check(lib().kvq_regrade_layer(self._h, layer, _ints(k_codec), _ints(v_codec), _ptr(scratch),
                                       scratch.numel() * scratch.element_size(), _stream(stream)))

    def bytes_in_use(self) -> int:
        v = ctypes.c_int64()
        _check(lib().kvq_plan_bytes_in_use(self._h, ctypes.byref(v)))
        return v.value

    def dequantize(self, layer: int, seq: int, t0: int, t1: int, k_out=None, v_out=None, stream=None):
        _check(lib().kvq_dequantize(self._h, layer, seq, t0, t1, _ptr(k_out), _ptr(v_out), _stream(stream)))

    def row_bytes(self, layer: int, head: int, kv: int):
        cb, sb = ctypes.c_int(), ctypes.c_int()
        _check(lib().kvq_row_bytes(self._h, layer, head, kv, ctypes.byref(cb), ctypes.byref(sb)))
        return cb.value, sb.value

    def read_rows(self, layer: int, seq: int, t0: int, t1: int, kv: int, codes: torch.Tensor, scales: torch.Tensor,
                  stream=None):
        _check(lib().kvq_read_rows(self._h, layer, seq, t0, t1, kv, _ptr(codes), _ptr(scales), _stream(stream)))

    def seq_length(self, seq: int, layer: int) -> int:
        v = ctypes.c_int64()
        _check(lib().kvq_seq_length(self._h, seq, layer, ctypes.byref(v)))
        return v.value

    def seq_reset(self, seq: int):
        _check(lib().kvq_seq_reset(self._h, seq))

    def check_device_error(self, stream=None):
        _check(lib().kvq_check_device_error(self._h, _stream(stream)))

    def prefill(self, layer: int, seq: int, q: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, stream=None):
        """Causal attention of the last q.shape[0] tokens of `seq` (already appended)."""
        _check(lib().kvq_prefill_attention(self._h, layer, seq, q.shape[0], _ptr(q), _ptr(out), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream)))

    def debug_set_decode_split(self, pages_per_split: int):
        """Test-only: fixed pages per split-K piece (0 = automatic)."""
        _check(lib().kvq_debug_set_decode_split(self._h, pages_per_split))

    def debug_set_prefill_path(self, path: int):
        """Test-only: 0 = tensor-core prefill where the layer allows it, 1 = decode kernel."""
        _check(lib().kvq_debug_set_prefill_path(self._h, int(path)))

    def debug_fault_injection(self, wait_limit_ns: int = 2_000_000_000, drop_last_tile: bool = False):
        """Test-only: bounded-wait limit of the decode kernels and dropped last tiles."""
        _check(lib().kvq_debug_fault_injection(self._h, int(wait_limit_ns), int(bool(drop_last_tile))))

    def debug_rotate(self, layer: int, head: int, kv: int, x: torch.Tensor, y: torch.Tensor, layout: int = 0,
                     stream=None):
        _check(lib().kvq_debug_rotate(self._h, layer, head, kv, x.shape[0], _ptr(x), _ptr(y), layout,
                                      _stream(stream)))


def cobra_allocate(lambdas: np.ndarray, bpd: float, eps) -> tuple:
    """Per-head (ranks, bits, bits used) for direction variances lambdas [n][128]."""
    lam = np.ascontiguousarray(lambdas, np.float64)
    e = np.ascontiguousarray(eps, np.float64)
    n = lam.shape[0]
    r = np.zeros(n, np.int32)
    b = np.zeros(n, np.int32)
    used = ctypes.c_int()
    st = lib().kvq_cobra_allocate(n, lam.ctypes.data_as(_P), float(bpd), e.ctypes.data_as(_P),
                                  r.ctypes.data_as(_IP), b.ctypes.data_as(_IP), ctypes.byref(used))
    if st != 0:
        raise KVQError(st, "kvq_cobra_allocate: invalid spectra, bpd or budget")
    return r, b, used.value


def vbr_next(k_codec, v_codec, bytes_in_use: int, budget: int, floor_codec: int):
    """VBR policy step: (layer, new K codecs, new V codecs), layer -1 if nothing to do.
    k_codec, v_codec: [n_layers][n_kv_heads]."""
    kc = np.ascontiguousarray(k_codec, np.int32)
    vc = np.ascontiguousarray(v_codec, np.int32)
    L, H = kc.shape
    layer = ctypes.c_int()
    nk = np.zeros(H, np.int32)
    nv = np.zeros(H, np.int32)
    st = lib().kvq_vbr_next(L, H, kc.ctypes.data_as(_IP), vc.ctypes.data_as(_IP), int(bytes_in_use), int(budget),
                            int(floor_codec), ctypes.byref(layer), nk.ctypes.data_as(_IP), nv.ctypes.data_as(_IP))
    if st != 0:
        raise KVQError(st, "kvq_vbr_next: codecs off the ladder or bad arguments")
    return layer.value, nk.tolist(), nv.tolist()


UB_FFMA, UB_DP2A, UB_DP4A, UB_FMA2, UB_MIX, UB_READ = range(6)   # kvq_microbench_kind


def microbench(kind: int, iters: int, ctas: int, sink: torch.Tensor, buf: Optional[torch.Tensor] = None,
               stream=None) -> float:
    """Enqueue one micro-benchmark launch; returns its work count (multiply-adds or bytes)."""
    work = ctypes.c_double()
    nbytes = 0 if buf is None else buf.numel() * buf.element_size()
    _check(lib().kvq_microbench(kind, iters, ctas, _ptr(buf), nbytes, _ptr(sink), ctypes.byref(work),
                                _stream(stream)))
    return work.value


def launch_count() -> int:
    v = ctypes.c_uint64()
    _check(lib().kvq_launch_count(ctypes.byref(v)))
    return v.value


def calibrate_varnorm(x: torch.Tensor, n_channels: int, row_stride: int, inv_rms: torch.Tensor, stream=None):
    _check(lib().kvq_calibrate_varnorm(x.shape[0], n_channels, row_stride, _ptr(x), _ptr(inv_rms), _stream(stream)))


def debug_quantize_f32(codec: int, r: int, b: int, y: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                       layout: int = 0, stream=None):
    _check(lib().kvq_debug_quantize_f32(codec, r, b, y.shape[0], _ptr(y), _ptr(codes), _ptr(scales), layout,
                                        _stream(stream)))
