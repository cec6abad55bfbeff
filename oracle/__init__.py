"""CPU oracle for the quantized KV cache hot path.

TEST INFRASTRUCTURE ONLY.  The product package never imports this module.
It may be used by the test suite, by ``__graft_entry__.smoke()`` (to check the
GPU result) and by ``bench.py``'s CPU-baseline leg.

The arithmetic lives in ``kvq_oracle.c`` (plain C, fp32 steps in written order,
fp64 for the attention and the inverse transforms).  This wrapper only
marshals numpy arrays; it adds no arithmetic of its own.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Codec and rotation ids (same numbering as the public C header, by value).
F16, Q8_0, Q6_0, Q4_0, Q3_0, Q2_0, Q8_1, Q6_1, Q4_1, Q3_1, Q2_1, RANK, Q5_0, Q5_1 = range(14)
ROT_NONE, ROT_HADAMARD, ROT_VARNORM_HADAMARD, ROT_PROJECTION = range(4)
CODEC_BITS = {F16: 16, Q8_0: 8, Q6_0: 6, Q5_0: 5, Q4_0: 4, Q3_0: 3, Q2_0: 2,
              Q8_1: 8, Q6_1: 6, Q5_1: 5, Q4_1: 4, Q3_1: 3, Q2_1: 2}
CODEC_NAMES = {F16: "f16", Q8_0: "q8_0", Q6_0: "q6_0", Q5_0: "q5_0", Q4_0: "q4_0", Q3_0: "q3_0", Q2_0: "q2_0",
               Q8_1: "q8_1", Q6_1: "q6_1", Q5_1: "q5_1", Q4_1: "q4_1", Q3_1: "q3_1", Q2_1: "q2_1", RANK: "rank"}
D = 128


def build(force: bool = False) -> str:
    """Compile kvq_oracle.c into liboracle.so (gcc, no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            _declare(_lib)
        return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int


def _declare(L):
    L.orc_f16_rn.restype = ctypes.c_uint16
    L.orc_f16_rn.argtypes = [ctypes.c_float]
    L.orc_f16_rd.restype = ctypes.c_uint16
    L.orc_f16_rd.argtypes = [ctypes.c_float]
    L.orc_f16_to_f32.restype = ctypes.c_float
    L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_f32.restype = ctypes.c_float
    L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    for name in ("orc_f16_rn_array", "orc_f16_rd_array"):
        getattr(L, name).argtypes = [_P, _P, _I64]
    L.orc_f16_to_f32_array.argtypes = [_P, _P, _I64]
    L.orc_hadamard_matrix.argtypes = [_I, _P]
    L.orc_hadamard_c.restype = ctypes.c_float
    L.orc_rotate_dense.argtypes = [_I64, _P, _P]
    L.orc_fwht_spec.argtypes = [_I64, _P]
    L.orc_row_bytes.argtypes = [_I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]
    L.orc_pack_codes.argtypes = [_P, _I, _I, _P]
    L.orc_unpack_codes.argtypes = [_P, _I, _I, _P]
    L.orc_quantize_rows.argtypes = [_I, _I, _I, _I64, _P, _P, _P]
    L.orc_dequantize_rows.argtypes = [_I, _I, _I, _I64, _P, _P, _P]
    L.orc_varnorm_inv_rms.argtypes = [_I64, _I, _I64, _P, _P]
    L.orc_fuse_projection.argtypes = [_I, _P, _P]
    L.orc_to_stored_basis_dt.argtypes = [_I, _I, _I, _I, _P, _P, _I64, _P, _P]
    L.orc_encode_rows_dt.argtypes = [_I, _I, _I, _I, _I, _P, _P, _I64, _P, _P, _P]
    L.orc_decode_rows_original.argtypes = [_I, _I, _I, _I, _P, _P, _I64, _P, _P, _P]
    L.orc_attention.argtypes = [_I64, _P, _P, _P, ctypes.c_double, _P]
    L.orc_decode_head_dt.argtypes = [_I, _I64, _I, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P,
                                     ctypes.c_float, _P]
    L.orc_decode_packed_dt.argtypes = [_I, _I64, _P, _P, _P, _P, _I64, _P, _P, _I, _P,
                                       _I, _I, _I, _I, _I, _I, _P, _P, _P, ctypes.c_float, _P]
    L.orc_cobra_error.restype = ctypes.c_double
    L.orc_cobra_error.argtypes = [_P, _I, _I, _P]
    L.orc_cobra_best.argtypes = [_P, _I, _P, ctypes.POINTER(_I), ctypes.POINTER(_I)]
    L.orc_cobra_allocate.argtypes = [_I, _P, ctypes.c_double, _P, _P, _P]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------------------- fp16
def f16_rn(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f16_rn_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_rd(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f16_rd_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_to_f32(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().orc_f16_to_f32_array(_ptr(h), _ptr(out), h.size)
    return out


# ----------------------------------------------------------------------------- rotation
def bf16_to_f32(h):
    """uint16 bf16 bit patterns -> float32 (exact widening), element by element."""
    h = np.asarray(h, np.uint16)
    return np.array([lib().orc_bf16_to_f32(int(x)) for x in h.reshape(-1)], np.float32).reshape(h.shape)


def hadamard_matrix(n=D):
    H = np.empty((n, n), np.int8)
    lib().orc_hadamard_matrix(n, _ptr(H))
    return H


def hadamard_c() -> float:
    return float(np.float32(lib().orc_hadamard_c()))


def rotate_dense(x):
    x = _c(x, np.float64).reshape(-1, D)
    y = np.empty_like(x)
    lib().orc_rotate_dense(x.shape[0], _ptr(x), _ptr(y))
    return y


def fwht_spec(x):
    y = _c(x, np.float32).reshape(-1, D).copy()
    lib().orc_fwht_spec(y.shape[0], _ptr(y))
    return y


# ----------------------------------------------------------------------------- codecs
def row_bytes(codec, r=D, b=0):
    cb, sb = _I(), _I()
    lib().orc_row_bytes(codec, r, b, ctypes.byref(cb), ctypes.byref(sb))
    return cb.value, sb.value


def pack_codes(u, bits):
    u = _c(u, np.uint8)
    n = u.shape[-1]
    out = np.empty(n * bits // 8, np.uint8)
    lib().orc_pack_codes(_ptr(u), n, bits, _ptr(out))
    return out


def unpack_codes(packed, n, bits):
    packed = _c(packed, np.uint8)
    out = np.empty(n, np.uint8)
    lib().orc_unpack_codes(_ptr(packed), n, bits, _ptr(out))
    return out


def quantize_rows(codec, y, r=D, b=0):
    """fp32 rows in the stored basis -> (codes uint8 [n][cb], scales uint16 [n][sb/2])."""
    n_in = r if codec == RANK else D
    y = _c(y, np.float32).reshape(-1, n_in)
    cb, sb = row_bytes(codec, r, b)
    codes = np.zeros((y.shape[0], cb), np.uint8)
    scales = np.zeros((y.shape[0], max(sb // 2, 1)), np.uint16)
    lib().orc_quantize_rows(codec, r, b, y.shape[0], _ptr(y), _ptr(codes), _ptr(scales))
    return codes, scales[:, : sb // 2]


def dequantize_rows(codec, codes, scales, r=D, b=0):
    cb, sb = row_bytes(codec, r, b)
    codes = _c(codes, np.uint8).reshape(-1, cb)
    n = codes.shape[0]
    sc = np.zeros((n, max(sb // 2, 1)), np.uint16)
    if sb:
        sc[:, : sb // 2] = np.asarray(scales, np.uint16).reshape(n, sb // 2)
    n_out = r if codec == RANK else D
    y = np.empty((n, n_out), np.float32)
    lib().orc_dequantize_rows(codec, r, b, n, _ptr(codes), _ptr(sc), _ptr(y))
    return y


# ----------------------------------------------------------------------------- varnorm / projection
def varnorm_inv_rms(x_f16):
    """x_f16: uint16 [n_tok][n_ch] fp16 bit patterns -> float32 [n_ch]."""
    x = _c(x_f16, np.uint16)
    n_tok, n_ch = x.shape
    out = np.empty(n_ch, np.float32)
    lib().orc_varnorm_inv_rms(n_tok, n_ch, n_ch, _ptr(x), _ptr(out))
    return out


def fuse_projection(P):
    """P: float64 [128][r] orthonormal columns -> fp32 M [r][128] = R_r P^T."""
    P = _c(P, np.float64)
    r = P.shape[1]
    M = np.empty((r, D), np.float32)
    lib().orc_fuse_projection(r, _ptr(P), _ptr(M))
    return M


# ----------------------------------------------------------------------------- encode / decode
def to_stored_basis(codec, rot, x_f16, inv_s=None, M=None, r=D, bf16=False):
    """x_f16: uint16 raw rows [n][128] (fp16 bits, or bf16 bits when bf16)."""
    x = _c(x_f16, np.uint16).reshape(-1, D)
    n_out = r if codec == RANK else D
    y = np.empty((x.shape[0], n_out), np.float32)
    inv_s = None if inv_s is None else _c(inv_s, np.float32)
    M = None if M is None else _c(M, np.float32)
    lib().orc_to_stored_basis_dt(int(bf16), codec, rot, r, _ptr(inv_s), _ptr(M), x.shape[0], _ptr(x), _ptr(y))
    return y


def encode_rows(codec, rot, x_f16, inv_s=None, M=None, r=D, b=0, bf16=False):
    """x_f16: uint16 raw rows [n][128] (fp16 bits, or bf16 bits when bf16)."""
    x = _c(x_f16, np.uint16).reshape(-1, D)
    cb, sb = row_bytes(codec, r, b)
    codes = np.zeros((x.shape[0], cb), np.uint8)
    scales = np.zeros((x.shape[0], max(sb // 2, 1)), np.uint16)
    inv_s = None if inv_s is None else _c(inv_s, np.float32)
    M = None if M is None else _c(M, np.float32)
    lib().orc_encode_rows_dt(int(bf16), codec, rot, r, b, _ptr(inv_s), _ptr(M), x.shape[0], _ptr(x), _ptr(codes),
                             _ptr(scales))
    return codes, scales[:, : sb // 2]


def regrade_rows(old_codec, new_codec, rot, codes, scales, inv_s=None):
    """VBR regrade of packed rows ("Introducing a new KV format: VBR (Variable Bit
    Rate)", first post: the cache is requantized layer by layer as the session
    grows).  F16 rows (their codes are the raw fp16 values) are encoded with the
    new codec exactly as an append would; block-codec rows are dequantized in the
    stored basis and quantized again with the new codec.  Returns (codes, scales)."""
    if old_codec == F16:
        raw = _c(codes, np.uint8).reshape(-1, 2 * D).view(np.uint16)
        return encode_rows(new_codec, rot, raw, inv_s=inv_s)
    y = dequantize_rows(old_codec, codes, scales)
    return quantize_rows(new_codec, y)


def decode_rows_original(codec, rot, codes, scales, inv_s=None, M=None, r=D, b=0):
    cb, sb = row_bytes(codec, r, b)
    codes = _c(codes, np.uint8).reshape(-1, cb)
    n = codes.shape[0]
    sc = np.zeros((n, max(sb // 2, 1)), np.uint16)
    if sb:
        sc[:, : sb // 2] = np.asarray(scales, np.uint16).reshape(n, sb // 2)
    out = np.empty((n, D), np.float64)
    inv_s = None if inv_s is None else _c(inv_s, np.float32)
    M = None if M is None else _c(M, np.float32)
    lib().orc_decode_rows_original(codec, rot, r, b, _ptr(inv_s), _ptr(M), n, _ptr(codes), _ptr(sc), _ptr(out))
    return out


def attention(q, K, V, scale):
    q = _c(q, np.float64).reshape(D)
    K = _c(K, np.float64).reshape(-1, D)
    V = _c(V, np.float64).reshape(-1, D)
    out = np.empty(D, np.float64)
    lib().orc_attention(K.shape[0], _ptr(q), _ptr(K), _ptr(V), float(scale), _ptr(out))
    return out


def decode_head(K_f16, V_f16, q_f16, k_codec, v_codec, rot, tail=0, r=D, kb=0, vb=0,
                inv_s_k=None, inv_s_v=None, M=None, scale=None, bf16=False):
    """Decode attention for one (seq, layer, kv-head).  K_f16/V_f16: uint16 [len][128]
    history; q_f16: uint16 [G][128] (fp16 bits, or bf16 bits when bf16).  Returns
    float32 [G][128]."""
    K = _c(K_f16, np.uint16).reshape(-1, D)
    V = _c(V_f16, np.uint16).reshape(-1, D)
    q = _c(q_f16, np.uint16).reshape(-1, D)
    G = q.shape[0]
    out = np.empty((G, D), np.float32)
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(D)))
    inv_s_k = None if inv_s_k is None else _c(inv_s_k, np.float32)
    inv_s_v = None if inv_s_v is None else _c(inv_s_v, np.float32)
    M = None if M is None else _c(M, np.float32)
    lib().orc_decode_head_dt(int(bf16), K.shape[0], int(tail), G, _ptr(K), _ptr(V), _ptr(q), k_codec, v_codec, rot,
                             r, kb, vb, _ptr(inv_s_k), _ptr(inv_s_v), _ptr(M), float(scale), _ptr(out))
    return out


def decode_packed(ck, sk, cv, sv, Kt, Vt, q_f16, k_codec, v_codec, rot, r=D, kb=0, vb=0,
                  inv_s_k=None, inv_s_v=None, M=None, scale=None, bf16=False):
    """Decode attention from the oracle's own packed rows plus raw tail rows."""
    q = _c(q_f16, np.uint16).reshape(-1, D)
    G = q.shape[0]
    nq = 0 if ck is None else ck.shape[0]
    Kt = np.zeros((0, D), np.uint16) if Kt is None else _c(Kt, np.uint16).reshape(-1, D)
    Vt = np.zeros((0, D), np.uint16) if Vt is None else _c(Vt, np.uint16).reshape(-1, D)
    out = np.empty((G, D), np.float32)
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(D)))
    args = [_c(a, t) if a is not None else None for a, t in ((ck, np.uint8), (sk, np.uint16), (cv, np.uint8), (sv, np.uint16))]
    inv_s_k = None if inv_s_k is None else _c(inv_s_k, np.float32)
    inv_s_v = None if inv_s_v is None else _c(inv_s_v, np.float32)
    M = None if M is None else _c(M, np.float32)
    lib().orc_decode_packed_dt(int(bf16), nq, *[_ptr(a) for a in args], Kt.shape[0], _ptr(Kt), _ptr(Vt), G, _ptr(q),
                               k_codec, v_codec, rot, r, kb, vb, _ptr(inv_s_k), _ptr(inv_s_v), _ptr(M), float(scale),
                               _ptr(out))
    return out


# ----------------------------------------------------------------------------- KV-COBRA allocation
def cobra_error(lam, r, b, eps):
    lam = _c(lam, np.float64)
    eps = _c(eps, np.float64)
    return lib().orc_cobra_error(_ptr(lam), r, b, _ptr(eps))


def cobra_best(lam, budget, eps):
    lam = _c(lam, np.float64)
    eps = _c(eps, np.float64)
    r, b = _I(0), _I(0)
    ok = lib().orc_cobra_best(_ptr(lam), budget, _ptr(eps), ctypes.byref(r), ctypes.byref(b))
    return (r.value, b.value) if ok else None


def cobra_allocate(lambdas, bpd, eps):
    """lambdas: [n_heads][128] direction variances, each sorted decreasing.
    Returns (ranks int32 [n], bits int32 [n], bits used)."""
    lam = _c(lambdas, np.float64)
    eps = _c(eps, np.float64)
    n = lam.shape[0]
    r = np.zeros(n, np.int32)
    b = np.zeros(n, np.int32)
    used = lib().orc_cobra_allocate(n, _ptr(lam), float(bpd), _ptr(eps), _ptr(r), _ptr(b))
    return r, b, used
