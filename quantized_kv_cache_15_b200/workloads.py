"""Seeded synthetic inputs for the five workloads (and scaled-down copies of them).

This module holds NO arithmetic of the quantized-cache method: it only draws
inputs (fp16 K/V rows, fp16 queries, context lengths, per-head projection
bases, codec maps) with the shapes and value distributions of the workloads.
Both the product (bench) and the tests' oracle side use it, so that the same
rows can be regenerated on either device, chunk by chunk.

Random numbers come from a counter-based generator: a 32-bit integer hash of
(stream key, element index) evaluated with int64 torch ops, which gives the
same bits on CPU and CUDA.  Normal N(0,1) values come by inversion: the top 16
bits of a 32-bit uniform pick a cell of a table of standard-normal quantiles
(65537 fp32 values at u = k / 65536, computed once on the host; the two end
points at u = 2^-33 and 1 - 2^-33, about 6.2 sigma) and the low 16 bits
interpolate linearly inside the cell, with correctly rounded fp32 subtract,
multiply and add (also device independent).  The heavy-tailed term is a
Student-t (nu = 3) built as Z / sqrt(chi2_3 / 3) from four such values.
"""
from __future__ import annotations

import dataclasses
import math
import statistics
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

D = 128
M32 = 0xFFFFFFFF

# codec ids (same numbering as include/kvq.h)
F16, Q8_0, Q6_0, Q4_0, Q3_0, Q2_0, Q8_1, Q6_1, Q4_1, Q3_1, Q2_1, RANK, Q5_0, Q5_1 = range(14)
ROT_NONE, ROT_HADAMARD, ROT_VARNORM_HADAMARD, ROT_PROJECTION = range(4)

RANKS = (16, 32, 64, 96, 128)
BITS = (1, 2, 3, 4)


# ----------------------------------------------------------------------------- counter-based hash
def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for x in [0, 2^32), without int64 overflow."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & M32


def _hash32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _hash32_int(x: int) -> int:
    x &= M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & M32
    x ^= x >> 16
    return x


def stream_key(*parts: int) -> int:
    k = 0x2545F491
    for p in parts:
        k = _hash32_int(k ^ ((p * 0x9E3779B1) & M32))
        k = _hash32_int(k + 0x632BE5AB)
    return k


def random_bits(key: int, start: int, n: int, device) -> torch.Tensor:
    """32 random bits (int64 holding [0, 2^32)) for counters start .. start+n-1."""
    i = torch.arange(start, start + n, dtype=torch.int64, device=device)
    a = _hash32((i & M32) ^ key)
    return _hash32((a + (i >> 32) + 0x632BE5AB) & M32)


def uniform16(key: int, start: int, n: int, device) -> torch.Tensor:
    """fp32 uniforms (k + 1/2) / 65536, two per hash (device independent)."""
    bits = random_bits(key, start, (n + 1) // 2, device)
    u = torch.stack(((bits & 0xFFFF), (bits >> 16)), dim=1).reshape(-1)[:n]
    return (u.to(torch.float32) + 0.5) * (1.0 / 65536.0)


_QUANTILES: Dict[str, torch.Tensor] = {}


def normal_quantiles(device) -> torch.Tensor:
    """fp32 standard-normal quantiles at u = k / 65536, k = 0 .. 65536, the ends
    taken at u = 2^-33 and 1 - 2^-33 (host double precision, rounded once)."""
    dev = str(torch.device(device))
    if dev not in _QUANTILES:
        if "cpu" not in _QUANTILES:
            nd = statistics.NormalDist()
            eps = 2.0 ** -33
            q = [nd.inv_cdf(min(max(k / 65536.0, eps), 1.0 - eps)) for k in range(65537)]
            _QUANTILES["cpu"] = torch.tensor(q, dtype=torch.float64).to(torch.float32)
        _QUANTILES[dev] = _QUANTILES["cpu"].to(device)
    return _QUANTILES[dev]


def gauss(key: int, start: int, n: int, device) -> torch.Tensor:
    """N(0,1) values by inversion (see the module docstring), fp32, exactly
    reproducible on any device: cell k = bits >> 16, f = ((bits & 0xFFFF) + 1/2) / 65536,
    x = T[k] + (T[k+1] - T[k]) * f."""
    bits = random_bits(key, start, n, device)
    t = normal_quantiles(device)
    k = bits >> 16
    f = ((bits & 0xFFFF).to(torch.float32) + 0.5) * (1.0 / 65536.0)
    lo = t[k]
    return lo + (t[k + 1] - lo) * f


def student_t3(key: int, start: int, n: int, device) -> torch.Tensor:
    """Z0 / sqrt((Z1^2 + Z2^2 + Z3^2) / 3), evaluated in fp64 (where division and
    square root are correctly rounded on every device) and rounded once to fp32."""
    z = gauss(key, 4 * start, 4 * n, device).reshape(n, 4).to(torch.float64)
    chi = (z[:, 1] * z[:, 1] + z[:, 2] * z[:, 2]) + z[:, 3] * z[:, 3]
    return (z[:, 0] / torch.sqrt(chi / 3.0)).to(torch.float32)


# ----------------------------------------------------------------------------- workloads
@dataclasses.dataclass
class Workload:
    """Shapes, codecs and data recipe of one workload."""
    name: str
    cfg_id: int                      # 1..5, the data recipe
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    ctx: List[int]                   # context length per sequence (tokens already cached)
    tail: int = 0
    rot: int = ROT_HADAMARD
    k_codec: Optional[List[List[int]]] = None      # [L][Hkv]
    v_codec: Optional[List[List[int]]] = None
    rank: Optional[List[List[int]]] = None         # [L][Hkv] (RANK codec)
    k_bits: Optional[List[List[int]]] = None
    v_bits: Optional[List[List[int]]] = None
    append_tokens: int = 0           # tokens appended per decode step (per appended sequence)
    append_seqs: int = 0             # sequences that get the append each step
    seed: int = 0

    @property
    def G(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def batch(self) -> int:
        return len(self.ctx)

    # --- per-element recipes ------------------------------------------------
    def _outlier_channels(self, layer: int, head: int) -> List[int]:
        """4 distinct channels per (layer, kv-head), fixed across tokens (R18)."""
        key = stream_key(self.seed, 11, layer, head)
        chans: List[int] = []
        i = 0
        while len(chans) < 4:
            c = _hash32_int(key + i) % D
            if c not in chans:
                chans.append(c)
            i += 1
        return chans

    def _k_sigma(self, layer: int) -> torch.Tensor:
        """Config 2: per-(head, channel) std, log-uniform in [0.1, 10]."""
        key = stream_key(self.seed, 12, layer)
        u = uniform16(key, 0, self.n_kv_heads * D, "cpu").to(torch.float64)
        return torch.pow(10.0, 2.0 * u - 1.0).to(torch.float32).reshape(self.n_kv_heads, D)

    def rows(self, kind: str, layer: int, seq: int, t0: int, t1: int, device="cpu") -> torch.Tensor:
        """fp16 rows [t1-t0][Hkv][128] of K (kind='K') or V ('V') for tokens t0..t1-1."""
        n = (t1 - t0) * self.n_kv_heads * D
        kid = 1 if kind == "K" else 2
        key = stream_key(self.seed, kid, layer, seq)
        start = t0 * self.n_kv_heads * D
        if self.cfg_id == 4 and kind == "K":
            return self._lowrank_keys(layer, seq, t0, t1, device)
        x = gauss(key, start, n, device).reshape(t1 - t0, self.n_kv_heads, D)
        if kind == "K" and self.cfg_id in (1, 3, 5):
            scale = torch.ones(self.n_kv_heads, D, dtype=torch.float32)
            for h in range(self.n_kv_heads):
                for c in self._outlier_channels(layer, h):
                    scale[h, c] = 20.0
            x = x * scale.to(device)
            if self.cfg_id == 3:
                tkey = stream_key(self.seed, 13, layer, seq)
                x = x + student_t3(tkey, start, n, device).reshape(x.shape)
        elif kind == "K" and self.cfg_id == 2:
            x = x * self._k_sigma(layer).to(device)
        return x.to(torch.float16)

    def _lowrank_keys(self, layer: int, seq: int, t0: int, t1: int, device) -> torch.Tensor:
        """Config 4 keys: A B + 0.1 N(0,1); A [T][8] N(0,1), B [8][128] N(0,1/8) per head.
        The product is written as eight elementwise multiply-then-add steps in a fixed
        order so that CPU and GPU produce the same bits."""
        T = t1 - t0
        H = self.n_kv_heads
        akey = stream_key(self.seed, 14, layer, seq)
        A = gauss(akey, t0 * H * 8, T * H * 8, device).reshape(T, H, 8)
        bkey = stream_key(self.seed, 15, layer)
        B = gauss(bkey, 0, H * 8 * D, device).reshape(H, 8, D) * float(np.float32(math.sqrt(1.0 / 8.0)))
        acc = A[:, :, 0:1] * B[None, :, 0, :]
        for k in range(1, 8):
            acc = acc + A[:, :, k:k + 1] * B[None, :, k, :]
        nkey = stream_key(self.seed, 1, layer, seq)
        noise = gauss(nkey, t0 * H * D, T * H * D, device).reshape(T, H, D)
        return (acc + noise * 0.1).to(torch.float16)

    def queries(self, layer: int, seq: int, step: int, device="cpu") -> torch.Tensor:
        """fp16 [Hq][128] ~ N(0,1) query of `seq` at decode step `step`."""
        key = stream_key(self.seed, 3, layer, seq, step)
        return gauss(key, 0, self.n_q_heads * D, device).reshape(self.n_q_heads, D).to(torch.float16)

    def calib_rows(self, kind: str, layer: int, n: int = 512, device="cpu") -> torch.Tensor:
        """Calibration prefix (R10): n tokens drawn like the workload's own rows, from
        a separate stream (sequence id -1)."""
        return self.rows(kind, layer, -1 & 0xFFFF, 0, n, device)

    def proj_basis(self, layer: int, head: int) -> np.ndarray:
        """Config 4: a random orthonormal 128 x r basis (QR of a seeded Gaussian,
        diag(R) made positive), float64."""
        r = self.rank[layer][head]
        key = stream_key(self.seed, 16, layer, head)
        g = gauss(key, 0, D * r, "cpu").to(torch.float64).numpy().reshape(D, r)
        Q, R = np.linalg.qr(g)
        s = np.sign(np.diag(R))
        s[s == 0] = 1.0
        return np.ascontiguousarray(Q * s[None, :])

    # --- derived sizes -------------------------------------------------------
    def codec_lists(self):
        return self.k_codec, self.v_codec


def _const_map(L: int, H: int, v: int) -> List[List[int]]:
    return [[v] * H for _ in range(L)]


def vbr_codec_map(L: int, H: int) -> Tuple[List[List[int]], List[List[int]]]:
    """Config 3 (R13): the listed codec per layer band is V's; K is one step richer
    on the ladder F16 > q8_0 > q6_0 > q4_1 > q2_1.  Bands are scaled to L layers."""
    ladder = [F16, Q8_0, Q6_0, Q4_1, Q2_1]
    bands = [(0, 4, F16), (4, 16, Q8_0), (16, 32, Q6_0), (32, 48, Q4_1), (48, 64, Q2_1)]
    kmap, vmap = [], []
    for l in range(L):
        l64 = (l * 64) // L
        v = next(c for a, b, c in bands if a <= l64 < b)
        k = ladder[max(0, ladder.index(v) - 1)]
        kmap.append([k] * H)
        vmap.append([v] * H)
    return kmap, vmap


def rank_bits_map(L: int, H: int, seed: int, bpd: float = 1.0) -> Tuple[List[List[int]], List[List[int]]]:
    """Config 4 (R14): per-head (r, b) with r in {16,32,64,96,128}, b in {1..4}, such that
    sum_h r_h b_h = bpd * 128 * (number of heads) exactly.  Heads first draw (r, b)
    uniformly from the 20 pairs; while the total is above budget a seeded head is
    lowered to a uniformly drawn pair of smaller r*b; then while below budget a seeded
    head is raised to a pair whose increase fits the remaining deficit."""
    pairs = [(r, b) for r in RANKS for b in BITS]
    n = L * H
    target = int(round(bpd * D * n))
    key = stream_key(seed, 17)
    ctr = [0]

    def draw(m: int) -> int:
        v = _hash32_int(key + ctr[0]) % m
        ctr[0] += 1
        return v

    cur = [pairs[draw(len(pairs))] for _ in range(n)]
    total = sum(r * b for r, b in cur)
    while total > target:
        h = draw(n)
        rb = cur[h][0] * cur[h][1]
        lower = [p for p in pairs if p[0] * p[1] < rb]
        if not lower:
            continue
        p = lower[draw(len(lower))]
        total += p[0] * p[1] - rb
        cur[h] = p
    while total < target:
        h = draw(n)
        rb = cur[h][0] * cur[h][1]
        up = [p for p in pairs if rb < p[0] * p[1] <= rb + (target - total)]
        if not up:
            continue
        p = up[draw(len(up))]
        total += p[0] * p[1] - rb
        cur[h] = p
    ranks = [[cur[l * H + h][0] for h in range(H)] for l in range(L)]
    bits = [[cur[l * H + h][1] for h in range(H)] for l in range(L)]
    return ranks, bits


def ragged_contexts(batch: int, lo: int, hi: int, seed: int) -> List[int]:
    key = stream_key(seed, 18)
    return [lo + (_hash32_int(key + i) % (hi - lo + 1)) for i in range(batch)]


def make_workload(cfg_id: int, scale: str = "full", **over) -> Workload:
    """The five workloads.  scale='full' is the stated size; scale='small' keeps the
    structure (codecs, GQA, tail, raggedness) with fewer layers and tokens so that
    the oracle finishes in seconds."""
    small = scale == "small"
    if cfg_id == 1:
        w = Workload("tiny-q4_0", 1, 1, 8, 2, [1024], tail=0, rot=ROT_HADAMARD, seed=1)
        w.k_codec = _const_map(1, 2, Q4_0)
        w.v_codec = _const_map(1, 2, Q4_0)
    elif cfg_id == 2:
        L, T = (2, 2000) if small else (32, 32768)
        w = Workload("llama8b-q8_0k-q4_0v-32k", 2, L, 32, 8, [T], tail=0, rot=ROT_HADAMARD,
                     append_tokens=1, append_seqs=1, seed=2)
        w.k_codec = _const_map(L, 8, Q8_0)
        w.v_codec = _const_map(L, 8, Q4_0)
    elif cfg_id == 3:
        L, T, tail = (5, 1500, 256) if small else (64, 65536, 1024)
        w = Workload("vbr-mix-tail1024-64k", 3, L, 24, 4, [T], tail=tail, rot=ROT_HADAMARD, seed=3)
        w.k_codec, w.v_codec = vbr_codec_map(L, 4)
    elif cfg_id == 4:
        L, T = (2, 1500) if small else (32, 131072)
        w = Workload("cobra-rank-bits-128k", 4, L, 32, 8, [T], tail=0, rot=ROT_PROJECTION, seed=4)
        w.rank, w.k_bits = rank_bits_map(L, 8, seed=4)
        w.v_bits = w.k_bits
        w.k_codec = _const_map(L, 8, RANK)
        w.v_codec = _const_map(L, 8, RANK)
    elif cfg_id == 5:
        if small:
            L, B, lo, hi, tail, chunk, nap = 2, 6, 100, 1200, 64, 200, 2
        else:
            L, B, lo, hi, tail, chunk, nap = 32, 64, 1024, 32768, 256, 2048, 8
        w = Workload("batch64-kvarn4-tail256", 5, L, 32, 8, ragged_contexts(B, lo, hi, 5), tail=tail,
                     rot=ROT_VARNORM_HADAMARD, append_tokens=chunk, append_seqs=nap, seed=5)
        w.k_codec = _const_map(L, 8, Q4_0)
        w.v_codec = _const_map(L, 8, Q4_0)
    else:
        raise ValueError(cfg_id)
    for k, v in over.items():
        setattr(w, k, v)
    return w
