// Warp-cooperative row transform and block quantization.
//
// One warp owns one row of 128 values; lane l holds elements 4l .. 4l+3 in
// registers.  A block of 32 values is 8 consecutive lanes.
//
// Bit exactness: every scale and code is produced by the same sequence of
// correctly rounded binary32 operations as the CPU reference (explicit _rn
// intrinsics, no contraction), and every reduction is a max/min (order
// independent).  The staged Hadamard transform performs, in each of its seven
// stages, one add or subtract per output, in the stage order h = 1, 2, ..., 64
// followed by the multiplication by c = fp32(1/sqrt(128)) -- so the rotated
// values are identical to the reference's as well.
//
// Quantizers (BeeLlama v0.4.0 news, §新增标准 KV cache 类型; the tiny
// workload's q4_0 formula; KV-COBRA explainer §Jargon, scalar quantization to
// 2^b levels):
//   _0   : d = fp16_rn(min(amax / (2^(b-1)-1), 65504)); code = clamp(rint(x * (1/d)),
//          -2^(b-1), 2^(b-1)-1); stored u = code + 2^(b-1); d == 0 -> u = 2^(b-1).
//   _1   : m = fp16_rd(clamp(min x, +-65504)); d = fp16_rn(min((max - m)/(2^b-1), 65504));
//          u = clamp(rint((x - m) * (1/d)), 0, 2^b-1); d == 0 -> u = 0.
//   rank : d = fp16_rn(min(amax / (2^(b-1) - 1/2), 65504));
//          u = clamp(floor(x * (1/d)), -2^(b-1), 2^(b-1)-1) + 2^(b-1); d == 0 -> u = 2^(b-1).
// Canonical packed row: b = 8 one byte per value; 4, 2, 1 bit fields LSB-first;
// 6 bits = 4-bit plane (n/2 bytes) then 2-bit plane (n/4); 5 bits = 4-bit plane
// then 1-bit plane (n/8); 3 bits = 2-bit plane
// (n/4) then 1-bit plane (n/8).  Scales: _0 and rank d_0..d_{nb-1}; _1 pairs
// (d_k, m_k).  F16: the fp16 values.
#pragma once

#include "kvq_internal.h"

namespace kvq {

__device__ __forceinline__ float hadamard_c() { return __uint_as_float(0x3db504f3u); }  // fp32(1/sqrt(128))

// In-place staged Hadamard transform of the warp's row (4 values per lane),
// followed by the multiplication by c.
__device__ __forceinline__ void fwht_row(float v[4]) {
  const int lane = threadIdx.x & 31;
  {  // h = 1
    float a = v[0], b = v[1];
    v[0] = __fadd_rn(a, b); v[1] = __fsub_rn(a, b);
    a = v[2]; b = v[3];
    v[2] = __fadd_rn(a, b); v[3] = __fsub_rn(a, b);
  }
  {  // h = 2
    float a = v[0], b = v[2];
    v[0] = __fadd_rn(a, b); v[2] = __fsub_rn(a, b);
    a = v[1]; b = v[3];
    v[1] = __fadd_rn(a, b); v[3] = __fsub_rn(a, b);
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {  // h = 4 m
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
  const float c = hadamard_c();
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __fmul_rn(v[i], c);
}

// Reduce over the `width` lanes of a block (width = 8 for 32-value blocks,
// 4 for the 16-value blocks of rank 16).
__device__ __forceinline__ float block_max(float v, int width) {
  for (int m = 1; m < width; m <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}
__device__ __forceinline__ float block_min(float v, int width) {
  for (int m = 1; m < width; m <<= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// Quantize the lane's 4 values.  Returns the 4 codes (u) in bytes 0..3 of the
// result; *d_h (and *m_h for _1) receive the block's fp16 scale (and minimum).
// kind: 0 = symmetric (_0), 1 = scale+min (_1), 2 = mid-rise (rank).
__device__ __forceinline__ uint32_t quantize4(const float x[4], int kind, int bits, int width, __half* d_h,
                                             __half* m_h) {
  uint32_t out = 0;
  if (kind == 1) {
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mn = block_min(mn, width);
    mx = block_max(mx, width);
    mn = fminf(fmaxf(mn, -65504.0f), 65504.0f);
    __half mh = __float2half_rd(mn);
    float mf = __half2float(mh);
    const int umax = (1 << bits) - 1;
    float d = __fdiv_rn(__fsub_rn(mx, mf), (float)umax);
    d = fminf(d, 65504.0f);
    __half dh = __float2half_rn(d);
    float df = __half2float(dh);
    *d_h = dh; *m_h = mh;
    if (df == 0.0f) return 0u;
    float inv = __fdiv_rn(1.0f, df);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float r = rintf(__fmul_rn(__fsub_rn(x[i], mf), inv));
      r = fminf(fmaxf(r, 0.0f), (float)umax);
      out |= (uint32_t)(int)r << (8 * i);
    }
    return out;
  }
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  amax = block_max(amax, width);
  const int half = 1 << (bits - 1);
  float den = (kind == 0) ? (float)(half - 1) : __fsub_rn((float)half, 0.5f);
  float d = __fdiv_rn(amax, den);
  d = fminf(d, 65504.0f);
  __half dh = __float2half_rn(d);
  float df = __half2float(dh);
  *d_h = dh;
  if (df == 0.0f) return (uint32_t)half * 0x01010101u;
  float inv = __fdiv_rn(1.0f, df);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float t = __fmul_rn(x[i], inv);
    float r = (kind == 0) ? rintf(t) : floorf(t);
    r = fminf(fmaxf(r, (float)(-half)), (float)(half - 1));
    out |= (uint32_t)((int)r + half) << (8 * i);
  }
  return out;
}

// Pieces of the canonical packed row written by one lane.  A lane's pieces are
// byte-contiguous and never straddle a w-byte boundary (w >= 2).
struct LanePieces {
  int n;                // pieces (0..2)
  int off[2];           // byte offset in the canonical row
  int len[2];           // 1, 2, 4 or 8 bytes; 0 means "half byte" merged by the even lane
  uint64_t val[2];
};

// Pack the 4 codes u (bytes) of lane `lane` of a row of n values at `bits`.
// Half-byte pieces (1-bit fields of 4 values) are merged with the odd neighbour
// through a shuffle; only even lanes then own the byte.
__device__ __forceinline__ LanePieces pack_lane(uint32_t u, int bits, int n, int lane) {
  LanePieces p;
  p.n = 0;
  const uint32_t u0 = u & 0xff, u1 = (u >> 8) & 0xff, u2 = (u >> 16) & 0xff, u3 = u >> 24;
  auto nib1 = [&](uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
    return (a0 & 1) | ((a1 & 1) << 1) | ((a2 & 1) << 2) | ((a3 & 1) << 3);
  };
  if (bits == 8) {
    p.n = 1; p.off[0] = 4 * lane; p.len[0] = 4; p.val[0] = u;
  } else if (bits == 4) {
    p.n = 1; p.off[0] = 2 * lane; p.len[0] = 2; p.val[0] = u0 | (u1 << 4) | (u2 << 8) | (u3 << 12);
  } else if (bits == 2) {
    p.n = 1; p.off[0] = lane; p.len[0] = 1; p.val[0] = u0 | (u1 << 2) | (u2 << 4) | (u3 << 6);
  } else if (bits == 1) {
    uint32_t nib = nib1(u0, u1, u2, u3);
    uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
    p.n = 1; p.off[0] = lane >> 1; p.len[0] = (lane & 1) ? 0 : 1; p.val[0] = nib | (other << 4);
  } else if (bits == 6) {
    p.n = 2;
    p.off[0] = 2 * lane; p.len[0] = 2;
    p.val[0] = (u0 & 15) | ((u1 & 15) << 4) | ((u2 & 15) << 8) | ((u3 & 15) << 12);
    p.off[1] = n / 2 + lane; p.len[1] = 1;
    p.val[1] = (u0 >> 4) | ((u1 >> 4) << 2) | ((u2 >> 4) << 4) | ((u3 >> 4) << 6);
  } else if (bits == 5) {
    p.n = 2;
    p.off[0] = 2 * lane; p.len[0] = 2;
    p.val[0] = (u0 & 15) | ((u1 & 15) << 4) | ((u2 & 15) << 8) | ((u3 & 15) << 12);
    uint32_t nib = nib1(u0 >> 4, u1 >> 4, u2 >> 4, u3 >> 4);
    uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
    p.off[1] = n / 2 + (lane >> 1); p.len[1] = (lane & 1) ? 0 : 1; p.val[1] = nib | (other << 4);
  } else if (bits == 3) {
    p.n = 2;
    p.off[0] = lane; p.len[0] = 1;
    p.val[0] = (u0 & 3) | ((u1 & 3) << 2) | ((u2 & 3) << 4) | ((u3 & 3) << 6);
    uint32_t nib = nib1(u0 >> 2, u1 >> 2, u2 >> 2, u3 >> 2);
    uint32_t other = __shfl_xor_sync(0xffffffffu, nib, 1);
    p.off[1] = n / 4 + (lane >> 1); p.len[1] = (lane & 1) ? 0 : 1; p.val[1] = nib | (other << 4);
  }
  return p;
}

__device__ __forceinline__ void store_piece(uint8_t* dst, int len, uint64_t v) {
  switch (len) {
    case 1: *dst = (uint8_t)v; break;
    case 2: *reinterpret_cast<uint16_t*>(dst) = (uint16_t)v; break;
    case 4: *reinterpret_cast<uint32_t*>(dst) = (uint32_t)v; break;
    case 8: *reinterpret_cast<uint64_t*>(dst) = v; break;
    default: break;
  }
}

// Address of canonical-row byte `i` of token row `t` (0..63) inside a K code plane
// (interleaved) or a V / scale plane (row-major).
__device__ __forceinline__ int kplane_off(int cb, int t, int i) {
  const int w = interleave_w(cb);
  return ((i / w) * PAGE + t) * w + (i % w);
}

// Quantize one row held by the warp (lane: 4 values) and write it to a page row.
//   codes: base of the code plane; scales: base of the scale plane; t: row (0..63)
//   interleaved: K plane layout (true) or row-major (false).
// For codec F16 the values are written as fp16 (they are fp16 values already).
__device__ __forceinline__ void quantize_store_row(const float x[4], int codec, int r, int bits, uint8_t* codes,
                                                   uint8_t* scales, int t, bool interleaved) {
  const int lane = threadIdx.x & 31;
  const int n = (codec == KVQ_RANK) ? r : D;
  int cb, sb;
  row_bytes(codec, r, bits, &cb, &sb);
  const bool active = 4 * lane < n;
  if (codec == KVQ_F16) {
    __half2 h01 = __floats2half2_rn(x[0], x[1]);
    __half2 h23 = __floats2half2_rn(x[2], x[3]);
    uint64_t v = (uint64_t)(*reinterpret_cast<uint32_t*>(&h01)) |
                 ((uint64_t)(*reinterpret_cast<uint32_t*>(&h23)) << 32);
    int off = 8 * lane;
    uint8_t* dst = codes + (interleaved ? kplane_off(cb, t, off) : t * cb + off);
    store_piece(dst, 8, v);
    return;
  }
  const int kind = (codec == KVQ_RANK) ? 2 : (codec_is_asym(codec) ? 1 : 0);
  const int blk = n < 32 ? n : 32;
  const int width = blk / 4;
  float xs[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) xs[i] = active ? x[i] : 0.0f;
  __half dh, mh;
  uint32_t u = quantize4(xs, kind, bits, width, &dh, &mh);
  LanePieces p = pack_lane(u, bits, n, lane);
  if (active) {
    for (int k = 0; k < p.n; ++k) {
      if (p.len[k] == 0) continue;
      uint8_t* dst = codes + (interleaved ? kplane_off(cb, t, p.off[k]) : t * cb + p.off[k]);
      store_piece(dst, p.len[k], p.val[k]);
    }
    if ((lane % width) == 0) {
      const int b = (4 * lane) / blk;
      if (kind == 1) {
        __half2 dm = __halves2half2(dh, mh);
        *reinterpret_cast<__half2*>(scales + t * sb + 4 * b) = dm;
      } else {
        *reinterpret_cast<__half*>(scales + t * sb + 2 * b) = dh;
      }
    }
  }
}

// The warp's fp16 row (lane: 4 values) as fp32.
__device__ __forceinline__ void load_row_f16(const __half* src, float x[4]) {
  const int lane = threadIdx.x & 31;
  uint2 v = *reinterpret_cast<const uint2*>(src + 4 * lane);
  __half2 a = *reinterpret_cast<__half2*>(&v.x);
  __half2 b = *reinterpret_cast<__half2*>(&v.y);
  float2 fa = __half22float2(a), fb = __half22float2(b);
  x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
}

// Transform the warp's row into the stored basis (lane: 4 values): the raw
// values for F16 and unrotated plans; x * inv_s (variance normalisation) and the
// staged Hadamard transform otherwise.  The projection (rank codec) runs on the
// tensor cores in project.cu.
__device__ __forceinline__ void transform_row(float x[4], int codec, int rot, const float* inv_s) {
  const int lane = threadIdx.x & 31;
  if (codec == KVQ_F16 || codec == KVQ_RANK || rot == KVQ_ROT_NONE) return;
  if (rot == KVQ_ROT_VARNORM_HADAMARD) {
    float4 s = *reinterpret_cast<const float4*>(inv_s + 4 * lane);
    x[0] = __fmul_rn(x[0], s.x); x[1] = __fmul_rn(x[1], s.y);
    x[2] = __fmul_rn(x[2], s.z); x[3] = __fmul_rn(x[3], s.w);
  }
  fwht_row(x);
}

// The lane's 4 codes (values 4l .. 4l+3 of a row of n values) from a code plane.
__device__ __forceinline__ void lane_codes(const uint8_t* plane, int cb, int t, bool interleaved, int bits, int n,
                                           int lane, uint32_t u[4]) {
  auto at = [&](int i) -> uint32_t { return plane[interleaved ? kplane_off(cb, t, i) : t * cb + i]; };
  switch (bits) {
    case 8: for (int i = 0; i < 4; ++i) u[i] = at(4 * lane + i); break;
    case 4: { uint32_t w = at(2 * lane) | (at(2 * lane + 1) << 8);
      for (int i = 0; i < 4; ++i) u[i] = (w >> (4 * i)) & 15u; } break;
    case 2: { uint32_t w = at(lane); for (int i = 0; i < 4; ++i) u[i] = (w >> (2 * i)) & 3u; } break;
    case 1: { uint32_t w = (at(lane >> 1) >> (4 * (lane & 1))) & 15u;
      for (int i = 0; i < 4; ++i) u[i] = (w >> i) & 1u; } break;
    case 6: { uint32_t lo = at(2 * lane) | (at(2 * lane + 1) << 8); uint32_t hi = at(n / 2 + lane);
      for (int i = 0; i < 4; ++i) u[i] = ((lo >> (4 * i)) & 15u) | (((hi >> (2 * i)) & 3u) << 4); } break;
    case 3: { uint32_t lo = at(lane); uint32_t hi = (at(n / 4 + (lane >> 1)) >> (4 * (lane & 1))) & 15u;
      for (int i = 0; i < 4; ++i) u[i] = ((lo >> (2 * i)) & 3u) | (((hi >> i) & 1u) << 2); } break;
    case 5: { uint32_t lo = at(2 * lane) | (at(2 * lane + 1) << 8);
      uint32_t hi = (at(n / 2 + (lane >> 1)) >> (4 * (lane & 1))) & 15u;
      for (int i = 0; i < 4; ++i) u[i] = ((lo >> (4 * i)) & 15u) | (((hi >> i) & 1u) << 4); } break;
    default: u[0] = u[1] = u[2] = u[3] = 0;
  }
}

}  // namespace kvq
