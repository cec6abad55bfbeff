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

#include <cuda_bf16.h>

#include "kvq_internal.h"

namespace kvq {

__device__ __forceinline__ float hadamard_c() { return __uint_as_float(0x3db504f3u); }  // fp32(1/sqrt(128))

// One word of two raw 16-bit values (bf16 or fp16) -> two floats (exact).
__device__ __forceinline__ float2 raw2_to_float2(uint32_t w, bool bf16) {
  if (bf16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
// Two floats -> one word of raw 16-bit values, rounded to nearest even (exact for
// values that came from raw rows of the same dtype).
__device__ __forceinline__ uint32_t float2_to_raw2(float a, float b, bool bf16) {
  if (bf16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

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
                                                   uint8_t* scales, int t, bool interleaved, bool bf16 = false) {
  const int lane = threadIdx.x & 31;
  const int n = (codec == KVQ_RANK) ? r : D;
  int cb, sb;
  row_bytes(codec, r, bits, &cb, &sb);
  const bool active = 4 * lane < n;
  if (codec == KVQ_F16) {
    const uint64_t v = (uint64_t)float2_to_raw2(x[0], x[1], bf16) | ((uint64_t)float2_to_raw2(x[2], x[3], bf16) << 32);
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

// The warp's raw 16-bit row (lane: 4 values; bf16 or fp16) as fp32.
__device__ __forceinline__ void load_row_raw(const __half* src, float x[4], bool bf16) {
  const int lane = threadIdx.x & 31;
  const uint2 v = *reinterpret_cast<const uint2*>(src + 4 * lane);
  const float2 fa = raw2_to_float2(v.x, bf16), fb = raw2_to_float2(v.y, bf16);
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

// ---- four threads per row, one 32-value block each
//
// Lane q = threadIdx.x & 3 of an aligned group of four ("quad") holds values
// 32q .. 32q+31 of the row in registers.  The Hadamard stages h = 1 .. 16 stay
// inside the thread, h = 32 and 64 pair the quad's lanes through shuffles, and a
// block's scale, codes and packing need no communication at all.  Every value
// goes through the same correctly rounded binary32 operations in the same order as
// in the warp quantizer above (fwht_row, quantize4), so the stored bytes are the
// same.  Neighbouring quads own consecutive tokens of one (kv head, K|V), so the
// interleaved K planes and the row-major V planes are written in coalesced runs.

// The quad's lanes within the warp (shuffle member mask); all four lanes of a
// quad always take the same path.
__device__ __forceinline__ unsigned quad_mask() { return 0xfu << (threadIdx.x & 28); }

// Staged Hadamard transform (h = 1, 2, ..., 64, then x c) of the quad's row.
__device__ __forceinline__ void fwht_quad(float v[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
  const unsigned mask = quad_mask();
  const int q = threadIdx.x & 3;
#pragma unroll
  for (int m = 1; m < 4; m <<= 1) {  // h = 32 m
    const bool upper = (q & m) != 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float o = __shfl_xor_sync(mask, v[i], m);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
  const float c = hadamard_c();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], c);
}

// The stored basis of the quad's raw row: x * inv_s (variance normalisation) and
// the staged Hadamard transform, as transform_row above.  inv_s: the row's 128
// factors.
__device__ __forceinline__ void transform_row_quad(float v[32], int rot, const float* inv_s) {
  if (rot == KVQ_ROT_NONE) return;
  if (rot == KVQ_ROT_VARNORM_HADAMARD) {
    const float4* s4 = reinterpret_cast<const float4*>(inv_s) + 8 * (threadIdx.x & 3);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 s = s4[c];
      v[4 * c] = __fmul_rn(v[4 * c], s.x); v[4 * c + 1] = __fmul_rn(v[4 * c + 1], s.y);
      v[4 * c + 2] = __fmul_rn(v[4 * c + 2], s.z); v[4 * c + 3] = __fmul_rn(v[4 * c + 3], s.w);
    }
  }
  fwht_quad(v);
}

// 16 bytes of raw 16-bit values (bf16 or fp16) -> 8 floats.
__device__ __forceinline__ void chunk_to_float(const uint4 w, float* x, bool bf16) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = raw2_to_float2(u[k], bf16);
    x[2 * k] = f.x; x[2 * k + 1] = f.y;
  }
}

// Address of word wi of the canonical packed row of token row t: K planes are
// interleaved in 16-byte chunks, V planes row-major (cb bytes per row).
__device__ __forceinline__ uint8_t* row_word_ptr(uint8_t* codes, bool kplane, int cb, int t, int wi) {
  return kplane ? codes + ((wi / 4) * PAGE + t) * 16 + 4 * (wi % 4) : codes + t * cb + 4 * wi;
}
__device__ __forceinline__ const uint8_t* row_word_ptr(const uint8_t* codes, bool kplane, int cb, int t, int wi) {
  return kplane ? codes + ((wi / 4) * PAGE + t) * 16 + 4 * (wi % 4) : codes + t * cb + 4 * wi;
}

// Store / load words [first + W b, first + W (b + 1)) of a row: the block's share
// of a plane of W-bit fields (W words per 32-value block; 8 words = two chunks).
template <int W>
__device__ __forceinline__ void store_plane(uint8_t* codes, bool kplane, int cb, int t, int first, int b,
                                            const uint32_t w[W]) {
  const int wi = first + W * b;
  if constexpr (W == 8) {
    *reinterpret_cast<uint4*>(row_word_ptr(codes, kplane, cb, t, wi)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(row_word_ptr(codes, kplane, cb, t, wi + 4)) = make_uint4(w[4], w[5], w[6], w[7]);
  } else if constexpr (W == 4) {
    *reinterpret_cast<uint4*>(row_word_ptr(codes, kplane, cb, t, wi)) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (W == 2) {
    *reinterpret_cast<uint2*>(row_word_ptr(codes, kplane, cb, t, wi)) = make_uint2(w[0], w[1]);
  } else {
    *reinterpret_cast<uint32_t*>(row_word_ptr(codes, kplane, cb, t, wi)) = w[0];
  }
}
template <int W>
__device__ __forceinline__ void load_plane(const uint8_t* codes, bool kplane, int cb, int t, int first, int b,
                                           uint32_t w[W]) {
  const int wi = first + W * b;
  if constexpr (W == 8 || W == 4) {
#pragma unroll
    for (int h = 0; h < W / 4; ++h) {
      const uint4 x = *reinterpret_cast<const uint4*>(row_word_ptr(codes, kplane, cb, t, wi + 4 * h));
      w[4 * h] = x.x; w[4 * h + 1] = x.y; w[4 * h + 2] = x.z; w[4 * h + 3] = x.w;
    }
  } else if constexpr (W == 2) {
    const uint2 x = *reinterpret_cast<const uint2*>(row_word_ptr(codes, kplane, cb, t, wi));
    w[0] = x.x; w[1] = x.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(row_word_ptr(codes, kplane, cb, t, wi));
  }
}

// The low / high planes of a BITS-bit codec: 8, 4, 2 one plane; 6 = 4 + 2,
// 5 = 4 + 1, 3 = 2 + 1 (the high plane after the 128 * LO / 8 bytes of the low).
template <int BITS> struct Planes {
  static constexpr int LO = (BITS == 6 || BITS == 5) ? 4 : (BITS == 3 ? 2 : BITS);
  static constexpr int HI = BITS - LO;
};

// Quantize this lane's block b = q (values v[0..31] in the stored basis) with a
// _0 (KIND 0) or _1 (KIND 1) codec of BITS bits and write its codes to token row
// t; returns the block's scale word (_0: d in the low half; _1: d | m << 16).
template <int KIND, int BITS>
__device__ __forceinline__ uint32_t quantize_block_quad(const float v[32], uint8_t* codes, int t, bool kplane,
                                                        int cb) {
  constexpr int LO = Planes<BITS>::LO, HI = Planes<BITS>::HI;
  const int b = threadIdx.x & 3;
  uint32_t u[32];
  uint32_t sc;
  if constexpr (KIND == 1) {
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int j = 1; j < 32; ++j) { mn = fminf(mn, v[j]); mx = fmaxf(mx, v[j]); }
    mn = fminf(fmaxf(mn, -65504.0f), 65504.0f);
    const __half mh = __float2half_rd(mn);
    const float mf = __half2float(mh);
    constexpr int umax = (1 << BITS) - 1;
    float d = __fdiv_rn(__fsub_rn(mx, mf), (float)umax);
    d = fminf(d, 65504.0f);
    const __half dh = __float2half_rn(d);
    const float df = __half2float(dh);
    sc = (uint32_t)__half_as_ushort(dh) | ((uint32_t)__half_as_ushort(mh) << 16);
    const float inv = __fdiv_rn(1.0f, df);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float r = rintf(__fmul_rn(__fsub_rn(v[j], mf), inv));
      r = fminf(fmaxf(r, 0.0f), (float)umax);
      u[j] = df == 0.0f ? 0u : (uint32_t)(int)r;
    }
  } else {
    float amax = fabsf(v[0]);
#pragma unroll
    for (int j = 1; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    constexpr int half = 1 << (BITS - 1);
    float d = __fdiv_rn(amax, (float)(half - 1));
    d = fminf(d, 65504.0f);
    const __half dh = __float2half_rn(d);
    const float df = __half2float(dh);
    sc = __half_as_ushort(dh);
    const float inv = __fdiv_rn(1.0f, df);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float r = rintf(__fmul_rn(v[j], inv));
      r = fminf(fmaxf(r, (float)(-half)), (float)(half - 1));
      u[j] = df == 0.0f ? (uint32_t)half : (uint32_t)((int)r + half);
    }
  }
  {
    constexpr int per = 32 / LO;
    uint32_t w[LO];
#pragma unroll
    for (int k = 0; k < LO; ++k) {
      uint32_t x = 0;
#pragma unroll
      for (int i = 0; i < per; ++i) x |= (u[k * per + i] & ((1u << LO) - 1u)) << (LO * i);
      w[k] = x;
    }
    store_plane<LO>(codes, kplane, cb, t, 0, b, w);
  }
  if constexpr (HI > 0) {
    constexpr int per = 32 / HI;
    uint32_t w[HI];
#pragma unroll
    for (int k = 0; k < HI; ++k) {
      uint32_t x = 0;
#pragma unroll
      for (int i = 0; i < per; ++i) x |= ((u[k * per + i] >> LO) & ((1u << HI) - 1u)) << (HI * i);
      w[k] = x;
    }
    store_plane<HI>(codes, kplane, cb, t, 4 * LO, b, w);
  }
  return sc;
}

// Write the quad's row (v: this lane's block; stored basis, or raw values for
// F16) with `codec` to token row t: F16 as fp16 values, block codecs through
// quantize_block_quad, the four scale words written by lane 0 of the quad.
__device__ __forceinline__ void quantize_row_quad(int codec, const float v[32], uint8_t* codes, uint8_t* scales,
                                                  int t, bool kplane, int cb, int sb, bool bf16 = false) {
  const int b = threadIdx.x & 3;
  uint32_t sc = 0;
  switch (codec) {
    case KVQ_F16:
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = float2_to_raw2(v[8 * c + 2 * k], v[8 * c + 2 * k + 1], bf16);
        *reinterpret_cast<uint4*>(row_word_ptr(codes, kplane, cb, t, 16 * b + 4 * c)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      return;
    case KVQ_Q8_0: sc = quantize_block_quad<0, 8>(v, codes, t, kplane, cb); break;
    case KVQ_Q6_0: sc = quantize_block_quad<0, 6>(v, codes, t, kplane, cb); break;
    case KVQ_Q5_0: sc = quantize_block_quad<0, 5>(v, codes, t, kplane, cb); break;
    case KVQ_Q4_0: sc = quantize_block_quad<0, 4>(v, codes, t, kplane, cb); break;
    case KVQ_Q3_0: sc = quantize_block_quad<0, 3>(v, codes, t, kplane, cb); break;
    case KVQ_Q2_0: sc = quantize_block_quad<0, 2>(v, codes, t, kplane, cb); break;
    case KVQ_Q8_1: sc = quantize_block_quad<1, 8>(v, codes, t, kplane, cb); break;
    case KVQ_Q6_1: sc = quantize_block_quad<1, 6>(v, codes, t, kplane, cb); break;
    case KVQ_Q5_1: sc = quantize_block_quad<1, 5>(v, codes, t, kplane, cb); break;
    case KVQ_Q4_1: sc = quantize_block_quad<1, 4>(v, codes, t, kplane, cb); break;
    case KVQ_Q3_1: sc = quantize_block_quad<1, 3>(v, codes, t, kplane, cb); break;
    case KVQ_Q2_1: sc = quantize_block_quad<1, 2>(v, codes, t, kplane, cb); break;
    default: return;
  }
  const unsigned mask = quad_mask();
  const uint32_t s1 = __shfl_down_sync(mask, sc, 1, 4);
  const uint32_t s2 = __shfl_down_sync(mask, sc, 2, 4);
  const uint32_t s3 = __shfl_down_sync(mask, sc, 3, 4);
  if (b == 0) {
    if (codec_is_asym(codec))
      *reinterpret_cast<uint4*>(scales + t * sb) = make_uint4(sc, s1, s2, s3);
    else
      *reinterpret_cast<uint2*>(scales + t * sb) = make_uint2(sc | (s1 << 16), s2 | (s3 << 16));
  }
}

// Exact dequantization of this lane's block b = q of token row t of a _0 (KIND 0)
// or _1 (KIND 1) codec of BITS bits into the stored basis: _0 (u - 2^(b-1)) d,
// _1 u d + m.
template <int KIND, int BITS>
__device__ __forceinline__ void dequantize_block_quad(const uint8_t* codes, const uint8_t* scales, int t, bool kplane,
                                                      int cb, int sb, float v[32]) {
  constexpr int LO = Planes<BITS>::LO, HI = Planes<BITS>::HI;
  const int b = threadIdx.x & 3;
  float d, off;
  if constexpr (KIND == 1) {
    const __half2 dm = *reinterpret_cast<const __half2*>(scales + t * sb + 4 * b);
    d = __low2float(dm);
    off = __high2float(dm);
  } else {
    d = __half2float(*reinterpret_cast<const __half*>(scales + t * sb + 2 * b));
    off = -(float)(1 << (BITS - 1)) * d;
  }
  uint32_t w0[LO];
  load_plane<LO>(codes, kplane, cb, t, 0, b, w0);
  uint32_t w1[HI > 0 ? HI : 1];
  if constexpr (HI > 0) load_plane<HI>(codes, kplane, cb, t, 4 * LO, b, w1);
  constexpr int per0 = 32 / LO;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    uint32_t u = (w0[j / per0] >> (LO * (j % per0))) & ((1u << LO) - 1u);
    if constexpr (HI > 0) {
      constexpr int per1 = 32 / (HI > 0 ? HI : 1);
      u |= ((w1[j / per1] >> (HI * (j % per1))) & ((1u << HI) - 1u)) << LO;
    }
    v[j] = fmaf((float)u, d, off);
  }
}

}  // namespace kvq
