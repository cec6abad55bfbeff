// Inner loops of decode attention for the block codecs, shaped for the B200
// SM's issue pipes.
//
// Key scores (q'.khat) run as integer dot products: q' (the query in the stored
// basis, already scaled) is quantized once per CTA to int16 with one scale per
// head, and dp2a multiplies two int16 query values with two unsigned code bytes
// per instruction, accumulating exactly in int32.  Offset-binary codes need no
// conversion at all; nibble, 2-bit and 1-bit planes are spread into bytes with
// one mask (shared by all G heads); the query pairs are pre-arranged in the
// order those masks produce ("pair tables").  Per 32-value block the integer
// sum is corrected for the code offset with an exact integer block sum of the
// quantized query, converted once and scaled by the block's fp16 scale.
// The 16-bit query carries a relative error of at most 2^-16 of its largest
// element, far inside the 2e-3 output tolerance.
//
// Values run as integer dot products too (value_tile_int below) for the 8-, 4-
// and 2-bit code planes; the other value codecs (F16 pages and tail, rank, 6-,
// 5- and 3-bit) use packed fp32 FMAs (fma.rn.f32x2) on dequantized floats.
#pragma once

#include "kvq_internal.h"
#include "pair_tables.h"

namespace kvq {

__device__ __forceinline__ int dp2a_lo(uint32_t q, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(q), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi(uint32_t q, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(q), "r"(b), "r"(c));
  return d;
}
// Signed-byte forms (centred value codes).
__device__ __forceinline__ int dp2a_lo_s(uint32_t w, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi_s(uint32_t w, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(b), "r"(c));
  return d;
}

// 2^x and 1/x with the SFU's approximate instructions (relative error ~2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed fp32 helpers (a pair lives in one 64-bit register)
__device__ __forceinline__ uint64_t pack2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Two exact code values from two magic floats (2^23 + v): subtract 2^23.
__device__ __forceinline__ uint64_t demagic2(uint32_t f0, uint32_t f1) {
  const uint64_t neg = 0xCB000000CB000000ull;   // {-2^23, -2^23}
  uint64_t x;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(f0), "r"(f1));
  return add2(x, neg);
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Block epilogue of the integer score: s += (A - half*qsum) * d   (_0)
//                                     s += A * d + qsum * m       (_1)
template <int G, bool asym>
__device__ __forceinline__ void score_block_epilogue(const uint8_t* ks, int sb, int half, int b, int t0,
                                                     const int* qsi, const int a0[G], const int a1[G], float s0[G],
                                                     float s1[G]) {
  float d0, m0 = 0.f, d1, m1 = 0.f;
  if constexpr (asym) {
    const __half2 x0 = *reinterpret_cast<const __half2*>(ks + t0 * sb + 4 * b);
    const __half2 x1 = *reinterpret_cast<const __half2*>(ks + (t0 + 32) * sb + 4 * b);
    d0 = __low2float(x0); m0 = __high2float(x0);
    d1 = __low2float(x1); m1 = __high2float(x1);
  } else {
    d0 = __half2float(*reinterpret_cast<const __half*>(ks + t0 * sb + 2 * b));
    d1 = __half2float(*reinterpret_cast<const __half*>(ks + (t0 + 32) * sb + 2 * b));
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int qs = qsi[g * 4 + b];
    if constexpr (asym) {
      s0[g] = fmaf((float)a0[g], d0, fmaf((float)qs, m0, s0[g]));
      s1[g] = fmaf((float)a1[g], d1, fmaf((float)qs, m1, s1[g]));
    } else {
      s0[g] = fmaf((float)(a0[g] - half * qs), d0, s0[g]);
      s1[g] = fmaf((float)(a1[g] - half * qs), d1, s1[g]);
    }
  }
}

// Unscaled integer-domain scores of tokens t0 and t0+32 for the block codecs.
// tab0/tab1: pair tables [G][64] of the code planes; qsi: [G][4] block sums.
// KCLASS selects the code planes compiled in: 8 (q8), 4 (a nibble plane, plus a
// 2-bit or 1-bit high plane for 6 / 5 bits), 2 (a 2-bit plane, plus a 1-bit high
// plane for 3 bits).
template <int G, int KCLASS, bool KASYM>
__device__ __forceinline__ void score2_block_codec(int kc, const uint8_t* kp, const uint8_t* ks, int sb, int t0,
                                                   const uint32_t* tab0, const uint32_t* tab1, const int* qsi,
                                                   float s0[G], float s1[G]) {
#pragma unroll
  for (int g = 0; g < G; ++g) { s0[g] = 0.f; s1[g] = 0.f; }
  const int bits = codec_bits(kc);
  const int half = 1 << (bits - 1);
  KVQ_UNROLL(KVQ_SCORE_UNROLL)
  for (int b = 0; b < 4; ++b) {
    int a0[G], a1[G];
#pragma unroll
    for (int g = 0; g < G; ++g) { a0[g] = 0; a1[g] = 0; }
    if (KCLASS == 8) {
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const uint4 k0 = *reinterpret_cast<const uint4*>(kp + ((2 * b + ch) * PAGE + t0) * 16);
        const uint4 k1 = *reinterpret_cast<const uint4*>(kp + ((2 * b + ch) * PAGE + t0 + 32) * 16);
        const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w}, w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint4 qa = *reinterpret_cast<const uint4*>(tab0 + g * 64 + 16 * b + 8 * ch);
          const uint4 qb = *reinterpret_cast<const uint4*>(tab0 + g * 64 + 16 * b + 8 * ch + 4);
          const uint32_t q[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            a0[g] = dp2a_hi(q[2 * i + 1], w0[i], dp2a_lo(q[2 * i], w0[i], a0[g]));
            a1[g] = dp2a_hi(q[2 * i + 1], w1[i], dp2a_lo(q[2 * i], w1[i], a1[g]));
          }
        }
      }
    } else if (KCLASS == 4) {
      // nibble plane: chunk b holds the block's 32 low nibbles
      const uint4 k0 = *reinterpret_cast<const uint4*>(kp + (b * PAGE + t0) * 16);
      const uint4 k1 = *reinterpret_cast<const uint4*>(kp + (b * PAGE + t0 + 32) * 16);
      const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w}, w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo0 = w0[i] & 0x0F0F0F0Fu, hi0 = (w0[i] >> 4) & 0x0F0F0F0Fu;
        const uint32_t lo1 = w1[i] & 0x0F0F0F0Fu, hi1 = (w1[i] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint4 q = *reinterpret_cast<const uint4*>(tab0 + g * 64 + 16 * b + 4 * i);
          a0[g] = dp2a_hi(q.w, hi0, dp2a_lo(q.z, hi0, dp2a_hi(q.y, lo0, dp2a_lo(q.x, lo0, a0[g]))));
          a1[g] = dp2a_hi(q.w, hi1, dp2a_lo(q.z, hi1, dp2a_hi(q.y, lo1, dp2a_lo(q.x, lo1, a1[g]))));
        }
      }
      if (bits == 6) {
        // 2-bit plane (high bits, weight 16): bytes 64 + 8b .. of the row
        const uint2 h0 = *reinterpret_cast<const uint2*>(kp + ((4 + (b >> 1)) * PAGE + t0) * 16 + 8 * (b & 1));
        const uint2 h1 = *reinterpret_cast<const uint2*>(kp + ((4 + (b >> 1)) * PAGE + t0 + 32) * 16 + 8 * (b & 1));
        const uint32_t x0[2] = {h0.x, h0.y}, x1[2] = {h1.x, h1.y};
        int e0[G], e1[G];
#pragma unroll
        for (int g = 0; g < G; ++g) { e0[g] = 0; e1[g] = 0; }
#pragma unroll
        for (int ww = 0; ww < 2; ++ww)
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint32_t y0 = (x0[ww] >> (2 * s)) & 0x03030303u, y1 = (x1[ww] >> (2 * s)) & 0x03030303u;
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const uint2 q = *reinterpret_cast<const uint2*>(tab1 + g * 64 + 8 * (2 * b + ww) + 2 * s);
              e0[g] = dp2a_hi(q.y, y0, dp2a_lo(q.x, y0, e0[g]));
              e1[g] = dp2a_hi(q.y, y1, dp2a_lo(q.x, y1, e1[g]));
            }
          }
#pragma unroll
        for (int g = 0; g < G; ++g) { a0[g] += 16 * e0[g]; a1[g] += 16 * e1[g]; }
      }
      if (bits == 5) {
        // 1-bit plane (high bit, weight 16): bytes 64 .. 79 of the row = chunk 4, word b
        const uint32_t z0 = *reinterpret_cast<const uint32_t*>(kp + (4 * PAGE + t0) * 16 + 4 * b);
        const uint32_t z1 = *reinterpret_cast<const uint32_t*>(kp + (4 * PAGE + t0 + 32) * 16 + 4 * b);
        int e0[G], e1[G];
#pragma unroll
        for (int g = 0; g < G; ++g) { e0[g] = 0; e1[g] = 0; }
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t y0 = (z0 >> s) & 0x01010101u, y1 = (z1 >> s) & 0x01010101u;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint2 q = *reinterpret_cast<const uint2*>(tab1 + g * 64 + 16 * b + 2 * s);
            e0[g] = dp2a_hi(q.y, y0, dp2a_lo(q.x, y0, e0[g]));
            e1[g] = dp2a_hi(q.y, y1, dp2a_lo(q.x, y1, e1[g]));
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) { a0[g] += 16 * e0[g]; a1[g] += 16 * e1[g]; }
      }
    } else {
      // 2-bit plane (q2, and the low bits of q3): chunk b/2, half b%2
      const uint2 h0 = *reinterpret_cast<const uint2*>(kp + ((b >> 1) * PAGE + t0) * 16 + 8 * (b & 1));
      const uint2 h1 = *reinterpret_cast<const uint2*>(kp + ((b >> 1) * PAGE + t0 + 32) * 16 + 8 * (b & 1));
      const uint32_t x0[2] = {h0.x, h0.y}, x1[2] = {h1.x, h1.y};
#pragma unroll
      for (int ww = 0; ww < 2; ++ww)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t y0 = (x0[ww] >> (2 * s)) & 0x03030303u, y1 = (x1[ww] >> (2 * s)) & 0x03030303u;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint2 q = *reinterpret_cast<const uint2*>(tab0 + g * 64 + 8 * (2 * b + ww) + 2 * s);
            a0[g] = dp2a_hi(q.y, y0, dp2a_lo(q.x, y0, a0[g]));
            a1[g] = dp2a_hi(q.y, y1, dp2a_lo(q.x, y1, a1[g]));
          }
        }
      if (bits == 3) {
        // 1-bit plane (weight 4): chunk 2, word b covers the block
        const uint32_t z0 = *reinterpret_cast<const uint32_t*>(kp + (2 * PAGE + t0) * 16 + 4 * b);
        const uint32_t z1 = *reinterpret_cast<const uint32_t*>(kp + (2 * PAGE + t0 + 32) * 16 + 4 * b);
        int e0[G], e1[G];
#pragma unroll
        for (int g = 0; g < G; ++g) { e0[g] = 0; e1[g] = 0; }
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t y0 = (z0 >> s) & 0x01010101u, y1 = (z1 >> s) & 0x01010101u;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint2 q = *reinterpret_cast<const uint2*>(tab1 + g * 64 + 16 * b + 2 * s);
            e0[g] = dp2a_hi(q.y, y0, dp2a_lo(q.x, y0, e0[g]));
            e1[g] = dp2a_hi(q.y, y1, dp2a_lo(q.x, y1, e1[g]));
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) { a0[g] += 4 * e0[g]; a1[g] += 4 * e1[g]; }
      }
    }
    score_block_epilogue<G, KASYM>(ks, sb, half, b, t0, qsi, a0, a1, s0, s1);
  }
}

// ---- rank codec keys: the projected row z (r values, b bits) of a KV-COBRA head.
// Word k (4 bytes) of token t's code row in an interleaved K plane of chunk width w.
// Bytes past the row are other data of the tile; the pair tables hold zeros for
// channels >= r, so they contribute nothing.
__device__ __forceinline__ uint32_t kword(const uint8_t* kp, int w, int t, int k) {
  const int lw = __ffs(w) - 1;                     // w is a power of two
  if (w >= 4) return *reinterpret_cast<const uint32_t*>(kp + ((((4 * k) >> lw) * PAGE + t) << lw) + ((4 * k) & (w - 1)));
  const uint32_t lo = *reinterpret_cast<const uint16_t*>(kp + ((2 * k) * PAGE + t) * 2);
  const uint32_t hi = *reinterpret_cast<const uint16_t*>(kp + ((2 * k + 1) * PAGE + t) * 2);
  return lo | (hi << 16);
}

// Unscaled-to-log2 scores of tokens t0, t0+32 for a rank head with B-bit codes.
// Block b (min(32, r) channels): s += d_b * (A_b - c * qsum_b), c = (2^B - 1) / 2,
// taken exactly as (2 A_b - (2^B - 1) qsum_b) / 2.
template <int G, int B>
__device__ __forceinline__ void score2_rank(int r, const uint8_t* kp, const uint8_t* ks, int cbK, int sbK, int t0,
                                            const uint32_t* tab0, const uint32_t* tab1, const int* qsi,
                                            float s0[G], float s1[G]) {
  const int w = interleave_w(cbK);
  const int blk = r < 32 ? r : 32, nb = r / blk;
#pragma unroll
  for (int g = 0; g < G; ++g) { s0[g] = 0.f; s1[g] = 0.f; }
#pragma unroll 1
  for (int b = 0; b < nb; ++b) {
    int a0[G], a1[G];
#pragma unroll
    for (int g = 0; g < G; ++g) { a0[g] = 0; a1[g] = 0; }
    if (B == 4) {
      const int nw = blk / 8;                        // 4 words per block (2 when r = 16)
#pragma unroll 4
      for (int i = 0; i < nw; ++i) {
        const int k = 4 * b + i;
        const uint32_t x0 = kword(kp, w, t0, k), x1 = kword(kp, w, t0 + 32, k);
        const uint32_t lo0 = x0 & 0x0F0F0F0Fu, hi0 = (x0 >> 4) & 0x0F0F0F0Fu;
        const uint32_t lo1 = x1 & 0x0F0F0F0Fu, hi1 = (x1 >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint4 q = *reinterpret_cast<const uint4*>(tab0 + g * 64 + 4 * k);
          a0[g] = dp2a_hi(q.w, hi0, dp2a_lo(q.z, hi0, dp2a_hi(q.y, lo0, dp2a_lo(q.x, lo0, a0[g]))));
          a1[g] = dp2a_hi(q.w, hi1, dp2a_lo(q.z, hi1, dp2a_hi(q.y, lo1, dp2a_lo(q.x, lo1, a1[g]))));
        }
      }
    } else if (B == 2 || B == 3) {
      const int nw = blk / 16;                       // 2 words per block (1 when r = 16)
#pragma unroll 2
      for (int i = 0; i < nw; ++i) {
        const int k = 2 * b + i;
        const uint32_t x0 = kword(kp, w, t0, k), x1 = kword(kp, w, t0 + 32, k);
#pragma unroll
        for (int sft = 0; sft < 4; ++sft) {
          const uint32_t y0 = (x0 >> (2 * sft)) & 0x03030303u, y1 = (x1 >> (2 * sft)) & 0x03030303u;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint2 q = *reinterpret_cast<const uint2*>(tab0 + g * 64 + 8 * k + 2 * sft);
            a0[g] = dp2a_hi(q.y, y0, dp2a_lo(q.x, y0, a0[g]));
            a1[g] = dp2a_hi(q.y, y1, dp2a_lo(q.x, y1, a1[g]));
          }
        }
      }
      if (B == 3) {                                  // 1-bit high plane, weight 4, after r/4 bytes
        const int k = r / 16 + b;
        const uint32_t z0 = kword(kp, w, t0, k), z1 = kword(kp, w, t0 + 32, k);
        int e0[G], e1[G];
#pragma unroll
        for (int g = 0; g < G; ++g) { e0[g] = 0; e1[g] = 0; }
#pragma unroll
        for (int sft = 0; sft < 8; ++sft) {
          const uint32_t y0 = (z0 >> sft) & 0x01010101u, y1 = (z1 >> sft) & 0x01010101u;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint2 q = *reinterpret_cast<const uint2*>(tab1 + g * 64 + 16 * b + 2 * sft);
            e0[g] = dp2a_hi(q.y, y0, dp2a_lo(q.x, y0, e0[g]));
            e1[g] = dp2a_hi(q.y, y1, dp2a_lo(q.x, y1, e1[g]));
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) { a0[g] += 4 * e0[g]; a1[g] += 4 * e1[g]; }
      }
    } else {                                         // B == 1: one word per block
      const uint32_t z0 = kword(kp, w, t0, b), z1 = kword(kp, w, t0 + 32, b);
#pragma unroll
      for (int sft = 0; sft < 8; ++sft) {
        const uint32_t y0 = (z0 >> sft) & 0x01010101u, y1 = (z1 >> sft) & 0x01010101u;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint2 q = *reinterpret_cast<const uint2*>(tab0 + g * 64 + 16 * b + 2 * sft);
          a0[g] = dp2a_hi(q.y, y0, dp2a_lo(q.x, y0, a0[g]));
          a1[g] = dp2a_hi(q.y, y1, dp2a_lo(q.x, y1, a1[g]));
        }
      }
    }
    const float d0 = 0.5f * __half2float(*reinterpret_cast<const __half*>(ks + t0 * sbK + 2 * b));
    const float d1 = 0.5f * __half2float(*reinterpret_cast<const __half*>(ks + (t0 + 32) * sbK + 2 * b));
    constexpr int C2 = (1 << B) - 1;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int qs = C2 * qsi[g * 4 + b];
      s0[g] = fmaf((float)(2 * a0[g] - qs), d0, s0[g]);
      s1[g] = fmaf((float)(2 * a1[g] - qs), d1, s1[g]);
    }
  }
}

// ---- values as integer dot products
//
// Per 64-token tile the softmax weight of token t for block b and head g,
// w = p_tg * d_tb (p: softmax numerator, d: the block's fp16 scale), is rounded to
// an integer W = rint(w / sigma_g) with sigma_g = (max_t p_tg) * (max_tb d_tb) / WMAX,
// so 0 <= W <= WMAX < 2^15.  Lane j owns the token pair (j, j + 32): it packs
// (W_j, W_j+32) as two int16 and publishes them per block and head.  Every lane then
// walks the 32 pairs for its 4 channels: byte permutes put the two tokens' codes of
// a channel side by side, centred (u - 2^(b-1), moved to the top bits of the byte
// and sign-flipped, so a constant power-of-two factor rides along), and signed
// dp2a adds W_j u_j + W_j+32 u_j+32 exactly in int32.  At the end of the tile the
// integer sums are converted once, scaled by sigma_g / factor and added to the
// fp32 accumulators.  Centring matters: W's rounding error (at most sigma_g / 2)
// then multiplies a centred code, so the per-token errors do not add up to a
// constant vector that the inverse Hadamard transform would concentrate into one
// channel.  For the _1 codecs the rest of the value, m + 2^(b-1) d, is accumulated
// separately in fp32 from the exact weights.
constexpr float WMAX = 32000.0f;                   // below 2^15 with room for rounding
constexpr float RINT_MAGIC = 12582912.0f;          // 1.5 * 2^23: x + MAGIC holds rint(x) in its low bits

template <int G>
__host__ __device__ constexpr int wq_row_words() { return 4 * G + 4; }  // token-pair row: [4 blocks][G] words + pad

// One row of G words of the integer weight table.
template <int G>
__device__ __forceinline__ void load_wrow(const uint32_t* w, uint32_t out[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int g = 0; g < G; g += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(w + g);
      out[g] = v.x; out[g + 1] = v.y; out[g + 2] = v.z; out[g + 3] = v.w;
    }
  } else if constexpr (G % 2 == 0) {
#pragma unroll
    for (int g = 0; g < G; g += 2) {
      const uint2 v = *reinterpret_cast<const uint2*>(w + g);
      out[g] = v.x; out[g + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) out[g] = w[g];
  }
}

// Integer value sums of one tile for the lane's 4 channels (slot order of the
// class, see slot_channel): acc[g][k] += sum_j W_j c_j + W_j+32 c_j+32 with c the
// centred code times the class factor.
// VB 8: slots = channels 0,1,2,3, factor 1.  VB 4: slots = channels 0, 2, 1, 3,
// factor 16.  VB 2: slots = channels 0,1,2,3, factor 64.
// The row stride of a V plane of VB-bit codes is 16 VB bytes (128 channels), a
// compile-time constant.  kM / kC hold 0xF0F0F0F0 and 0x80808080 in registers (the
// caller derives them from a run-time value), so that "(x & mask) ^ 0x80" takes one
// three-input logic op rather than two with immediates.
template <int G, int VB>
__device__ __forceinline__ void value_dots(const uint8_t* vp, int lane, const uint32_t* wr, uint32_t kM, uint32_t kC,
                                           int acc[G][4]) {
  constexpr int WRS = wq_row_words<G>();
  constexpr int cbV = 16 * VB;
  KVQ_UNROLL(KVQ_VDOT_UNROLL)
  for (int j = 0; j < 32; ++j) {
    uint32_t X, Y;
    if (VB == 8) {
      const uint32_t a = *reinterpret_cast<const uint32_t*>(vp + j * cbV + 4 * lane);
      const uint32_t b = *reinterpret_cast<const uint32_t*>(vp + (j + 32) * cbV + 4 * lane);
      X = prmt(a, b, 0x5140u) ^ kC;                   // u - 128 as a signed byte
      Y = prmt(a, b, 0x7362u) ^ kC;
    } else if (VB == 4) {
      const uint32_t a = *reinterpret_cast<const uint16_t*>(vp + j * cbV + 2 * lane);
      const uint32_t b = *reinterpret_cast<const uint16_t*>(vp + (j + 32) * cbV + 2 * lane);
      const uint32_t z = prmt(a, b, 0x5140u);
      X = ((z << 4) & kM) ^ kC;                       // 16 (u - 8): low nibbles moved up
      Y = (z & kM) ^ kC;                              // 16 (u - 8): high nibbles
    } else {
      const uint32_t a = vp[j * cbV + lane];
      const uint32_t b = vp[(j + 32) * cbV + lane];
      const uint32_t z = prmt(a, b, 0x4040u);          // [a, b, a, b]
      X = (((z << 6) & 0x0000C0C0u) | ((z << 4) & 0xC0C00000u)) ^ 0x80808080u;   // 64 (u - 2), fields 0, 1
      Y = (((z << 2) & 0x0000C0C0u) | (z & 0xC0C00000u)) ^ 0x80808080u;          // fields 2, 3
    }
    uint32_t w[G];
    load_wrow<G>(wr + j * WRS, w);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      acc[g][0] = dp2a_lo_s(w[g], X, acc[g][0]);
      acc[g][1] = dp2a_hi_s(w[g], X, acc[g][1]);
      acc[g][2] = dp2a_lo_s(w[g], Y, acc[g][2]);
      acc[g][3] = dp2a_hi_s(w[g], Y, acc[g][3]);
    }
  }
}

// Channel (0..3 within the lane) and reciprocal position factor of slot k.
template <int VB>
__device__ __forceinline__ void slot_channel(int k, int& ch, float& inv_factor) {
  if (VB == 8) { ch = k; inv_factor = 1.0f; }
  else if (VB == 4) { ch = (k == 1) ? 2 : (k == 2) ? 1 : k; inv_factor = 1.0f / 16.0f; }
  else { ch = k; inv_factor = 1.0f / 64.0f; }
}

// Softmax weights of one 64-token tile as int16 pairs: lane j publishes row j of
// the warp's table ([4 blocks][G] words of (W_j, W_j+32)) and sigma_g is returned.
// nb: blocks per row (absent blocks get weight 0).  For the _1 codecs
// off[g][b] += p * (m + fcoef * d) per own token.
template <int G, bool vasym>
__device__ __forceinline__ void tile_weights(int nb, float fcoef, const uint8_t* vs, int sbV, int nvalid,
                                             int lane, uint32_t* wq, const float p0[G], const float p1[G],
                                             const float pm[G], float sg[G], float off[G][4]) {
  constexpr int WRS = wq_row_words<G>();
  float d0[4], d1[4], f0[4], f1[4];
  float dm = 0.f;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    d0[b] = 0.f; d1[b] = 0.f; f0[b] = 0.f; f1[b] = 0.f;
    if (b < nb && lane < nvalid) {
      if constexpr (vasym) {
        const __half2 x = *reinterpret_cast<const __half2*>(vs + lane * sbV + 4 * b);
        d0[b] = __low2float(x); f0[b] = fmaf(fcoef, d0[b], __high2float(x));
      } else {
        d0[b] = __half2float(*reinterpret_cast<const __half*>(vs + lane * sbV + 2 * b));
      }
    }
    if (b < nb && lane + 32 < nvalid) {
      if constexpr (vasym) {
        const __half2 x = *reinterpret_cast<const __half2*>(vs + (lane + 32) * sbV + 4 * b);
        d1[b] = __low2float(x); f1[b] = fmaf(fcoef, d1[b], __high2float(x));
      } else {
        d1[b] = __half2float(*reinterpret_cast<const __half*>(vs + (lane + 32) * sbV + 2 * b));
      }
    }
    dm = fmaxf(dm, fmaxf(d0[b], d1[b]));
  }
  // dm >= 0: its bits order like the values, so one unsigned reduction gives the max
  dm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(dm)));
  uint32_t wv[4][G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float top = pm[g] * dm;                      // largest p * d of the tile
    const float inv = top > 0.f ? WMAX * rcp_approx(top) : 0.f;
    sg[g] = top * (1.0f / WMAX);
    const float q0 = p0[g] * inv, q1 = p1[g] * inv;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float w0 = fmaf(q0, d0[b], RINT_MAGIC), w1 = fmaf(q1, d1[b], RINT_MAGIC);
      wv[b][g] = prmt(__float_as_uint(w0), __float_as_uint(w1), 0x5410u);
      if constexpr (vasym) off[g][b] = fmaf(p0[g], f0[b], fmaf(p1[g], f1[b], off[g][b]));
    }
  }
  uint32_t* row = wq + lane * WRS;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    if constexpr (G % 4 == 0) {
#pragma unroll
      for (int g = 0; g < G; g += 4)
        *reinterpret_cast<uint4*>(row + b * G + g) = make_uint4(wv[b][g], wv[b][g + 1], wv[b][g + 2], wv[b][g + 3]);
    } else if constexpr (G % 2 == 0) {
#pragma unroll
      for (int g = 0; g < G; g += 2) *reinterpret_cast<uint2*>(row + b * G + g) = make_uint2(wv[b][g], wv[b][g + 1]);
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) row[b * G + g] = wv[b][g];
    }
  }
  __syncwarp();
}

// One 64-token tile of the value accumulation on the centred integer path
// (8-, 4- and 2-bit planes).  p0/p1: softmax numerators of the lane's tokens
// (lane, lane + 32); pm: the tile's largest numerator per head.  O2: packed fp32
// accumulators of the lane's channels (already rescaled for this tile); off:
// per-block offsets of the _1 codecs.
template <int G, int VB, bool VASYM>
__device__ __forceinline__ void value_tile_int(float vhalf, const uint8_t* vp, const uint8_t* vs, int sbV, int nvalid,
                                               int lane, int blane, uint32_t* wq, uint32_t kM, uint32_t kC,
                                               const float p0[G], const float p1[G], const float pm[G],
                                               uint64_t O2[G][2], float off[G][4]) {
  float sg[G];
  tile_weights<G, VASYM>(4, vhalf, vs, sbV, nvalid, lane, wq, p0, p1, pm, sg, off);
  int acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[g][k] = 0;
  value_dots<G, VB>(vp, lane, wq + blane * G, kM, kC, acc);
  __syncwarp();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float v[4], f[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int ch; float inv_f;
      slot_channel<VB>(k, ch, inv_f);
      v[ch] = (float)acc[g][k];
      f[ch] = sg[g] * inv_f;
    }
    O2[g][0] = fma2(pack2(v[0], v[1]), pack2(f[0], f[1]), O2[g][0]);
    O2[g][1] = fma2(pack2(v[2], v[3]), pack2(f[2], f[3]), O2[g][1]);
  }
}

// ---- values as unsigned code planes with an exact weight sum
//
// For the codecs whose codes span two bit planes (6 = 4 + 2, 5 = 4 + 1, 3 = 2 + 1
// bits) and for the rank codec (1..4 bits, mid-rise levels (u - (2^b - 1)/2) d), the
// codes enter dp2a unsigned, plane by plane, and the weights' exact integer sum
// SW = sum_t W_t is accumulated beside them (one more dp2a per pair and head), so
// sum_t W_t (u_t - c) = sum_t W_t u_t - c SW is exact for any centre c: W's rounding
// errors still multiply centred codes.
// Plane words of the two tokens (rows r0, r1) for the lane's 4 channels, and the
// slot layout: BITS 4: (ch0, ch2, 16 ch1, 16 ch3); 2: (ch0, 4 ch1, 16 ch2, 64 ch3);
// 1: (ch0, 2 ch1, 4 ch2, 8 ch3).
template <int BITS>
__device__ __forceinline__ void plane_words(const uint8_t* r0, const uint8_t* r1, int lane, uint32_t& X, uint32_t& Y) {
  if (BITS == 4) {
    const uint32_t a = *reinterpret_cast<const uint16_t*>(r0 + 2 * lane);
    const uint32_t b = *reinterpret_cast<const uint16_t*>(r1 + 2 * lane);
    const uint32_t z = prmt(a, b, 0x5140u);
    X = z & 0x0F0F0F0Fu;
    Y = z & 0xF0F0F0F0u;
  } else if (BITS == 2) {
    const uint32_t z = prmt(r0[lane], r1[lane], 0x4040u);
    X = z & 0x0C0C0303u;
    Y = z & 0xC0C03030u;
  } else {
    const uint32_t a = (r0[lane >> 1] >> (4 * (lane & 1))) & 15u;
    const uint32_t b = (r1[lane >> 1] >> (4 * (lane & 1))) & 15u;
    const uint32_t z = prmt(a, b, 0x4040u);
    X = z & 0x02020101u;
    Y = z & 0x08080404u;
  }
}
template <int BITS>
__device__ __forceinline__ void plane_slot(int k, int& ch, double& inv_f) {
  if (BITS == 4) { ch = (k == 1) ? 2 : (k == 2) ? 1 : k; inv_f = (k < 2) ? 1.0 : 1.0 / 16.0; }
  else if (BITS == 2) { ch = k; inv_f = (k == 0) ? 1.0 : (k == 1) ? 0.25 : (k == 2) ? 1.0 / 16.0 : 1.0 / 64.0; }
  else { ch = k; inv_f = (k == 0) ? 1.0 : (k == 1) ? 0.5 : (k == 2) ? 0.25 : 0.125; }
}

// LO: bits of the low plane (4, 2, 1); HI: bits of the high plane (2, 1) or 0;
// offB: byte offset of the high plane in a row; cen: the codes' centre (the _1
// codecs' rest m + cen d goes to off); nb: blocks of blk channels per row.
// Rows of fewer than 128 channels (rank heads) use cl = n/4 lanes per token pair
// and 32/cl pairs side by side, summed over the lane groups at the end of the tile;
// lane cg < cl then holds channels 4cg .. 4cg+3 (the other lanes hold copies for
// channels that do not exist).
template <int G, int LO, int HI, bool VASYM>
__device__ __forceinline__ void value_tile_planes(int nb, int blk, int cl, float cen, int offB,
                                                  const uint8_t* vp, const uint8_t* vs, int cbV, int sbV, int nvalid,
                                                  int lane, uint32_t* wq, const float p0[G], const float p1[G],
                                                  const float pm[G], uint64_t O2[G][2], float off[G][4]) {
  constexpr int WRS = wq_row_words<G>();
  float sg[G];
  tile_weights<G, VASYM>(nb, cen, vs, sbV, nvalid, lane, wq, p0, p1, pm, sg, off);
  const int grp = lane / cl, cg = lane - grp * cl, ngrp = 32 / cl;
  const int blane = ((4 * cg) / blk) & 3;
  int accA[G][4], accB[G][4], sw[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    sw[g] = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) { accA[g][k] = 0; accB[g][k] = 0; }
  }
  const uint32_t* wr = wq + blane * G;
#pragma unroll 4
  for (int j = grp; j < 32; j += ngrp) {
    const uint8_t* r0 = vp + j * cbV;
    const uint8_t* r1 = vp + (j + 32) * cbV;
    uint32_t XA, YA, XB = 0u, YB = 0u;
    plane_words<LO>(r0, r1, cg, XA, YA);
    if (HI) plane_words<HI ? HI : 1>(r0 + offB, r1 + offB, cg, XB, YB);
    uint32_t w[G];
    load_wrow<G>(wr + j * WRS, w);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      accA[g][0] = dp2a_lo(w[g], XA, accA[g][0]);
      accA[g][1] = dp2a_hi(w[g], XA, accA[g][1]);
      accA[g][2] = dp2a_lo(w[g], YA, accA[g][2]);
      accA[g][3] = dp2a_hi(w[g], YA, accA[g][3]);
      if (HI) {
        accB[g][0] = dp2a_lo(w[g], XB, accB[g][0]);
        accB[g][1] = dp2a_hi(w[g], XB, accB[g][1]);
        accB[g][2] = dp2a_lo(w[g], YB, accB[g][2]);
        accB[g][3] = dp2a_hi(w[g], YB, accB[g][3]);
      }
      sw[g] = dp2a_lo(w[g], 0x00000101u, sw[g]);
    }
  }
  for (int m = cl; m < 32; m <<= 1) {                // sum over the lane groups
#pragma unroll
    for (int g = 0; g < G; ++g) {
      sw[g] += __shfl_xor_sync(0xffffffffu, sw[g], m);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        accA[g][k] += __shfl_xor_sync(0xffffffffu, accA[g][k], m);
        if (HI) accB[g][k] += __shfl_xor_sync(0xffffffffu, accB[g][k], m);
      }
    }
  }
  __syncwarp();
  // exact in double: sums of integers below 2^31 times powers of two
#pragma unroll
  for (int g = 0; g < G; ++g) {
    double v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = -(double)cen * (double)sw[g];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int ch; double inv_f;
      plane_slot<LO>(k, ch, inv_f);
      v[ch] += (double)accA[g][k] * inv_f;
      if (HI) {
        plane_slot<HI ? HI : 1>(k, ch, inv_f);
        v[ch] += (double)accB[g][k] * inv_f * (double)(1 << LO);
      }
    }
    O2[g][0] = fma2(pack2((float)v[0], (float)v[1]), pack2(sg[g], sg[g]), O2[g][0]);
    O2[g][1] = fma2(pack2((float)v[2], (float)v[3]), pack2(sg[g], sg[g]), O2[g][1]);
  }
}

}  // namespace kvq
