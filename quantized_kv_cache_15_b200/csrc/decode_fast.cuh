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
// Value accumulation runs as packed fp32 FMAs (fma.rn.f32x2: two FMAs per
// issue slot).  Codes are turned into exact floats with one ALU op each (a
// byte permute or a mask OR-ed into the exponent of 2^23) plus one packed
// subtract per pair.  A code at bit position 4k (nibbles) or 2k (2-bit fields)
// comes out multiplied by 16^k or 4^k; that power of two is carried by the
// channel's accumulator and divided out exactly after the last tile.  The block
// scale is folded into the softmax weight (w = p * d) and the block offset
// (-2^(b-1) d, or the minimum m) into one accumulator per block.
#pragma once

#include "kvq_internal.h"

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

// ---- pair tables: word w of a table packs two int16 query values (low, high)
enum { TAB_NAT = 0, TAB_Q4 = 1, TAB_Q2 = 2, TAB_Q1 = 3 };
__device__ __forceinline__ void tab_channels(int type, int w, int& c0, int& c1) {
  switch (type) {
    case TAB_NAT: c0 = 2 * w; c1 = c0 + 1; break;                              // bytes in order
    case TAB_Q4: {                                                              // masks 0x0F0F0F0F, >>4
      const int k = w >> 2, j = w & 3;
      c0 = 8 * k + ((j == 0) ? 0 : (j == 1) ? 4 : (j == 2) ? 1 : 5);
      c1 = c0 + 2;
    } break;
    case TAB_Q2: {                                                              // masks 0x03030303, >>2s
      const int k = w >> 3, j = w & 7, s = j >> 1;
      c0 = 16 * k + s + ((j & 1) ? 8 : 0);
      c1 = c0 + 4;
    } break;
    default: {                                                                  // masks 0x01010101, >>s
      const int k = w >> 4, j = w & 15, s = j >> 1;
      c0 = 32 * k + s + ((j & 1) ? 16 : 0);
      c1 = c0 + 8;
    } break;
  }
}

// Block epilogue of the integer score: s += (A - half*qsum) * d   (_0)
//                                     s += A * d + qsum * m       (_1)
template <int G>
__device__ __forceinline__ void score_block_epilogue(const uint8_t* ks, int sb, bool asym, int half, int b, int t0,
                                                     const int* qsi, const int a0[G], const int a1[G], float s0[G],
                                                     float s1[G]) {
  float d0, m0 = 0.f, d1, m1 = 0.f;
  if (asym) {
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
    if (asym) {
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
template <int G>
__device__ __forceinline__ void score2_block_codec(int kc, const uint8_t* kp, const uint8_t* ks, int sb, int t0,
                                                   const uint32_t* tab0, const uint32_t* tab1, const int* qsi,
                                                   float s0[G], float s1[G]) {
#pragma unroll
  for (int g = 0; g < G; ++g) { s0[g] = 0.f; s1[g] = 0.f; }
  const bool asym = codec_is_asym(kc);
  const int bits = codec_bits(kc);
  const int half = 1 << (bits - 1);
#pragma unroll 1
  for (int b = 0; b < 4; ++b) {
    int a0[G], a1[G];
#pragma unroll
    for (int g = 0; g < G; ++g) { a0[g] = 0; a1[g] = 0; }
    if (bits == 8) {
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
    } else if (bits == 4 || bits == 6 || bits == 5) {
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
    score_block_epilogue<G>(ks, sb, asym, half, b, t0, qsi, a0, a1, s0, s1);
  }
}

// Pair-table layouts the K codec uses (plane 0, plane 1; -1 = none).
__host__ __device__ inline void codec_tables(int kc, int* t0, int* t1) {
  switch (codec_bits(kc)) {
    case 8: *t0 = TAB_NAT; *t1 = -1; break;
    case 6: *t0 = TAB_Q4; *t1 = TAB_Q2; break;
    case 5: *t0 = TAB_Q4; *t1 = TAB_Q1; break;
    case 4: *t0 = TAB_Q4; *t1 = -1; break;
    case 3: *t0 = TAB_Q2; *t1 = TAB_Q1; break;
    case 2: *t0 = TAB_Q2; *t1 = -1; break;
    default: *t0 = -1; *t1 = -1; break;
  }
}

// V fast modes: the lane's 4 channels of token row t as two exact-value pairs
// (position factors 1 / 16^k / 4^k folded into the accumulators).
// mode 8: 4 code bytes; mode 4: 4 nibbles; mode 2: 4 two-bit fields.
__device__ __forceinline__ void v_codes_fast(int mode, const uint8_t* row, int lane, uint64_t& u01, uint64_t& u23) {
  const uint32_t magic = 0x4B000000u;
  if (mode == 8) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(row + 4 * lane);
    u01 = demagic2(prmt(w, magic, 0x7540u), prmt(w, magic, 0x7541u));
    u23 = demagic2(prmt(w, magic, 0x7542u), prmt(w, magic, 0x7543u));
  } else if (mode == 4) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(row + 2 * lane);
    u01 = demagic2((w & 0x000Fu) | magic, (w & 0x00F0u) | magic);
    u23 = demagic2((w & 0x0F00u) | magic, (w & 0xF000u) | magic);
  } else {
    const uint32_t w = row[lane];
    u01 = demagic2((w & 0x03u) | magic, (w & 0x0Cu) | magic);
    u23 = demagic2((w & 0x30u) | magic, (w & 0xC0u) | magic);
  }
}
// Factor carried by channel position k (0..3) of the lane in fast mode `mode`.
__device__ __forceinline__ float v_position_factor(int mode, int k) {
  if (mode == 4) return (float)(1 << (4 * k));
  if (mode == 2) return (float)(1 << (2 * k));
  return 1.0f;
}

}  // namespace kvq
