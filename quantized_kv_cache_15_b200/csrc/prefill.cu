// Chunked-prefill attention over the quantized cache on the 5th-generation tensor
// cores (tcgen05.mma, fp32 accumulators in tensor memory).
//
// Forum thread on KV compression (attention paragraph): every query dots every
// prior key, softmax, weighted average of the values.  Unlike decode, a prefill
// chunk brings many queries at once, so a key/value tile is shared by a block of
// queries: one CTA takes QB = 128 / G consecutive query positions of one kv head
// (128 rows: row j*G + g is query position j of the block, query head g of the
// group) and walks the positions its last query can see, 64 at a time.  Per tile:
//
//   S   = Q' K^T      [128 x 64]   (tcgen05, M = 128, N = 64, K = 128 channels)
//   P   = exp2(S - m) (online softmax, causal mask, one thread per row)
//   O  += P V         [128 x 128]  (tcgen05, M = 128, N = 128, K = 64 tokens)
//
// Keys and values are dequantized once per CTA into fp16 operand images in shared
// memory, in the stored (rotated) basis: y = d * (u - 2^(b-1)) for the _0
// codecs, y = u * d + m for the _1 codecs (the keys' hi part is one rounding of
// the exact product, the lo part the exact remainder; the _1 keys go through the
// reference dequantizer's fp32 value).  fp16 holds 11 significant bits,
// so the keys are split y = y_hi + y_lo (both fp16) and the query
// q' = R (s_k * q) * softmax_scale * log2(e) likewise, and S accumulates the
// three products Qhi Khi + Qlo Khi + Qhi Klo (the fourth is below fp32's
// rounding of S).  The values and P enter as single fp16 roundings: measured on
// the workloads' data (emulated on the CPU) this keeps the output within about
// 5e-4 relative of exact attention, a quarter of the parity bar.
//
// The tail (raw F16 rows of the newest positions) is brought into the same
// basis on the fly: y = R (inv_s * x) for keys and values, exactly the append's
// transform before quantization, so one query image and one accumulator serve
// every tile; the output is O_row / l taken back through R and s_v.
//
// Warp roles (320 threads, one CTA per SM: 512 tensor-memory columns, at most
// 227 KiB of shared memory -- three operand stages of 48 KiB and two to four raw
// page-head stages):
//   warps 0-3  softmax: thread = row = TMEM lane; the query image (into tensor
//              memory), online softmax with a lazy rescale (O is rescaled only
//              when the running max grows by more than 8 in log2 units), P over
//              its tile's S columns, and the epilogue;
//   warps 4-7  dequantizers (one instantiation per block codec): quantized tiles
//              from the raw ring, tail tiles straight from the ring in global
//              memory, into the operand stages (key half released when S
//              completes, value half when P V does);
//   warp 8     producer: one cp.async.bulk per 64-token page-head into the raw ring;
//   warp 9     tensor memory allocation and, on one thread, the MMA issue, which
//              polls its barriers without suspending and issues whichever of S
//              (next tile) and P V (oldest tile with P ready) can go.
// The key and value images in shared memory use the canonical 128-byte-swizzled
// layout: a 64-token x 128-channel tile is two 8 KiB halves (channels 0-63 and
// 64-127); in a half, token t owns the 128-byte row t, and its 16-byte chunk j
// (channels 8j .. 8j+7 of the half) sits at chunk position j XOR (t % 8), so
// the eight rows of an 8-token group spread every chunk over all banks.  Read as
// K-major with rows = tokens (keys: B of S) the 8-token groups are 1024 bytes
// apart (stride byte offset) and a 16-channel step moves the start 32 bytes
// inside the half; read as MN-major with N = channels and K = tokens (values: B
// of P V) the two halves are 8 KiB apart (leading byte offset), the 8-token
// groups 1024 (stride byte offset), and a 16-token step moves the start 2 KiB.
// The query image and P live in tensor memory (A operands).
// Every wait is bounded; a timeout latches an error bit and sends every role out
// of its loop; in-flight copies and MMAs are waited for (bounded) and the tensor
// memory is always freed.
#include "kvq_internal.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace kvq {

namespace {

constexpr int PF_ROWS = 128;
constexpr int PF_TOK = 64;
constexpr int PF_THREADS = 320;
constexpr int PF_TILE_BYTES = PF_TOK * D * 2;          // one fp16 image of a 64-token tile
constexpr int PF_OP_BYTES = 3 * PF_TILE_BYTES;         // V, K hi, K lo
constexpr int PF_NO = 3;                               // operand stages
constexpr int PF_OFF_RAW = PF_NO * PF_OP_BYTES;        // 147456
constexpr int PF_MISC = 256;                           // barriers, TMEM address, abort flag
constexpr int PF_SMEM_MAX = 232448;                    // 227 KiB opt-in per CTA
// Tensor memory (512 columns x 128 lanes, lane = row): S of tiles i (i even) and
// i (i odd) in columns 0-63 and 64-127, each overwritten in place by the tile's
// fp16 P (32 columns of pairs); O in 128-255; the query image q' hi in 256-319
// and lo in 320-383 (fp16 pairs).
constexpr uint32_t PF_TMEM_COLS = 512;
constexpr uint32_t PF_O_COL = 128;
constexpr uint32_t PF_QH_COL = 256;
constexpr uint32_t PF_QL_COL = 320;
constexpr float PF_RESCALE = 8.0f;                     // lazy rescale threshold (log2 units)

// Shared-memory matrix descriptor of a 128-byte-swizzled operand (atoms 1024-byte
// aligned, so the base offset is 0).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version for sm_100
  d |= (uint64_t)2 << 61;   // layout: 128-byte swizzle
  return d;
}
// kind::f16 instruction descriptor: D fp32, A and B fp16, A K-major, B K-major or
// MN-major, M = 128, N = n.
__device__ __forceinline__ uint32_t umma_idesc(int n, bool b_mn_major) {
  return (1u << 4) | (b_mn_major ? (1u << 16) : 0u) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(PF_ROWS >> 4) << 24);
}
// D (tensor memory) = A B (+ D when `accumulate` is nonzero), kind::f16, with A
// read from tensor memory (M rows in lanes, K along columns, two 16-bit elements
// per 32-bit column, the lower-indexed in the low half) and B from shared memory
// through its descriptor.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane (warp w: lanes 32(w%4)..),
// waited for inside the same statement so that no use of r can move above the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t r[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t r[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Staged Hadamard transform of a whole row held by one thread, times c = 1/sqrt(128)
// (the same butterflies and scaling as the warp-level transform of the append).
__device__ __forceinline__ void fwht128(float x[D]) {
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
#pragma unroll
    for (int i = 0; i < D; ++i) {
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = __fadd_rn(a, b);
        x[i + h] = __fsub_rn(a, b);
      }
    }
  }
  const float c = hadamard_c();
#pragma unroll
  for (int i = 0; i < D; ++i) x[i] = __fmul_rn(x[i], c);
}

// Byte offset of 16-byte chunk c8 (channels 8 c8 .. 8 c8 + 7) of token t in a key
// or value image: half c8 / 8, row t, chunk position (c8 % 8) XOR (t % 8).
__device__ __forceinline__ uint32_t op_off(int t, int c8) {
  return (uint32_t)(((c8 >> 3) << 13) + ((t >> 3) << 10) + ((t & 7) << 7) + (((c8 & 7) ^ (t & 7)) << 4));
}

// Eight values -> fp16 hi words and, when lo != null, the fp16 remainders.
__device__ __forceinline__ void split8(const float x[8], uint8_t* hi, uint8_t* lo, uint32_t off) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __half2 hh = __floats2half2_rn(x[2 * e], x[2 * e + 1]);
    h[e] = *reinterpret_cast<const uint32_t*>(&hh);
    if (lo) {
      const float2 hf = __half22float2(hh);
      const __half2 ll = __floats2half2_rn(__fsub_rn(x[2 * e], hf.x), __fsub_rn(x[2 * e + 1], hf.y));
      l[e] = *reinterpret_cast<const uint32_t*>(&ll);
    }
  }
  *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
  if (lo) *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

// One 32-channel block (block b of token t) of a page-head's K or V plane:
// its codes' low plane (lo, up to 32 bytes) and high plane (hi, up to 8 bytes).
// K planes are interleaved in 16-byte pieces (byte o of token t at
// ((o/16)*64 + t)*16 + o%16); V planes are row-major.  Every read is aligned.
template <int BITS, bool KPLANE>
__device__ __forceinline__ void block_planes(const uint8_t* codes, int cb, int t, int b, uint32_t lo[8],
                                             uint32_t hi[2]) {
  auto at = [&](int o) -> const uint8_t* {
    return KPLANE ? codes + ((((o >> 4) * PAGE + t) << 4) + (o & 15)) : codes + t * cb + o;
  };
  if (BITS == 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(at(32 * b));
    const uint4 c = *reinterpret_cast<const uint4*>(at(32 * b + 16));
    lo[0] = a.x; lo[1] = a.y; lo[2] = a.z; lo[3] = a.w; lo[4] = c.x; lo[5] = c.y; lo[6] = c.z; lo[7] = c.w;
  } else if (BITS >= 4) {                          // 4, 5, 6: nibble plane first
    const uint4 a = *reinterpret_cast<const uint4*>(at(16 * b));
    lo[0] = a.x; lo[1] = a.y; lo[2] = a.z; lo[3] = a.w;
  } else {                                         // 2, 3: 2-bit plane first
    const uint2 a = *reinterpret_cast<const uint2*>(at(8 * b));
    lo[0] = a.x; lo[1] = a.y;
  }
  if (BITS == 6) {
    const uint2 h = *reinterpret_cast<const uint2*>(at(64 + 8 * b));
    hi[0] = h.x; hi[1] = h.y;
  } else if (BITS == 5) {
    hi[0] = *reinterpret_cast<const uint32_t*>(at(64 + 4 * b));
  } else if (BITS == 3) {
    hi[0] = *reinterpret_cast<const uint32_t*>(at(32 + 4 * b));
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ __half2 as_h2(uint32_t w) { return *reinterpret_cast<const __half2*>(&w); }
__device__ __forceinline__ uint32_t as_u32(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

// The codes of channels 8J .. 8J+7 of a block as four fp16 pairs 1024 + u (bit
// pattern 0x6400 | u, exact for u < 1024): pair e holds channels 8J+2e (low
// half) and 8J+2e+1.  8- and 4-bit planes are spread with byte permutes (for
// nibbles, the sign-replicating selectors 8 + k give zero bytes: every byte is
// below 16); the other widths assemble their integer codes first.
template <int BITS, int J>
__device__ __forceinline__ void chunk_pairs(const uint32_t lo[8], const uint32_t hi[2], uint32_t W[4]) {
  if (BITS == 8) {
    const uint32_t a = lo[2 * J], c = lo[2 * J + 1];
    W[0] = prmt(a, 0x64646464u, 0x4140u);
    W[1] = prmt(a, 0x64646464u, 0x4342u);
    W[2] = prmt(c, 0x64646464u, 0x4140u);
    W[3] = prmt(c, 0x64646464u, 0x4342u);
  } else if (BITS == 4) {
    const uint32_t L = lo[J] & 0x0F0F0F0Fu, Hh = (lo[J] >> 4) & 0x0F0F0F0Fu;
    W[0] = prmt(L, Hh, 0xC480u) | 0x64006400u;
    W[1] = prmt(L, Hh, 0xD591u) | 0x64006400u;
    W[2] = prmt(L, Hh, 0xE6A2u) | 0x64006400u;
    W[3] = prmt(L, Hh, 0xF7B3u) | 0x64006400u;
  } else {
    uint32_t u[8];
    if (BITS >= 4) {
#pragma unroll
      for (int v = 0; v < 8; ++v) u[v] = (lo[J] >> (4 * v)) & 15u;
    } else {
      const uint32_t w = lo[J >> 1] >> (16 * (J & 1));
#pragma unroll
      for (int v = 0; v < 8; ++v) u[v] = (w >> (2 * v)) & 3u;
    }
    if (BITS == 6) {
      const uint32_t h = hi[J >> 1] >> (16 * (J & 1));
#pragma unroll
      for (int v = 0; v < 8; ++v) u[v] |= ((h >> (2 * v)) & 3u) << 4;
    } else if (BITS == 5 || BITS == 3) {
      const uint32_t h = hi[0] >> (8 * J);
#pragma unroll
      for (int v = 0; v < 8; ++v) u[v] |= ((h >> v) & 1u) << (BITS == 5 ? 4 : 2);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) W[e] = u[2 * e] | (u[2 * e + 1] << 16) | 0x64006400u;
  }
}

// Dequantize block b of token t (32 values) into operand chunks 4b .. 4b+3 of
// row t: the hi image, and for keys (KEY) the lo image.  Invalid rows become
// zeros.  In fp16 pairs: the centred code c = (1024 + u) - (1024 + 2^(BITS-1)) is
// exact, hi = c * d is one rounding of the exact product and lo = fma(c, d, -hi)
// is the exact remainder (c*d has at most 19 significant bits, hi the top 11, so
// the rest fits fp16).  The _1 codecs' values u*d + m are taken in fp32 for keys
// (the reference's rounding, then hi and lo) and as one fp16 fma for values.
template <int BITS, bool ASYM, bool KEY>
__device__ __forceinline__ void dequant_block(const uint8_t* codes, const uint8_t* scales, int cb, int sb, int t,
                                              int b, bool valid, uint8_t* hi, uint8_t* lo) {
  uint32_t lw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}, hw[2] = {0u, 0u};
  __half2 D2 = __float2half2_rn(0.f), M2 = D2;
  if (valid) {
    block_planes<BITS, KEY>(codes, cb, t, b, lw, hw);
    if (ASYM) {
      const __half2 dm = *reinterpret_cast<const __half2*>(scales + t * sb + 4 * b);
      D2 = __low2half2(dm);
      M2 = __high2half2(dm);
    } else {
      D2 = __half2half2(*reinterpret_cast<const __half*>(scales + t * sb + 2 * b));
    }
  }
  const __half2 C0 = as_h2(ASYM ? 0x64006400u : (0x6400u + (1u << (BITS - 1))) * 0x10001u);
  const float d = __low2float(D2), m = __low2float(M2);
#define KVQ_PF_CHUNK(J)                                                                       \
  {                                                                                           \
    uint32_t W[4], H[4], L[4];                                                                \
    chunk_pairs<BITS, J>(lw, hw, W);                                                          \
    _Pragma("unroll") for (int e = 0; e < 4; ++e) {                                           \
      const __half2 C = __hsub2(as_h2(W[e]), C0);                                             \
      if (ASYM && KEY) {                                                                      \
        const float2 f = __half22float2(C);                                                   \
        const float x0 = fmaf(f.x, d, m), x1 = fmaf(f.y, d, m);                               \
        const __half2 hh = __floats2half2_rn(x0, x1);                                         \
        const float2 hf = __half22float2(hh);                                                 \
        H[e] = as_u32(hh);                                                                    \
        L[e] = as_u32(__floats2half2_rn(__fsub_rn(x0, hf.x), __fsub_rn(x1, hf.y)));           \
      } else if (ASYM) {                                                                      \
        H[e] = as_u32(__hfma2(C, D2, M2));                                                    \
      } else {                                                                                \
        const __half2 hh = __hmul2(C, D2);                                                    \
        H[e] = as_u32(hh);                                                                    \
        if (KEY) L[e] = as_u32(__hfma2(C, D2, __hneg2(hh)));                                  \
      }                                                                                       \
    }                                                                                         \
    const uint32_t o = op_off(t, 4 * b + J);                                                  \
    *reinterpret_cast<uint4*>(hi + o) = make_uint4(H[0], H[1], H[2], H[3]);                   \
    if (KEY) *reinterpret_cast<uint4*>(lo + o) = make_uint4(L[0], L[1], L[2], L[3]);          \
  }
  KVQ_PF_CHUNK(0)
  KVQ_PF_CHUNK(1)
  KVQ_PF_CHUNK(2)
  KVQ_PF_CHUNK(3)
#undef KVQ_PF_CHUNK
}

// A dequantizer thread's two units of a 64-token tile: unit u = dt + 128 k is
// (token t, block b), 8 neighbouring threads on 8 neighbouring tokens (their
// 16-byte stores fill 128 contiguous bytes).  Rows at or past nq_end hold no data.
template <int BITS, bool ASYM, bool KEY>
__device__ __forceinline__ void dequant_units(const uint8_t* codes, const uint8_t* scales, int cb, int sb, int dt,
                                              int tok0, int nq_end, uint8_t* hi, uint8_t* lo) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int u = dt + 128 * k;
    const int t = (u & 7) | ((u >> 5) << 3), b = (u >> 3) & 3;
    dequant_block<BITS, ASYM, KEY>(codes, scales, cb, sb, t, b, tok0 + t < nq_end, hi, lo);
  }
}

// One instantiation per block codec, chosen once per tile (the codec is the same
// for every unit of a CTA, so each CTA runs one branch).
template <bool KEY>
__device__ __forceinline__ void dequant_tile(int codec, const uint8_t* codes, const uint8_t* scales, int cb, int sb,
                                             int dt, int tok0, int nq_end, uint8_t* hi, uint8_t* lo) {
  switch (codec) {
#define KVQ_PF_CASE(C, B, A) \
  case C: dequant_units<B, A, KEY>(codes, scales, cb, sb, dt, tok0, nq_end, hi, lo); break;
    KVQ_PF_CASE(KVQ_Q8_0, 8, false)
    KVQ_PF_CASE(KVQ_Q6_0, 6, false)
    KVQ_PF_CASE(KVQ_Q5_0, 5, false)
    KVQ_PF_CASE(KVQ_Q4_0, 4, false)
    KVQ_PF_CASE(KVQ_Q3_0, 3, false)
    KVQ_PF_CASE(KVQ_Q2_0, 2, false)
    KVQ_PF_CASE(KVQ_Q8_1, 8, true)
    KVQ_PF_CASE(KVQ_Q6_1, 6, true)
    KVQ_PF_CASE(KVQ_Q5_1, 5, true)
    KVQ_PF_CASE(KVQ_Q4_1, 4, true)
    KVQ_PF_CASE(KVQ_Q3_1, 3, true)
    KVQ_PF_CASE(KVQ_Q2_1, 2, true)
#undef KVQ_PF_CASE
    default: break;
  }
}

struct PfBars {
  uint64_t* raw_full;    // [n_raw]
  uint64_t* raw_empty;   // [n_raw]
  uint64_t* op_full;     // [PF_NO]
  uint64_t* opk_empty;   // [PF_NO] keys of the stage read (S done)
  uint64_t* opv_empty;   // [PF_NO] values of the stage read (P V done)
  uint64_t* s_full;      // [2] S of the buffer's tile complete
  uint64_t* p_full;      // [2] P of the buffer's tile in tensor memory
  uint64_t* p_empty;     // [2] P V of the buffer's tile complete (S buffer free again)
  uint64_t* q_ready;
  uint64_t* done;
};

// 2^x with the SFU's approximate instruction (relative error ~2^-22; 2^-inf = 0).
__device__ __forceinline__ float pf_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait shared by all roles: gives up at once once another role has
// aborted, and aborts the CTA on a timeout.  pf_wait1: one thread;
// pf_wait: a whole warp (warp-uniform result).
__device__ __forceinline__ bool pf_wait1(uint64_t* bar, uint32_t parity, const PrefillParams& p,
                                         volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity, p.wait_ns)) return true;
  *abort_flag = 1;
  atomicOr(p.err, ERR_TIMEOUT);
  return false;
}
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, const PrefillParams& p,
                                        volatile int* abort_flag) {
  return __all_sync(0xffffffffu, pf_wait1(bar, parity, p, abort_flag));
}

}  // namespace

__global__ void __launch_bounds__(PF_THREADS, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = (int)gridDim.x - 1 - (int)blockIdx.x;   // latest (longest) query blocks first
  const int head = blockIdx.y;
  const HeadInfo h = p.heads[head];
  const int G = p.G;
  const int q0 = qb * p.QB;                              // first query of the block
  const int nqb = min(p.QB, p.n_q - q0);                 // queries in the block
  const int P0 = p.len - p.n_q + q0;                     // its position
  const int vis_end = P0 + nqb;                          // positions the last query sees: [0, vis_end)
  const int n_qt = (min(p.nq_all, vis_end) + PF_TOK - 1) / PF_TOK;
  const int n_tt = (max(0, vis_end - p.nq_all) + PF_TOK - 1) / PF_TOK;
  const int n_tiles = n_qt + n_tt;
  const int NR = p.n_raw;
  const bool rotated = p.rot != KVQ_ROT_NONE;

  uint8_t* sOp = smem;                                   // [PF_NO][V | K hi | K lo]
  uint8_t* sRaw = smem + PF_OFF_RAW;                     // [NR] raw page-heads
  uint64_t* barmem = reinterpret_cast<uint64_t*>(sRaw + (size_t)NR * p.stage_bytes);
  PfBars B;
  B.raw_full = barmem;              // 0-3
  B.raw_empty = barmem + 4;         // 4-7
  B.op_full = barmem + 8;           // 8-10
  B.opk_empty = barmem + 11;        // 11-13
  B.opv_empty = barmem + 14;        // 14-16
  B.s_full = barmem + 17;           // 17-18
  B.p_full = barmem + 19;           // 19-20
  B.p_empty = barmem + 21;          // 21-22
  B.q_ready = barmem + 23;
  B.done = barmem + 24;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(barmem + 25);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(barmem + 26);

  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(PF_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    if (lane == 0) {
      for (int i = 0; i < NR; ++i) { mbar_init(&B.raw_full[i], 1); mbar_init(&B.raw_empty[i], 4); }
      for (int i = 0; i < PF_NO; ++i) {
        mbar_init(&B.op_full[i], 4); mbar_init(&B.opk_empty[i], 1); mbar_init(&B.opv_empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) { mbar_init(&B.s_full[i], 1); mbar_init(&B.p_full[i], 4); mbar_init(&B.p_empty[i], 1); }
      mbar_init(B.q_ready, 4);
      mbar_init(B.done, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    // lane j reads the block-table entry of tile i0 + j; lane 0 issues the copies
    int issued = 0;
    int pids = 0;
    for (int i = 0; i < n_qt; ++i) {
      if ((i & 31) == 0) {
        pids = 0;
        if (i + lane < n_qt) {
          pids = p.bt[i + lane];
          if (pids < 0) { atomicOr(p.err, ERR_NO_PAGE); pids = 0; }
        }
      }
      const int pid = __shfl_sync(0xffffffffu, pids, i & 31);
      const int st = i % NR;
      if (i >= NR && !pf_wait(&B.raw_empty[st], ((i / NR) - 1) & 1, p, abort_flag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&B.raw_full[st], h.bytes);
        bulk_g2s(sRaw + (size_t)st * p.stage_bytes, p.pool + (size_t)pid * p.page_bytes + h.off, h.bytes,
                 &B.raw_full[st]);
      }
      issued = i + 1;
    }
    // no copy may still be landing when the CTA exits
    if (lane == 0)
      for (int i = max(0, issued - NR); i < issued; ++i)
        if (!mbar_wait(&B.raw_full[i % NR], (i / NR) & 1, p.wait_ns)) atomicOr(p.err, ERR_TIMEOUT);
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idS = umma_idesc(PF_TOK, false), idPV = umma_idesc(D, true);
      const uint32_t aOp = smem_u32(sOp);
      bool ok = pf_wait1(B.q_ready, 0, p, abort_flag);
      tc_fence_after();
      auto issue_s = [&](int i) {                       // S = Q' K^T of tile i (A: q' from tensor memory)
        const int st = i % PF_NO;
        const uint32_t kh = aOp + (uint32_t)st * PF_OP_BYTES + PF_TILE_BYTES, kl = kh + PF_TILE_BYTES;
        const uint32_t dS = tmem + (uint32_t)(i & 1) * PF_TOK;
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t ko = (uint32_t)(s >> 2) * 8192u + (uint32_t)(s & 3) * 32u;
          const uint64_t bh = umma_desc_sw128(kh + ko, 16, 1024), bl = umma_desc_sw128(kl + ko, 16, 1024);
          umma_f16_tmem_a(dS, tmem + PF_QH_COL + 8 * s, bh, idS, s > 0 ? 1u : 0u);
          umma_f16_tmem_a(dS, tmem + PF_QL_COL + 8 * s, bh, idS, 1u);
          umma_f16_tmem_a(dS, tmem + PF_QH_COL + 8 * s, bl, idS, 1u);
        }
        umma_commit(&B.s_full[i & 1]);
        umma_commit(&B.opk_empty[st]);
      };
      auto issue_pv = [&](int i) {                      // O += P V of tile i (A: P from tensor memory)
        const int st = i % PF_NO;
        const uint32_t v0 = aOp + (uint32_t)st * PF_OP_BYTES;
        const uint32_t pa = tmem + (uint32_t)(i & 1) * PF_TOK;
#pragma unroll
        for (int s = 0; s < PF_TOK / 16; ++s)
          umma_f16_tmem_a(tmem + PF_O_COL, pa + 8 * s, umma_desc_sw128(v0 + 2048 * s, 8192, 1024), idPV,
                          (i > 0 || s > 0) ? 1u : 0u);
        umma_commit(&B.p_empty[i & 1]);
        umma_commit(&B.opv_empty[st]);
      };
      // Issue whichever product is ready, polling without suspending: P V of
      // tile np once its P is in tensor memory (np < ns), else S of tile ns once
      // its operands are in and P V of tile ns - 2 (the last reader of the S/P
      // columns it overwrites) has completed.  No phase of these barriers can run
      // ahead of the issue order, so each parity names one completion.
      int ns = 0, np = 0;
      uint64_t t_last = globaltimer_ns();
      while (ok && np < n_tiles) {
        bool progress = false;
        if (np < ns && mbar_test_wait(&B.p_full[np & 1], (np >> 1) & 1)) {
          tc_fence_after();
          issue_pv(np++);
          progress = true;
        } else if (ns < n_tiles && mbar_test_wait(&B.op_full[ns % PF_NO], (ns / PF_NO) & 1) &&
                   (ns < 2 || mbar_test_wait(&B.p_empty[ns & 1], ((ns >> 1) - 1) & 1))) {
          tc_fence_after();
          issue_s(ns++);
          progress = true;
        }
        if (progress) {
          t_last = globaltimer_ns();
        } else if (*abort_flag) {
          ok = false;
        } else if (globaltimer_ns() - t_last > p.wait_ns) {
          *abort_flag = 1;
          atomicOr(p.err, ERR_TIMEOUT);
          ok = false;
        }
      }
      // nothing of this CTA may still run on the tensor cores when it exits
      umma_commit(B.done);
      if (!mbar_wait(B.done, 0, p.wait_ns)) atomicOr(p.err, ERR_TIMEOUT);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- dequantizers
    const int dt = threadIdx.x - 128;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % PF_NO;
      const uint32_t prev = ((i / PF_NO) - 1) & 1;      // phase of the stage's previous tile
      uint8_t* opV = sOp + (size_t)st * PF_OP_BYTES;
      uint8_t* opKh = opV + PF_TILE_BYTES;
      uint8_t* opKl = opKh + PF_TILE_BYTES;
      if (i < n_qt) {
        const int rs = i % NR;
        if (!pf_wait(&B.raw_full[rs], (i / NR) & 1, p, abort_flag)) break;
        if (i >= PF_NO && !pf_wait(&B.opk_empty[st], prev, p, abort_flag)) break;
        const uint8_t* kcodes = sRaw + (size_t)rs * p.stage_bytes;
        const uint8_t* kscales = kcodes + PAGE * h.cbK;
        const uint8_t* vcodes = kscales + PAGE * h.sbK;
        const uint8_t* vscales = vcodes + PAGE * h.cbV;
        dequant_tile<true>(h.kcodec, kcodes, kscales, h.cbK, h.sbK, dt, i * PF_TOK, p.nq_all, opKh, opKl);
        if (i >= PF_NO && !pf_wait(&B.opv_empty[st], prev, p, abort_flag)) break;
        dequant_tile<false>(h.vcodec, vcodes, vscales, h.cbV, h.sbV, dt, i * PF_TOK, p.nq_all, opV, nullptr);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.raw_empty[rs]);
          mbar_arrive(&B.op_full[st]);
        }
      } else {
        // tail tile: thread dt takes key row dt (dt < 64) or value row dt - 64,
        // reads it from the ring and brings it into the quantized rows' basis
        const int r = dt & 63, kv = dt >> 6;            // warp-uniform: warps 4, 5 keys, 6, 7 values
        if (i >= PF_NO && !pf_wait(kv ? &B.opv_empty[st] : &B.opk_empty[st], prev, p, abort_flag)) break;
        const int pos = p.nq_all + (i - n_qt) * PF_TOK + r;
        float x[D];
        if (pos < vis_end) {
          const int slot = pos % p.T;
          const uint8_t* tp = p.ring + (size_t)head * p.T * (D * 2 * 2) + (size_t)(slot / TAIL_TOK) * TAIL_PAGE_BYTES;
          const int s16 = slot % TAIL_TOK;
#pragma unroll
          for (int c8 = 0; c8 < 16; ++c8) {
            const uint8_t* src = kv == 0 ? tp + (c8 * TAIL_TOK + s16) * 16 : tp + TAIL_TOK * D * 2 + s16 * (D * 2) + c8 * 16;
            const uint4 w = *reinterpret_cast<const uint4*>(src);
            const float2 a = raw2_to_float2(w.x, p.bf16), bq = raw2_to_float2(w.y, p.bf16);
            const float2 c = raw2_to_float2(w.z, p.bf16), e = raw2_to_float2(w.w, p.bf16);
            x[8 * c8 + 0] = a.x; x[8 * c8 + 1] = a.y; x[8 * c8 + 2] = bq.x; x[8 * c8 + 3] = bq.y;
            x[8 * c8 + 4] = c.x; x[8 * c8 + 5] = c.y; x[8 * c8 + 6] = e.x; x[8 * c8 + 7] = e.y;
          }
          if (rotated) {
            if (p.inv_s) {
              const float* sc = p.inv_s + ((size_t)head * 2 + kv) * D;
#pragma unroll
              for (int c = 0; c < D; ++c) x[c] = __fmul_rn(x[c], sc[c]);
            }
            fwht128(x);
          }
        } else {
#pragma unroll
          for (int c = 0; c < D; ++c) x[c] = 0.f;
        }
#pragma unroll
        for (int c8 = 0; c8 < 16; ++c8)
          split8(x + 8 * c8, kv == 0 ? opKh : opV, kv == 0 ? opKl : nullptr, op_off(r, c8));
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.op_full[st]);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax (rows)
    const int row = threadIdx.x;
    const int j = row / G, g = row - j * G;
    const bool valid = j < p.QB && j < nqb;
    const int pos_r = valid ? P0 + j : vis_end - 1;      // padding rows see what the block sees
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    {
      // query image in tensor memory: q' = R (s_k * q) * scale (log2 units), fp16 hi and lo
      float x[D];
      if (valid) {
        const __half* src = p.q + ((size_t)(q0 + j) * p.Hq + (size_t)head * G + g) * D;
#pragma unroll
        for (int c8 = 0; c8 < 16; ++c8) {
          const uint4 w = *reinterpret_cast<const uint4*>(src + 8 * c8);
          const float2 a = raw2_to_float2(w.x, p.bf16), bq = raw2_to_float2(w.y, p.bf16);
          const float2 c = raw2_to_float2(w.z, p.bf16), e = raw2_to_float2(w.w, p.bf16);
          x[8 * c8 + 0] = a.x; x[8 * c8 + 1] = a.y; x[8 * c8 + 2] = bq.x; x[8 * c8 + 3] = bq.y;
          x[8 * c8 + 4] = c.x; x[8 * c8 + 5] = c.y; x[8 * c8 + 6] = e.x; x[8 * c8 + 7] = e.y;
        }
        if (rotated) {
          if (p.s_k) {
            const float* sk = p.s_k + (size_t)head * D;
#pragma unroll
            for (int c = 0; c < D; ++c) x[c] *= sk[c];
          }
          fwht128(x);
        }
#pragma unroll
        for (int c = 0; c < D; ++c) x[c] *= p.qscale;
      } else {
#pragma unroll
        for (int c = 0; c < D; ++c) x[c] = 0.f;
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {             // columns of 64 values each
        uint32_t hw[32], lw[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float a = x[64 * half + 2 * e], bq = x[64 * half + 2 * e + 1];
          const __half2 hh = __floats2half2_rn(a, bq);
          const float2 hf = __half22float2(hh);
          hw[e] = as_u32(hh);
          lw[e] = as_u32(__floats2half2_rn(__fsub_rn(a, hf.x), __fsub_rn(bq, hf.y)));
        }
        tmem_st32(lane_base + PF_QH_COL + 32 * half, hw);
        tmem_st32(lane_base + PF_QL_COL + 32 * half, lw);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.q_ready);
    }
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int b = i & 1;
      if (!pf_wait(&B.s_full[b], (i >> 1) & 1, p, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float s[PF_TOK];
      {
        uint32_t r[32];
        tmem_ld32(lane_base + (uint32_t)b * PF_TOK, r);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(r[c]);
        tmem_ld32(lane_base + (uint32_t)b * PF_TOK + 32, r);
#pragma unroll
        for (int c = 0; c < 32; ++c) s[32 + c] = __uint_as_float(r[c]);
      }
      // causal mask and the end of the tile's segment (quantized rows, tail rows)
      const bool quant = i < n_qt;
      const int tok0 = quant ? i * PF_TOK : p.nq_all + (i - n_qt) * PF_TOK;
      const int lim = min(pos_r + 1, quant ? p.nq_all : p.len) - tok0;
      if (lim < PF_TOK) {
#pragma unroll
        for (int c = 0; c < PF_TOK; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mt = s[0];
#pragma unroll
      for (int c = 1; c < PF_TOK; ++c) mt = fmaxf(mt, s[c]);
      float alpha = 1.f;
      if (mt > m_run + PF_RESCALE) {                   // also the first tile (m_run = -inf)
        alpha = pf_ex2(m_run - mt);
        l *= alpha;
        m_run = mt;
      }
      uint32_t pw[PF_TOK / 2];
      float ls = 0.f;
#pragma unroll
      for (int e = 0; e < PF_TOK / 2; ++e) {
        const float a = pf_ex2(s[2 * e] - m_run), bq = pf_ex2(s[2 * e + 1] - m_run);
        ls += a + bq;
        pw[e] = as_u32(__floats2half2_rn(a, bq));
      }
      l += ls;
      // O is touched only by a rescale, which waits for P V of the previous tile
      if (i >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!pf_wait(&B.p_empty[(i - 1) & 1], ((i - 1) >> 1) & 1, p, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(lane_base + PF_O_COL + c0, r);
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
          tmem_st32(lane_base + PF_O_COL + c0, r);
        }
      }
      // P over the first half of this tile's S columns (S is in registers)
      tmem_st32(lane_base + (uint32_t)b * PF_TOK, pw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_full[b]);
    }
    // ---- epilogue: O / l, back to the original basis
    if (ok && n_tiles > 0 && pf_wait(&B.p_empty[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, p, abort_flag)) {
      tc_fence_after();
      float x[D];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + PF_O_COL + c0, r);
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c0 + c] = __uint_as_float(r[c]);
      }
      if (rotated) {
        fwht128(x);
        if (p.s_v) {
          const float* sv = p.s_v + (size_t)head * D;
#pragma unroll
          for (int c = 0; c < D; ++c) x[c] *= sv[c];
        }
      }
      if (valid) {
        const float invL = 1.0f / l;
        float* dst = p.out + ((size_t)(q0 + j) * p.Hq + (size_t)head * G + g) * D;
#pragma unroll
        for (int c = 0; c < D; c += 4)
          *reinterpret_cast<float4*>(dst + c) = make_float4(x[c] * invL, x[c + 1] * invL, x[c + 2] * invL, x[c + 3] * invL);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(PF_TMEM_COLS) : "memory");
  }
}

size_t prefill_smem_bytes(int stage_bytes, int n_raw) { return (size_t)PF_OFF_RAW + (size_t)n_raw * stage_bytes + PF_MISC; }

int prefill_raw_stages(int stage_bytes) {
  if (stage_bytes <= 0 || stage_bytes % 128) return 0;
  int n = (PF_SMEM_MAX - PF_OFF_RAW - PF_MISC) / stage_bytes;
  n = n > 4 ? 4 : n;
  return n >= 2 ? n : 0;
}

cudaError_t launch_prefill(const PrefillParams& p, cudaStream_t s) {
  if (p.n_q <= 0) return cudaSuccess;
  // the shared-memory opt-in is a property of the kernel on the current device:
  // set it on every launch (a host call; the plan may live on any device)
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM_MAX);
  if (e != cudaSuccess) return e;
  const int n_blocks = (p.n_q + p.QB - 1) / p.QB;
  dim3 grid(n_blocks, p.Hkv);
  prefill_kernel<<<grid, PF_THREADS, prefill_smem_bytes(p.stage_bytes, p.n_raw), s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
