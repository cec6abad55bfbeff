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
// Keys and values are dequantized once per CTA into fp16 operands in shared
// memory, in the stored (rotated) basis: y = d * (u - 2^(b-1)) for the _0
// codecs, y = u * d + m for the _1 codecs, each one correctly rounded fp32
// operation as in the reference dequantizer.  fp16 holds 11 significant bits,
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
// Warp roles (320 threads, one CTA per SM: 211 KiB of shared memory at most):
//   warps 0-3  softmax: thread = row = TMEM lane; query image, online softmax
//              with a lazy rescale (O is rescaled only when the running max
//              grows by more than 8 in log2 units), P to shared memory, and the
//              epilogue;
//   warps 4-7  dequantizers: quantized tiles from the raw ring, tail tiles
//              straight from the ring in global memory, into the operand ring;
//   warp 8     producer: one cp.async.bulk per 64-token page-head into the raw ring;
//   warp 9     tensor memory allocation and, on one thread, the MMA issue: S of
//              tile i is issued before P V of tile i-1, so the softmax of tile i
//              overlaps the value product of the tile before.
// Operands use the canonical no-swizzle layouts: 8-row x 16-byte core matrices;
// an operand "tile" of 64 tokens x 128 channels stores element (t, c) at byte
// ((t/8)*16 + c/8)*128 + (t%8)*16 + (c%8)*2.  Read as K-major with rows = tokens
// (keys: B of S) the leading byte offset is 128 and the stride byte offset 2048;
// read as MN-major with N = channels and K = tokens (values: B of P V) the
// 8-channel groups are 128 bytes apart (stride byte offset) and the 8-token
// groups 2048 (leading byte offset).
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
constexpr int PF_Q_BYTES = PF_ROWS * D * 2;            // one fp16 image of the 128 query rows
constexpr int PF_TILE_BYTES = PF_TOK * D * 2;          // one fp16 image of a 64-token tile
constexpr int PF_OP_BYTES = 3 * PF_TILE_BYTES;         // V, K hi, K lo
constexpr int PF_P_BYTES = PF_ROWS * PF_TOK * 2;
constexpr int PF_OFF_OP = 2 * PF_Q_BYTES;
constexpr int PF_OFF_P = PF_OFF_OP + 2 * PF_OP_BYTES;
constexpr int PF_OFF_RAW = PF_OFF_P + PF_P_BYTES;      // 180224
constexpr int PF_MISC = 256;                           // barriers, TMEM address, abort flag
constexpr int PF_SMEM_MAX = 232448;                    // 227 KiB opt-in per CTA
constexpr uint32_t PF_TMEM_COLS = 256;                 // S double buffer (2 x 64) + O (128)
constexpr uint32_t PF_O_COL = 128;
constexpr float PF_RESCALE = 8.0f;                     // lazy rescale threshold (log2 units)

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version for sm_100; base offset 0, no swizzle
  return d;
}
// kind::f16 instruction descriptor: D fp32, A and B fp16, A K-major, B K-major or
// MN-major, M = 128, N = n.
__device__ __forceinline__ uint32_t umma_idesc(int n, bool b_mn_major) {
  return (1u << 4) | (b_mn_major ? (1u << 16) : 0u) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(PF_ROWS >> 4) << 24);
}
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
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

// Byte offset of 16-byte chunk c8 (channels 8 c8 .. 8 c8 + 7) of row t in an
// operand image (64-token tiles and the 128-row query image alike).
__device__ __forceinline__ uint32_t op_off(int t, int c8) { return (uint32_t)((((t >> 3) << 4) + c8) << 7) + ((t & 7) << 4); }

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
__device__ __forceinline__ void block_planes(const uint8_t* codes, bool kplane, int cb, int t, int b, int bits,
                                             uint32_t lo[8], uint32_t hi[2]) {
  auto at = [&](int o) -> const uint8_t* {
    return kplane ? codes + ((((o >> 4) * PAGE + t) << 4) + (o & 15)) : codes + t * cb + o;
  };
  if (bits == 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(at(32 * b));
    const uint4 c = *reinterpret_cast<const uint4*>(at(32 * b + 16));
    lo[0] = a.x; lo[1] = a.y; lo[2] = a.z; lo[3] = a.w; lo[4] = c.x; lo[5] = c.y; lo[6] = c.z; lo[7] = c.w;
  } else if (bits >= 4) {                          // 4, 5, 6: nibble plane first
    const uint4 a = *reinterpret_cast<const uint4*>(at(16 * b));
    lo[0] = a.x; lo[1] = a.y; lo[2] = a.z; lo[3] = a.w;
  } else {                                         // 2, 3: 2-bit plane first
    const uint2 a = *reinterpret_cast<const uint2*>(at(8 * b));
    lo[0] = a.x; lo[1] = a.y;
  }
  if (bits == 6) {
    const uint2 h = *reinterpret_cast<const uint2*>(at(64 + 8 * b));
    hi[0] = h.x; hi[1] = h.y;
  } else if (bits == 5) {
    hi[0] = *reinterpret_cast<const uint32_t*>(at(64 + 4 * b));
  } else if (bits == 3) {
    hi[0] = *reinterpret_cast<const uint32_t*>(at(32 + 4 * b));
  }
}

// The 8 codes of channels 8 j8 .. 8 j8 + 7 of a block (j8 a compile-time index).
template <int J8>
__device__ __forceinline__ void chunk_codes(int bits, const uint32_t lo[8], const uint32_t hi[2], uint32_t u[8]) {
  if (bits == 8) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      u[v] = (lo[2 * J8] >> (8 * v)) & 255u;
      u[4 + v] = (lo[2 * J8 + 1] >> (8 * v)) & 255u;
    }
  } else if (bits >= 4) {
#pragma unroll
    for (int v = 0; v < 8; ++v) u[v] = (lo[J8] >> (4 * v)) & 15u;
  } else {
    const uint32_t w = lo[J8 >> 1] >> (16 * (J8 & 1));
#pragma unroll
    for (int v = 0; v < 8; ++v) u[v] = (w >> (2 * v)) & 3u;
  }
  if (bits == 6) {
    const uint32_t h = hi[J8 >> 1] >> (16 * (J8 & 1));
#pragma unroll
    for (int v = 0; v < 8; ++v) u[v] |= ((h >> (2 * v)) & 3u) << 4;
  } else if (bits == 5 || bits == 3) {
    const uint32_t h = hi[0] >> (8 * J8);
    const int sh = bits == 5 ? 4 : 2;
#pragma unroll
    for (int v = 0; v < 8; ++v) u[v] |= ((h >> v) & 1u) << sh;
  }
}

// Dequantize block b of token t (32 values) of one plane into operand chunks
// 4b .. 4b+3 of row t: hi image (and lo image for keys).  Invalid rows become zeros.
__device__ __forceinline__ void dequant_block(const uint8_t* codes, const uint8_t* scales, bool kplane, int cb,
                                              int sb, int bits, bool asym, int t, int b, bool valid, uint8_t* hi,
                                              uint8_t* lo) {
  uint32_t lw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}, hw[2] = {0u, 0u};
  float d = 0.f, off = 0.f;
  if (valid) {
    block_planes(codes, kplane, cb, t, b, bits, lw, hw);
    if (asym) {
      const __half2 dm = *reinterpret_cast<const __half2*>(scales + t * sb + 4 * b);
      d = __low2float(dm);
      off = __high2float(dm);
    } else {
      d = __half2float(*reinterpret_cast<const __half*>(scales + t * sb + 2 * b));
      off = -(float)(1 << (bits - 1)) * d;
    }
  }
  uint32_t u[8];
  float x[8];
#define KVQ_PF_CHUNK(J)                                                   \
  chunk_codes<J>(bits, lw, hw, u);                                        \
  _Pragma("unroll") for (int v = 0; v < 8; ++v) x[v] = fmaf((float)u[v], d, off); \
  split8(x, hi, lo, op_off(t, 4 * b + J));
  KVQ_PF_CHUNK(0)
  KVQ_PF_CHUNK(1)
  KVQ_PF_CHUNK(2)
  KVQ_PF_CHUNK(3)
#undef KVQ_PF_CHUNK
}

struct PfBars {
  uint64_t* raw_full;    // [n_raw]
  uint64_t* raw_empty;   // [n_raw]
  uint64_t* op_full;     // [2]
  uint64_t* op_empty;    // [2]
  uint64_t* s_full;      // [2]
  uint64_t* s_empty;     // [2]
  uint64_t* p_full;
  uint64_t* p_empty;
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

  uint8_t* sQh = smem;
  uint8_t* sQl = smem + PF_Q_BYTES;
  uint8_t* sOp = smem + PF_OFF_OP;                       // [2][V | K hi | K lo]
  uint8_t* sP = smem + PF_OFF_P;
  uint8_t* sRaw = smem + PF_OFF_RAW;
  uint64_t* barmem = reinterpret_cast<uint64_t*>(sRaw + (size_t)NR * p.stage_bytes);
  PfBars B;
  B.raw_full = barmem;
  B.raw_empty = barmem + 4;
  B.op_full = barmem + 8;
  B.op_empty = barmem + 10;
  B.s_full = barmem + 12;
  B.s_empty = barmem + 14;
  B.p_full = barmem + 16;
  B.p_empty = barmem + 17;
  B.q_ready = barmem + 18;
  B.done = barmem + 19;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(barmem + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(barmem + 21);

  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(PF_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    if (lane == 0) {
      for (int i = 0; i < NR; ++i) { mbar_init(&B.raw_full[i], 1); mbar_init(&B.raw_empty[i], 4); }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&B.op_full[i], 4); mbar_init(&B.op_empty[i], 1);
        mbar_init(&B.s_full[i], 1); mbar_init(&B.s_empty[i], 4);
      }
      mbar_init(B.p_full, 4);
      mbar_init(B.p_empty, 1);
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
      const uint32_t aQh = smem_u32(sQh), aQl = smem_u32(sQl), aP = smem_u32(sP), aOp = smem_u32(sOp);
      bool ok = pf_wait1(B.q_ready, 0, p, abort_flag);
      auto issue_pv = [&](int i) {                      // O += P V of tile i
        const uint32_t v0 = aOp + (uint32_t)(i & 1) * PF_OP_BYTES;
#pragma unroll
        for (int s = 0; s < PF_TOK / 16; ++s)
          umma_f16(tmem + PF_O_COL, umma_desc(aP + 256 * s, 128, 1024), umma_desc(v0 + 4096 * s, 2048, 128), idPV,
                   (i > 0 || s > 0) ? 1u : 0u);
        umma_commit(B.p_empty);
        umma_commit(&B.op_empty[i & 1]);
      };
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int b = i & 1;
        if (!pf_wait1(&B.op_full[b], (i >> 1) & 1, p, abort_flag)) break;
        if (i >= 2 && !pf_wait1(&B.s_empty[b], ((i >> 1) - 1) & 1, p, abort_flag)) break;
        tc_fence_after();
        const uint32_t kh = aOp + (uint32_t)b * PF_OP_BYTES + PF_TILE_BYTES, kl = kh + PF_TILE_BYTES;
        const uint32_t dS = tmem + (uint32_t)b * PF_TOK;
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint64_t qh = umma_desc(aQh + 256 * s, 128, 2048), ql = umma_desc(aQl + 256 * s, 128, 2048);
          const uint64_t bh = umma_desc(kh + 256 * s, 128, 2048), bl = umma_desc(kl + 256 * s, 128, 2048);
          umma_f16(dS, qh, bh, idS, s > 0 ? 1u : 0u);
          umma_f16(dS, ql, bh, idS, 1u);
          umma_f16(dS, qh, bl, idS, 1u);
        }
        umma_commit(&B.s_full[b]);
        if (i >= 1) {
          if (!pf_wait1(B.p_full, (i - 1) & 1, p, abort_flag)) break;
          tc_fence_after();
          issue_pv(i - 1);
        }
        if (i == n_tiles - 1) {
          if (!pf_wait1(B.p_full, i & 1, p, abort_flag)) break;
          tc_fence_after();
          issue_pv(i);
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
    const int kc = h.kcodec, vc = h.vcodec;
    const int kbits = h.kbits, vbits = h.vbits;
    const bool kasym = codec_is_asym(kc), vasym = codec_is_asym(vc);
    for (int i = 0; i < n_tiles; ++i) {
      const int b = i & 1;
      if (i >= 2 && !pf_wait(&B.op_empty[b], ((i >> 1) - 1) & 1, p, abort_flag)) break;
      uint8_t* opV = sOp + (size_t)b * PF_OP_BYTES;
      uint8_t* opKh = opV + PF_TILE_BYTES;
      uint8_t* opKl = opKh + PF_TILE_BYTES;
      if (i < n_qt) {
        const int st = i % NR;
        if (!pf_wait(&B.raw_full[st], (i / NR) & 1, p, abort_flag)) break;
        const uint8_t* kcodes = sRaw + (size_t)st * p.stage_bytes;
        const uint8_t* kscales = kcodes + PAGE * h.cbK;
        const uint8_t* vcodes = kscales + PAGE * h.sbK;
        const uint8_t* vscales = vcodes + PAGE * h.cbV;
#pragma unroll 1
        for (int k = 0; k < 2; ++k) {
          // unit (token t, block bb): 8 neighbouring threads take 8 neighbouring tokens
          const int u = dt + 128 * k;
          const int t = (u & 7) | ((u >> 5) << 3), bb = (u >> 3) & 3;
          const bool valid = i * PF_TOK + t < p.nq_all;   // rows past the last quantized row hold no data
          dequant_block(kcodes, kscales, true, h.cbK, h.sbK, kbits, kasym, t, bb, valid, opKh, opKl);
          dequant_block(vcodes, vscales, false, h.cbV, h.sbV, vbits, vasym, t, bb, valid, opV, nullptr);
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.raw_empty[st]);
          mbar_arrive(&B.op_full[b]);
        }
      } else {
        // tail tile: thread dt takes key row dt (dt < 64) or value row dt - 64,
        // reads it from the ring and brings it into the quantized rows' basis
        const int r = dt & 63, kv = dt >> 6;
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
              const float* s = p.inv_s + ((size_t)head * 2 + kv) * D;
#pragma unroll
              for (int c = 0; c < D; ++c) x[c] = __fmul_rn(x[c], s[c]);
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
        if (lane == 0) mbar_arrive(&B.op_full[b]);
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
      // query image: q' = R (s_k * q) * scale (log2 units), fp16 hi and lo
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
      for (int c8 = 0; c8 < 16; ++c8) split8(x + 8 * c8, sQh, sQl, op_off(row, c8));
      fence_proxy_async_shared();
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.s_empty[b]);
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
      // P's buffer and O are free once P V of the previous tile has completed
      if (i >= 1 && !pf_wait(B.p_empty, (i - 1) & 1, p, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (i >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(lane_base + PF_O_COL + c0, r);
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
          tmem_st32(lane_base + PF_O_COL + c0, r);
        }
        tmem_wait_st();
      }
      float ls = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < PF_TOK / 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = pf_ex2(s[8 * c8 + 2 * e] - m_run), bq = pf_ex2(s[8 * c8 + 2 * e + 1] - m_run);
          ls += a + bq;
          const __half2 hh = __floats2half2_rn(a, bq);
          w[e] = *reinterpret_cast<const uint32_t*>(&hh);
        }
        *reinterpret_cast<uint4*>(sP + (((row >> 3) * 8 + c8) << 7) + ((row & 7) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += ls;
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.p_full);
    }
    // ---- epilogue: O / l, back to the original basis
    if (ok && n_tiles > 0 && pf_wait(B.p_empty, (n_tiles - 1) & 1, p, abort_flag)) {
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
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM_MAX);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_blocks = (p.n_q + p.QB - 1) / p.QB;
  dim3 grid(n_blocks, p.Hkv);
  prefill_kernel<<<grid, PF_THREADS, prefill_smem_bytes(p.stage_bytes, p.n_raw), s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
