// Per-head projection of the rank/bit codec on the 5th-generation tensor cores.
//
// KV-COBRA explainer, §The news: each key is projected, rotated and quantized
// with frozen per-head settings, the rotation "fused into the same projection
// matrix" -- z = M_h x with M_h = R_r P_h^T (r x 128).  For a tile of 128 rows
// of one head this is a [128 x 128] x [128 x r] GEMM: the one place where the
// hot path is a dense contraction, so it runs as tcgen05.mma (kind::f16,
// fp32 accumulation in tensor memory).
//
//  * A (the fp16 rows) is exact in fp16.  M_h is split into fp16 hi + lo
//    (hi = fp16(M), lo = fp16(M - hi)), two MMAs per K step accumulate into the
//    same TMEM columns, so z carries ~22 bits of M.
//  * Operands live in shared memory in the canonical K-major layout without
//    swizzle: 8-row x 16-byte core matrices, K-adjacent core matrices 128 B apart
//    (leading byte offset), 8-row groups 2048 B apart (stride byte offset).  The
//    host prebuilds M_h's hi/lo images in exactly this layout, fetched with one
//    bulk copy; the A tile is gathered by the CTA's threads.
//  * One thread issues the 16 MMAs (8 K steps x hi/lo) and commits them to an
//    mbarrier; the epilogue reads the accumulator with tcgen05.ld (warp w owns
//    TMEM lanes 32w..32w+31 = rows), stages z in shared memory and runs the same
//    warp quantizer as the rotation path.
// Every wait is bounded; on a timeout the kernel latches an error bit, still
// frees its tensor memory and returns.
#include "kvq_internal.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace kvq {

namespace {

constexpr int TILE_M = 128;
constexpr int A_BYTES = TILE_M * D * 2;   // 32 KiB

__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version for sm_100; base offset 0, no swizzle
  return d;
}

// kind::f16 instruction descriptor: D fp32, A and B fp16, both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t umma_idesc_f16(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TILE_M >> 4) << 24);
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

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* out) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) out[i] = __uint_as_float(r[i]);
}

}  // namespace

__global__ void __launch_bounds__(128, 1) proj_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int head = p.z_out ? p.head_override : (int)blockIdx.y;
  const int kv = p.z_out ? p.kv_override : (int)blockIdx.z;
  const HeadInfo h = p.heads[head];
  const int codec = kv ? h.vcodec : h.kcodec;
  if (codec != KVQ_RANK) return;                      // F16 heads of a projection plan: append kernel
  const int r = h.r;
  const int bits = kv ? h.vbits : h.kbits;
  const uint32_t bbytes = (uint32_t)r * 256u;         // one fp16 image of M_h (r x 128)
  const uint32_t ncols = r <= 32 ? 32u : (r <= 64 ? 64u : 128u);

  uint8_t* sA = smem;                                  // 32 KiB, later reused for z
  uint8_t* sB = smem + A_BYTES;                        // hi image then lo image
  size_t off = A_BYTES + 2 * (size_t)bbytes;
  const uint8_t** rbase = reinterpret_cast<const uint8_t**>(smem + off); off += TILE_M * sizeof(void*);
  int* rstride = reinterpret_cast<int*>(smem + off); off += TILE_M * 4;
  int* rpos = reinterpret_cast<int*>(smem + off); off += TILE_M * 4;
  int* rseq = reinterpret_cast<int*>(smem + off); off += TILE_M * 4;
  off = (off + 15) & ~(size_t)15;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + off); off += 16;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + off);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  // ---- row sources: row i of the tile is quantize item tile*128 + i
  {
    const int q = tile * TILE_M + tid;
    const uint8_t* base = nullptr;
    int stride = 16, pos = -1, seq = -1;
    if (q < p.total_q) {
      if (p.z_out) {
        base = reinterpret_cast<const uint8_t*>(p.k_in + (size_t)q * p.in_stride);
        pos = q;
      } else {
        int si = 0;
        for (int i = 1; i < p.n_seqs; ++i)
          if (p.seqs[i].qitem0 <= q) si = i;
        const AppendSeq& sq = p.seqs[si];
        const int li = q - sq.qitem0;
        seq = sq.seq;
        const __half* in = kv ? p.v_in : p.k_in;
        if (li < sq.nE) {                                // from the tail ring
          pos = sq.e0 + li;
          const int slot = pos % p.T;
          const uint8_t* ring =
              p.tail + (((size_t)sq.seq * p.L + p.layer) * p.Hkv + head) * (size_t)p.T * (D * 2 * 2);
          const uint8_t* tp = ring + (size_t)(slot / TAIL_TOK) * TAIL_PAGE_BYTES;
          if (kv == 0) { base = tp + (slot % TAIL_TOK) * 16; stride = TAIL_TOK * 16; }
          else { base = tp + TAIL_TOK * D * 2 + (slot % TAIL_TOK) * (D * 2); }
        } else {                                         // straight from the input
          pos = sq.len_old + (li - sq.nE);
          const int row = sq.in_row0 + (pos - sq.len_old);
          base = reinterpret_cast<const uint8_t*>(in + (size_t)row * p.in_stride + (size_t)head * D);
        }
      }
    }
    rbase[tid] = base; rstride[tid] = stride; rpos[tid] = pos; rseq[tid] = seq;
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;

  if (tid == 0) {
    mbar_arrive_expect_tx(&bar[0], 2 * bbytes);
    bulk_g2s(sB, p.mimg + h.mimg_off, 2 * bbytes, &bar[0]);
  }
  // ---- A tile in the canonical layout: 128 rows x 16 chunks of 16 bytes
  for (int idx = tid; idx < TILE_M * 16; idx += 128) {
    const int row = idx >> 4, c = idx & 15;
    const uint8_t* b = rbase[row];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (b) v = *reinterpret_cast<const uint4*>(b + (size_t)c * rstride[row]);
    *reinterpret_cast<uint4*>(sA + ((row >> 3) * 16 + c) * 128 + (row & 7) * 16) = v;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();

  bool ok = true;
  if (tid == 0) {
    if (!mbar_wait(&bar[0], 0)) { atomicOr(p.err, ERR_TIMEOUT); ok = false; }
    if (ok) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t idesc = umma_idesc_f16(r);
      const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        umma_f16(tmem, umma_smem_desc(a0 + s * 256, 128, 2048), umma_smem_desc(b0 + s * 256, 128, 2048), idesc,
                 s > 0 ? 1u : 0u);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        umma_f16(tmem, umma_smem_desc(a0 + s * 256, 128, 2048), umma_smem_desc(b0 + bbytes + s * 256, 128, 2048),
                 idesc, 1u);
      umma_commit(&bar[1]);
    }
  }
  __syncthreads();
  // Wait for the accumulator (every thread polls the same barrier, bounded).
  if (!mbar_wait(&bar[1], 0)) {
    if (tid == 0) atomicOr(p.err, ERR_TIMEOUT);
    ok = false;
  }
  ok = __syncthreads_and(ok);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

  float* zs = reinterpret_cast<float*>(smem);          // [128][r+1], over A and B (no longer read)
  const int zst = r + 1;
  if (ok) {
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    for (int c0 = 0; c0 < r; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + lane_base + (uint32_t)c0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) zs[(32 * warp + lane) * zst + c0 + j] = v[j];
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
  if (!ok) return;

  // ---- epilogue: warp w quantizes (or exports) rows 32w .. 32w+31
  for (int i = 0; i < 32; ++i) {
    const int row = 32 * warp + i;
    const int pos = rpos[row];
    if (pos < 0) continue;
    float x[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = (4 * lane + k < r) ? zs[row * zst + 4 * lane + k] : 0.f;
    if (p.z_out) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (4 * lane + k < r) p.z_out[(size_t)pos * r + 4 * lane + k] = x[k];
      continue;
    }
    const int pid = p.block_table[(size_t)rseq[row] * p.max_pages_per_seq + pos / PAGE];
    if (pid < 0) {
      if (lane == 0) atomicOr(p.err, ERR_NO_PAGE);
      continue;
    }
    uint8_t* region = p.pool + (size_t)pid * p.page_bytes + h.off;
    uint8_t* codes = kv ? region + PAGE * (h.cbK + h.sbK) : region;
    const int cb = kv ? h.cbV : h.cbK;
    uint8_t* scales = codes + PAGE * cb;
    quantize_store_row(x, KVQ_RANK, r, bits, codes, scales, pos % PAGE, kv == 0);
  }
}

size_t proj_smem_bytes(int r) {
  size_t off = A_BYTES + 2 * (size_t)r * 256;
  off += TILE_M * (sizeof(void*) + 12);
  off = (off + 15) & ~(size_t)15;
  off += 16 + 16;
  const size_t zbytes = (size_t)TILE_M * (r + 1) * 4;
  return off > zbytes ? off : zbytes + 64;
}

cudaError_t launch_project(const ProjParams& p, int n_tiles, int n_heads, cudaStream_t s) {
  if (n_tiles <= 0) return cudaSuccess;
  size_t smem = proj_smem_bytes(128);
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(n_tiles, p.z_out ? 1 : n_heads, p.z_out ? 1 : 2);
  proj_kernel<<<grid, 128, smem, s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
