// Per-head projection of the rank/bit codec: z = M_h x, then the block quantizer.
//
// KV-COBRA explainer, §The news: each key is projected, rotated and quantized
// with frozen per-head settings, the rotation folded into the projection matrix
// -- M_h = R_r P_h^T (r x 128, stored fp32).  §Jargon "Scalar quantization": a
// block's step and each value's level are integer decisions taken on z, so two
// ways of forming z that differ in the last bits can store different codes (one
// level, or one fp16 ulp of a step, apart), and a key or value one level off
// moves the attention output well past the parity bar at 1-2 bits.
//
// So z is formed exactly as its definition states it for fp32 M_h and fp16 x:
// each product M_rc x_c is exact in double (24 + 11 significant bits), the 128
// products are added in channel order c = 0 .. 127 in double, and the sum is
// rounded once to fp32.  With an exact product, a double FMA is that same
// multiply-then-add, so the kernel's z -- and therefore its codes and scales --
// are the definition's, bit for bit, whatever the rows.
//
// One CTA: one (kv head, K|V) and up to 64 rows.  M_h^T (double, [128][r]) and
// the rows (double, [64][128]) are staged in shared memory; warp w takes rows w,
// w + 8, ... four at a time, lane l holds outputs 4l .. 4l+3 of all four (sixteen
// independent FMA chains over c, each M_h^T load shared by four rows), and the
// warp then quantizes each row with the same warp quantizer as the rotation path
// (lane l: values 4l .. 4l+3).
#include "kvq_internal.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace kvq {

namespace {
constexpr int PJ_ROWS = 64;                  // rows per CTA
constexpr int PJ_WARPS = 8;
constexpr int PJ_THREADS = 32 * PJ_WARPS;
}  // namespace

size_t proj_smem_bytes(int r) {
  return (size_t)D * r * 8 + (size_t)PJ_ROWS * D * 8 + (size_t)PJ_ROWS * (sizeof(void*) + 12);
}

__global__ void __launch_bounds__(PJ_THREADS, 1) proj_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int head = p.z_out ? p.head_override : (int)blockIdx.y;
  const int kv = p.z_out ? p.kv_override : (int)blockIdx.z;
  const HeadInfo h = p.heads[head];
  const int codec = kv ? h.vcodec : h.kcodec;
  if (codec != KVQ_RANK) return;                      // F16 heads of a projection plan: append kernel
  const int r = h.r;
  const int bits = kv ? h.vbits : h.kbits;

  double* mt = reinterpret_cast<double*>(smem);                      // [128 c][r] = M_h^T
  double* xs = mt + (size_t)D * r;                                   // [64 rows][128 c]
  const uint8_t** rbase = reinterpret_cast<const uint8_t**>(xs + (size_t)PJ_ROWS * D);
  int* rstride = reinterpret_cast<int*>(rbase + PJ_ROWS);
  int* rpos = rstride + PJ_ROWS;
  int* rseq = rpos + PJ_ROWS;

  // ---- M_h^T (exact widening of the stored fp32 M_h, precomputed by the plan)
  {
    const double2* src = reinterpret_cast<const double2*>(p.mt + h.mt_off);
    double2* dst = reinterpret_cast<double2*>(mt);
    for (int i = tid; i < D * r / 2; i += PJ_THREADS) dst[i] = src[i];
  }
  // ---- row sources: row i of the tile is quantize item tile * 64 + i
  if (tid < PJ_ROWS) {
    const int q = tile * PJ_ROWS + tid;
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
  __syncthreads();
  // ---- rows into shared memory as doubles (fp16 widens exactly); 16 chunks of 8 values
  for (int idx = tid; idx < PJ_ROWS * 16; idx += PJ_THREADS) {
    const int row = idx >> 4, c = idx & 15;
    const uint8_t* b = rbase[row];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (b) v = *reinterpret_cast<const uint4*>(b + (size_t)c * rstride[row]);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    double* dst = xs + (size_t)row * D + 8 * c;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      dst[2 * k] = (double)f.x;
      dst[2 * k + 1] = (double)f.y;
    }
  }
  __syncthreads();

  const int i0 = 4 * lane;
  const bool own = i0 < r;
  constexpr int RPP = 4;                                  // rows per pass of a warp
  for (int k = 0; k < PJ_ROWS / (RPP * PJ_WARPS); ++k) {
    int rows[RPP];
    bool any = false;
#pragma unroll
    for (int j = 0; j < RPP; ++j) {
      rows[j] = warp + PJ_WARPS * (RPP * k + j);
      any = any || rpos[rows[j]] >= 0;
    }
    if (!any) continue;                                   // warp-uniform
    double acc[RPP][4];
#pragma unroll
    for (int j = 0; j < RPP; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = 0.0;
    if (own) {
#pragma unroll 2
      for (int c = 0; c < D; ++c) {
        const double2 m01 = *reinterpret_cast<const double2*>(mt + (size_t)c * r + i0);
        const double2 m23 = *reinterpret_cast<const double2*>(mt + (size_t)c * r + i0 + 2);
#pragma unroll
        for (int j = 0; j < RPP; ++j) {
          const double x = xs[(size_t)rows[j] * D + c];
          acc[j][0] = fma(m01.x, x, acc[j][0]); acc[j][1] = fma(m01.y, x, acc[j][1]);
          acc[j][2] = fma(m23.x, x, acc[j][2]); acc[j][3] = fma(m23.y, x, acc[j][3]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < RPP; ++j) {
      const int row = rows[j];
      const int pos = rpos[row];
      if (pos < 0) continue;                              // warp-uniform
      float z[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) z[e] = own ? (float)acc[j][e] : 0.f;
      if (p.z_out) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (i0 + e < r) p.z_out[(size_t)pos * r + i0 + e] = z[e];
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
      quantize_store_row(z, KVQ_RANK, r, bits, codes, scales, pos % PAGE, kv == 0);
    }
  }
}

cudaError_t launch_project(const ProjParams& p, int n_items, int n_heads, cudaStream_t s) {
  if (n_items <= 0) return cudaSuccess;
  const size_t smem = proj_smem_bytes(128);
  // the shared-memory opt-in is a property of the kernel on the current device:
  // set it on every launch (a host call; the plan may live on any device)
  cudaError_t e = cudaFuncSetAttribute(proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_tiles = (n_items + PJ_ROWS - 1) / PJ_ROWS;
  dim3 grid(n_tiles, p.z_out ? 1 : n_heads, p.z_out ? 1 : 2);
  proj_kernel<<<grid, PJ_THREADS, smem, s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
