// Append-quantize: new K/V rows enter the F16 precision tail; rows leaving the
// tail (or every row without a tail) are transformed and block-quantized into
// the paged cache.
//
// BeeLlama v0.4.0 news, §KV cache 精度尾部 (the newest tokens stay F16, the rest
// is quantized) and §核心新特性：KVarN (variance normalisation + rotation);
// KV-COBRA explainer, §Jargon (Hadamard rotation) and §The news (each key is
// projected, rotated and quantized with frozen per-head settings).
//
// One warp (small appends) or four threads (chunks) per (work item, kv head,
// K|V).  For a sequence with len_old cached tokens, n new tokens and a tail of T:
//   E (evicted): positions [e0, e0+nE) leave the ring: read slot, quantize to a page,
//                then write the slot's final new occupant (same threads: no race);
//   P (pass-through): positions [len_old, len_old+nP) go straight from the input
//                to a page (only when n > T - ... i.e. they never stay in the tail);
//   F (final tail occupants): positions [f0, f0+nF) are copied into the ring,
//                unless their slot belongs to an E row.
#include "kvq_internal.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace kvq {

// What one (item, kv head, K|V) row of an append does.  Item kinds (the tail
// ring's E/P/F split, see AppendSeq): E quantizes the ring row leaving the tail
// (and refills its slot), P quantizes an input row, F only writes an input row
// into the ring.
struct RowWork {
  const AppendSeq* sq;
  int head, kv;
  int pos;          // position to quantize (-1: none)
  int src_row;      // input row index, or -1 when the source is the ring
  int ring_slot;    // ring slot read (E), or -1
  int write_slot;   // ring write after the quantization, or -1
  int write_row;
  uint8_t* ring;    // this (sequence, layer, kv head)'s tail ring
};

// Row `task` (consecutive tasks: consecutive items of one (kv head, K|V)).
// Returns false when the row has nothing to do.
__device__ __forceinline__ bool row_work(const AppendParams& p, long task, RowWork& w) {
  const long n_items = p.total_items;
  const int hk = (int)(task / n_items);
  const long item = task - (long)hk * n_items;
  w.head = hk >> 1;
  w.kv = hk & 1;
  // the sequence of this item: the last one whose first item is <= item
  int lo = 0, hi = p.n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seqs[mid].item0 <= item) lo = mid; else hi = mid - 1;
  }
  const AppendSeq& sq = p.seqs[lo];
  w.sq = &sq;
  const int li = (int)(item - sq.item0);
  const int T = p.T;
  w.ring = (T > 0) ? p.tail + (((size_t)sq.seq * p.L + p.layer) * p.Hkv + w.head) * (size_t)T * (D * 2 * 2)
                   : nullptr;
  w.src_row = -1; w.ring_slot = -1; w.write_slot = -1; w.write_row = -1;
  if (li < sq.nE) {
    w.pos = sq.e0 + li;
    w.ring_slot = w.pos % T;
    const int k = ((w.ring_slot - sq.f0) % T + T) % T;
    if (k < sq.nF) { w.write_slot = w.ring_slot; w.write_row = sq.in_row0 + (sq.f0 + k - sq.len_old); }
  } else if (li < sq.nE + sq.nP) {
    w.pos = sq.len_old + (li - sq.nE);
    w.src_row = sq.in_row0 + (w.pos - sq.len_old);
  } else {
    w.pos = -1;
    const int f = sq.f0 + (li - sq.nE - sq.nP);
    const int slot = f % T;
    const int k = ((slot - sq.e0) % T + T) % T;
    if (k < sq.nE) return false;                 // the E row of this slot writes it
    w.write_slot = slot; w.write_row = sq.in_row0 + (f - sq.len_old);
  }
  // rank-codec rows are quantized by the projection kernel, which runs first
  const HeadInfo& h = p.heads[w.head];
  if ((w.kv ? h.vcodec : h.kcodec) == KVQ_RANK) w.pos = -1;
  return true;
}

// 16-byte chunk c (0..15) of ring slot `slot`: a tail page holds TAIL_TOK rows,
// K interleaved in 16-byte chunks, V row-major.
__device__ __forceinline__ uint8_t* ring_chunk(uint8_t* ring, int slot, int kv, int c) {
  uint8_t* tp = ring + (size_t)(slot / TAIL_TOK) * TAIL_PAGE_BYTES;
  const int row = slot % TAIL_TOK;
  return kv == 0 ? tp + (c * TAIL_TOK + row) * 16 : tp + TAIL_TOK * D * 2 + row * (D * 2) + 16 * c;
}

// Destination page of a quantized position (the block-table entry; read before
// the row itself so that the two global loads are in flight together) and the
// page row's code and scale planes; false (and the error bit) when the block
// table has no page there.
__device__ __forceinline__ int page_of(const AppendParams& p, const RowWork& w) {
  return p.block_table[(size_t)w.sq->seq * p.max_pages_per_seq + w.pos / PAGE];
}
__device__ __forceinline__ bool page_row(const AppendParams& p, const RowWork& w, int pid, uint8_t** codes,
                                         uint8_t** scales, bool report) {
  if (pid < 0) {
    if (report) atomicOr(p.err, ERR_NO_PAGE);
    return false;
  }
  const HeadInfo& h = p.heads[w.head];
  uint8_t* region = p.pool + (size_t)pid * p.page_bytes + h.off;
  *codes = w.kv ? region + PAGE * (h.cbK + h.sbK) : region;
  *scales = *codes + PAGE * (w.kv ? h.cbV : h.cbK);
  return true;
}

// Small appends (a decode step's handful of rows): one warp per row, lane l
// holding values 4l .. 4l+3, so that a row's latency is a few hundred cycles.
__global__ void __launch_bounds__(256) append_warp_kernel(const __grid_constant__ AppendParams p) {
  // launched as a programmatic dependent (see ptx.cuh): set up while the previous
  // kernel drains, then wait for it before touching global data
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const long task = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (task >= (long)p.total_items * p.Hkv * 2) return;   // whole warps leave together
  RowWork w;
  if (!row_work(p, task, w)) return;
  const HeadInfo& h = p.heads[w.head];
  const int kv = w.kv;
  const __half* in = kv ? p.v_in : p.k_in;
  if (w.pos >= 0) {
    const int codec = kv ? h.vcodec : h.kcodec;
    const int pid = page_of(p, w);
    float x[4];
    if (w.ring_slot >= 0) {
      const uint2 r = *reinterpret_cast<const uint2*>(ring_chunk(w.ring, w.ring_slot, kv, lane >> 1) + 8 * (lane & 1));
      const float2 fa = raw2_to_float2(r.x, p.bf16), fb = raw2_to_float2(r.y, p.bf16);
      x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
    } else {
      load_row_raw(in + ((size_t)w.src_row * p.Hkv + w.head) * D, x, p.bf16);
    }
    transform_row(x, codec, p.rot, p.inv_s ? p.inv_s + ((size_t)w.head * 2 + kv) * D : nullptr);
    uint8_t *codes, *scales;
    if (!page_row(p, w, pid, &codes, &scales, lane == 0)) return;
    quantize_store_row(x, codec, h.r, kv ? h.vbits : h.kbits, codes, scales, w.pos % PAGE, kv == 0, p.bf16);
  }
  if (w.write_slot >= 0) {
    const uint2 r = *reinterpret_cast<const uint2*>(in + ((size_t)w.write_row * p.Hkv + w.head) * D + 4 * lane);
    *reinterpret_cast<uint2*>(ring_chunk(w.ring, w.write_slot, kv, lane >> 1) + 8 * (lane & 1)) = r;
  }
}

// Chunk appends: four threads per row, one 32-value block each (quad layout, see
// quant.cuh), so a row costs few instructions and no warp-wide shuffles;
// consecutive quads take consecutive items of one (kv head, K|V).
__global__ void __launch_bounds__(256) append_quad_kernel(const __grid_constant__ AppendParams p) {
  griddep_launch_dependents();
  griddep_wait();
  const int q = threadIdx.x & 3;
  const long task = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 2;
  if (task >= (long)p.total_items * p.Hkv * 2) return;   // whole quads leave together
  RowWork w;
  if (!row_work(p, task, w)) return;
  const HeadInfo& h = p.heads[w.head];
  const int kv = w.kv;
  const __half* in = kv ? p.v_in : p.k_in;
  if (w.pos >= 0) {
    const int codec = kv ? h.vcodec : h.kcodec;
    const int pid = page_of(p, w);
    uint4 r[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      r[c] = w.ring_slot >= 0
                 ? *reinterpret_cast<const uint4*>(ring_chunk(w.ring, w.ring_slot, kv, 4 * q + c))
                 : *reinterpret_cast<const uint4*>(in + ((size_t)w.src_row * p.Hkv + w.head) * D + 32 * q + 8 * c);
    uint8_t *codes, *scales;
    if (!page_row(p, w, pid, &codes, &scales, q == 0)) return;
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) chunk_to_float(r[c], v + 8 * c, p.bf16);
    if (codec != KVQ_F16)
      transform_row_quad(v, p.rot, p.inv_s ? p.inv_s + ((size_t)w.head * 2 + kv) * D : nullptr);
    quantize_row_quad(codec, v, codes, scales, w.pos % PAGE, kv == 0, kv ? h.cbV : h.cbK, kv ? h.sbV : h.sbK, p.bf16);
  }
  if (w.write_slot >= 0) {
    const uint4* src = reinterpret_cast<const uint4*>(in + ((size_t)w.write_row * p.Hkv + w.head) * D + 32 * q);
#pragma unroll
    for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(ring_chunk(w.ring, w.write_slot, kv, 4 * q + c)) = src[c];
  }
}

// Rows below which an append takes the warp-per-row kernel (its per-row latency
// is lower; above it the quad kernel's lower instruction count per row wins).
constexpr long APPEND_WARP_ROWS = 4096;

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  if (p.total_items <= 0) return cudaSuccess;
  const long rows = (long)p.total_items * p.Hkv * 2;
  const bool warp = rows < APPEND_WARP_ROWS;
  const long threads = rows * (warp ? 32 : 4);
  // small quad launches get narrow blocks so that the rows spread over more SMs
  const int bs = warp || threads >= 148L * 256 ? 256 : threads >= 148L * 128 ? 128 : threads >= 148L * 64 ? 64 : 32;
  const long blocks = (threads + bs - 1) / bs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, 1, 1);
  cfg.blockDim = dim3(bs, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = warp ? cudaLaunchKernelEx(&cfg, append_warp_kernel, p)
                             : cudaLaunchKernelEx(&cfg, append_quad_kernel, p);
  note_launches(1);
  return e;
}

// ---------------------------------------------------------------- block table
constexpr int BT_MAX = 256;
struct BlockTableUpdate {
  int* table;
  int n;
  int idx[BT_MAX];
  int val[BT_MAX];
};
__global__ void block_table_kernel(const __grid_constant__ BlockTableUpdate u) {
  const int i = threadIdx.x;
  if (i < u.n) u.table[u.idx[i]] = u.val[i];
}
cudaError_t launch_block_table_update(int* table, int n, const int* idx, const int* val, cudaStream_t s) {
  for (int k = 0; k < n; k += BT_MAX) {
    BlockTableUpdate u;
    u.table = table;
    u.n = (n - k) < BT_MAX ? (n - k) : BT_MAX;
    for (int i = 0; i < u.n; ++i) { u.idx[i] = idx[k + i]; u.val[i] = val[k + i]; }
    block_table_kernel<<<1, BT_MAX, 0, s>>>(u);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ---------------------------------------------------------------- calibration
// inv_rms[c] = fp32(1 / sqrt(sum_t x[t][c]^2 / n)) in double, tokens in order
// (BeeLlama v0.4.0 news, §KVarN); 1 where the RMS is below 1e-6.
__global__ void calibrate_kernel(int64_t n_tok, int n_ch, int64_t stride, const __half* x, float* inv) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n_ch) return;
  double s = 0.0;
  for (int64_t t = 0; t < n_tok; ++t) {
    double v = (double)__half2float(x[t * stride + c]);
    s = __dadd_rn(s, __dmul_rn(v, v));
  }
  double rms = __dsqrt_rn(__ddiv_rn(s, (double)n_tok));
  inv[c] = (rms < 1e-6) ? 1.0f : __double2float_rn(__ddiv_rn(1.0, rms));
}
cudaError_t launch_calibrate(int64_t n_tok, int n_ch, int64_t stride, const __half* x, float* inv, cudaStream_t s) {
  calibrate_kernel<<<(n_ch + 127) / 128, 128, 0, s>>>(n_tok, n_ch, stride, x, inv);
  note_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- debug hooks
// The row transform and the block quantizer alone, in either row layout.
__global__ void debug_rotate_kernel(HeadInfo h, int rot, int kv, const float* inv_s, int n, const __half* x,
                                    float* y, bool bf16) {
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + wib;
  if (row >= n) return;
  const int codec = kv ? h.vcodec : h.kcodec;
  float v[4];
  load_row_raw(x + (size_t)row * D, v, bf16);
  transform_row(v, codec, rot, inv_s);
#pragma unroll
  for (int i = 0; i < 4; ++i) y[(size_t)row * D + 4 * lane + i] = v[i];
}
__global__ void debug_rotate_quad_kernel(HeadInfo h, int rot, int kv, const float* inv_s, int n, const __half* x,
                                         float* y, bool bf16) {
  const int q = threadIdx.x & 3;
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 2;
  if (row >= n) return;                          // whole quads leave together
  const int codec = kv ? h.vcodec : h.kcodec;
  float v[32];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    chunk_to_float(*reinterpret_cast<const uint4*>(x + (size_t)row * D + 32 * q + 8 * c), v + 8 * c, bf16);
  if (codec != KVQ_F16) transform_row_quad(v, rot, inv_s);
#pragma unroll
  for (int i = 0; i < 32; ++i) y[(size_t)row * D + 32 * q + i] = v[i];
}
cudaError_t launch_debug_rotate(const HeadInfo& h, int rot, int kv, const float* inv_s, int n, const __half* x,
                                float* y, bool quad, bool bf16, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (quad)
    debug_rotate_quad_kernel<<<(n + 63) / 64, 256, 0, s>>>(h, rot, kv, inv_s, n, x, y, bf16);
  else
    debug_rotate_kernel<<<(n + 7) / 8, 256, 0, s>>>(h, rot, kv, inv_s, n, x, y, bf16);
  note_launches(1);
  return cudaGetLastError();
}

__global__ void debug_quantize_kernel(int codec, int r, int b, int n, const float* y, uint8_t* codes, uint8_t* scales) {
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + wib;
  if (row >= n) return;
  const int nin = codec == KVQ_RANK ? r : D;
  const int bits = codec == KVQ_RANK ? b : codec_bits(codec);
  int cb, sb;
  row_bytes(codec, r, b, &cb, &sb);
  float x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = (4 * lane + i < nin) ? y[(size_t)row * nin + 4 * lane + i] : 0.0f;
  quantize_store_row(x, codec, r, bits, codes + (size_t)row * cb, scales + (size_t)row * sb, 0, false);
}
__global__ void debug_quantize_quad_kernel(int codec, int n, const float* y, uint8_t* codes, uint8_t* scales) {
  const int q = threadIdx.x & 3;
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 2;
  if (row >= n) return;                          // whole quads leave together
  int cb, sb;
  row_bytes(codec, D, 0, &cb, &sb);
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = y[(size_t)row * D + 32 * q + i];
  quantize_row_quad(codec, v, codes + (size_t)row * cb, scales + (size_t)row * sb, 0, false, cb, sb);
}
cudaError_t launch_debug_quantize(int codec, int r, int b, int n, const float* y, uint8_t* codes, uint8_t* scales,
                                  bool quad, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (quad)
    debug_quantize_quad_kernel<<<(n + 63) / 64, 256, 0, s>>>(codec, n, y, codes, scales);
  else
    debug_quantize_kernel<<<(n + 7) / 8, 256, 0, s>>>(codec, r, b, n, y, codes, scales);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
