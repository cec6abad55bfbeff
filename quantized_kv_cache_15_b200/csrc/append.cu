// Append-quantize: new K/V rows enter the F16 precision tail; rows leaving the
// tail (or every row without a tail) are transformed and block-quantized into
// the paged cache.
//
// BeeLlama v0.4.0 news, §KV cache 精度尾部 (the newest tokens stay F16, the rest
// is quantized) and §核心新特性：KVarN (variance normalisation + rotation);
// KV-COBRA explainer, §Jargon (Hadamard rotation) and §The news (each key is
// projected, rotated and quantized with frozen per-head settings).
//
// One warp per (work item, kv head, K|V).  For a sequence with len_old cached
// tokens, n new tokens and a tail of T:
//   E (evicted): positions [e0, e0+nE) leave the ring: read slot, quantize to a page,
//                then write the slot's final new occupant (same warp: no race);
//   P (pass-through): positions [len_old, len_old+nP) go straight from the input
//                to a page (only when n > T - ... i.e. they never stay in the tail);
//   F (final tail occupants): positions [f0, f0+nF) are copied into the ring,
//                unless their slot belongs to an E warp.
#include "kvq_internal.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace kvq {

// Byte address of a tail ring row's lane piece (8 bytes = 4 fp16 values).
__device__ __forceinline__ uint8_t* ring_lane_ptr(uint8_t* ring, int slot, int kv) {
  const int lane = threadIdx.x & 31;
  uint8_t* tp = ring + (size_t)(slot / TAIL_TOK) * TAIL_PAGE_BYTES;
  const int row = slot % TAIL_TOK;
  if (kv == 0) return tp + ((lane >> 1) * TAIL_TOK + row) * 16 + (lane & 1) * 8;   // interleaved, cb = 256
  return tp + TAIL_TOK * D * 2 + row * (D * 2) + 8 * lane;                          // row-major
}

__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p) {
  // launched as a programmatic dependent (see ptx.cuh): set up while the previous
  // kernel drains, then wait for it before touching global data
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const long gw = (long)blockIdx.x * 8 + wib;
  const int per_item = p.Hkv * 2;
  const long item = gw / per_item;
  if (item >= p.total_items) return;
  const int rem = (int)(gw % per_item);
  const int head = rem >> 1, kv = rem & 1;
  int si = 0;
  for (int i = 1; i < p.n_seqs; ++i)
    if (p.seqs[i].item0 <= item) si = i;
  const AppendSeq& sq = p.seqs[si];
  const int li = (int)(item - sq.item0);
  const HeadInfo& h = p.heads[head];
  const int codec = kv ? h.vcodec : h.kcodec;
  const int bits = kv ? h.vbits : h.kbits;
  const int cb = kv ? h.cbV : h.cbK;
  const int sb = kv ? h.sbV : h.sbK;
  const __half* in = kv ? p.v_in : p.k_in;
  const int T = p.T;
  uint8_t* ring = (T > 0) ? p.tail + (((size_t)sq.seq * p.L + p.layer) * p.Hkv + head) * (size_t)T * (D * 2 * 2)
                          : nullptr;
  const float* inv_s = p.inv_s ? p.inv_s + ((size_t)head * 2 + kv) * D : nullptr;
  // rank-codec rows are quantized by the tensor-core kernel, which runs first
  const bool quantize_here = codec != KVQ_RANK;

  int pos;          // position to quantize (-1: none)
  int src_row = -1; // input row index, or -1 when the source is the ring
  int ring_slot = -1;
  int write_slot = -1, write_row = -1;  // ring write after the quantization
  if (li < sq.nE) {
    pos = sq.e0 + li;
    ring_slot = pos % T;
    int k = ((ring_slot - sq.f0) % T + T) % T;
    if (k < sq.nF) { write_slot = ring_slot; write_row = sq.in_row0 + (sq.f0 + k - sq.len_old); }
  } else if (li < sq.nE + sq.nP) {
    pos = sq.len_old + (li - sq.nE);
    src_row = sq.in_row0 + (pos - sq.len_old);
  } else {
    pos = -1;
    const int w = sq.f0 + (li - sq.nE - sq.nP);
    const int slot = w % T;
    const int k = ((slot - sq.e0) % T + T) % T;
    if (k < sq.nE) return;                       // the E warp of this slot writes it
    write_slot = slot; write_row = sq.in_row0 + (w - sq.len_old);
  }

  if (pos >= 0 && quantize_here) {
    float x[4];
    if (ring_slot >= 0) {
      uint2 v = *reinterpret_cast<const uint2*>(ring_lane_ptr(ring, ring_slot, kv));
      float2 fa = __half22float2(*reinterpret_cast<__half2*>(&v.x));
      float2 fb = __half22float2(*reinterpret_cast<__half2*>(&v.y));
      x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
    } else {
      load_row_f16(in + ((size_t)src_row * p.Hkv + head) * D, x);
    }
    transform_row(x, codec, p.rot, inv_s);
    const int lp = pos / PAGE;
    int pid = p.block_table[(size_t)sq.seq * p.max_pages_per_seq + lp];
    if (pid < 0) {
      if (lane == 0) atomicOr(p.err, ERR_NO_PAGE);
      return;
    }
    uint8_t* region = p.pool + (size_t)pid * p.page_bytes + h.off;
    uint8_t* codes = kv ? region + PAGE * (h.cbK + h.sbK) : region;
    uint8_t* scales = codes + PAGE * cb;
    quantize_store_row(x, codec, h.r, bits, codes, scales, pos % PAGE, kv == 0);
    (void)sb;
  }
  if (write_slot >= 0) {
    const uint2 v = *reinterpret_cast<const uint2*>(in + ((size_t)write_row * p.Hkv + head) * D + 4 * lane);
    *reinterpret_cast<uint2*>(ring_lane_ptr(ring, write_slot, kv)) = v;
  }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  if (p.total_items <= 0) return cudaSuccess;
  const long warps = (long)p.total_items * p.Hkv * 2;
  const long blocks = (warps + 7) / 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, append_kernel, p);
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
__global__ void debug_rotate_kernel(HeadInfo h, int rot, int kv, const float* inv_s, int n, const __half* x,
                                    float* y) {
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + wib;
  if (row >= n) return;
  const int codec = kv ? h.vcodec : h.kcodec;
  float v[4];
  load_row_f16(x + (size_t)row * D, v);
  transform_row(v, codec, rot, inv_s);
#pragma unroll
  for (int i = 0; i < 4; ++i) y[(size_t)row * D + 4 * lane + i] = v[i];
}
cudaError_t launch_debug_rotate(const HeadInfo& h, int rot, int kv, const float* inv_s, int n, const __half* x,
                                float* y, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  debug_rotate_kernel<<<(n + 7) / 8, 256, 0, s>>>(h, rot, kv, inv_s, n, x, y);
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
cudaError_t launch_debug_quantize(int codec, int r, int b, int n, const float* y, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  debug_quantize_kernel<<<(n + 7) / 8, 256, 0, s>>>(codec, r, b, n, y, codes, scales);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
