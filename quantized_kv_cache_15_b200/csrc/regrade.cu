// VBR regrade: requantize every cached row of one layer to other codecs.
//
// "Introducing a new KV format: VBR (Variable Bit Rate)", first post: the cache
// is quantized layer by layer as the session grows (F16 first, then F16 / 8-bit
// mixes and so on), within a VRAM budget (--vbr-vram) and above a quality floor
// (--vbr-floor).  This kernel is the transcode step such a policy runs on one
// layer: each row of the quantized segment is brought to the stored basis (raw
// F16 rows through the layer's variance normalisation and Hadamard transform,
// block-codec rows dequantized exactly) and quantized with the layer's new
// codec into a scratch copy of the layer's pages in the new layout; the host
// then copies the scratch over the layer's pool.  Rows of the F16 tail are not
// touched: they stay raw until they leave the tail.
#include "kvq_internal.h"
#include "quant.cuh"

namespace kvq {

// Four threads per (row, kv head, K|V), one 32-value block each (quad layout:
// quant.cuh); consecutive quads take consecutive rows, so both pools are read and
// written in coalesced runs.
__global__ void __launch_bounds__(256) regrade_kernel(const __grid_constant__ RegradeParams p) {
  const long task = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 2;
  const int q = threadIdx.x & 3;
  if (task >= p.total_rows * p.Hkv * 2) return;  // whole quads leave together
  const int hk = (int)(task / p.total_rows);
  const long row = task - (long)hk * p.total_rows;
  const int head = hk >> 1, kv = hk & 1;
  int lo = 0, hi = p.n_seqs - 1;                 // the last sequence whose first row is <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.row0[mid] <= row) lo = mid; else hi = mid - 1;
  }
  const long pos = row - p.row0[lo];
  const int pid = p.block_table[(size_t)p.seq[lo] * p.max_pages_per_seq + pos / PAGE];
  if (pid < 0) {
    if (q == 0) atomicOr(p.err, ERR_NO_PAGE);
    return;
  }
  const int t = (int)(pos % PAGE);
  const bool kplane = kv == 0;
  const HeadInfo& hs = p.src[head];
  const HeadInfo& hd = p.dst[head];
  const int cs = kv ? hs.vcodec : hs.kcodec;
  const int cd = kv ? hd.vcodec : hd.kcodec;
  const int cbs = kv ? hs.cbV : hs.cbK, sbs = kv ? hs.sbV : hs.sbK;
  const uint8_t* region = p.src_pool + (size_t)pid * p.src_page_bytes + hs.off;
  const uint8_t* codes = kv ? region + PAGE * (hs.cbK + hs.sbK) : region;
  const uint8_t* scales = codes + PAGE * cbs;
  float v[32];
  switch (cs) {
    case KVQ_F16: {
      // raw rows: into the stored basis of the new codec
#pragma unroll
      for (int c = 0; c < 4; ++c)
        chunk_to_float(*reinterpret_cast<const uint4*>(row_word_ptr(codes, kplane, cbs, t, 16 * q + 4 * c)), v + 8 * c,
                       p.bf16);
      if (cd != KVQ_F16)
        transform_row_quad(v, p.rot, p.inv_s ? p.inv_s + ((size_t)head * 2 + kv) * D : nullptr);
    } break;
    case KVQ_Q8_0: dequantize_block_quad<0, 8>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q6_0: dequantize_block_quad<0, 6>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q5_0: dequantize_block_quad<0, 5>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q4_0: dequantize_block_quad<0, 4>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q3_0: dequantize_block_quad<0, 3>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q2_0: dequantize_block_quad<0, 2>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q8_1: dequantize_block_quad<1, 8>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q6_1: dequantize_block_quad<1, 6>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q5_1: dequantize_block_quad<1, 5>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q4_1: dequantize_block_quad<1, 4>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q3_1: dequantize_block_quad<1, 3>(codes, scales, t, kplane, cbs, sbs, v); break;
    case KVQ_Q2_1: dequantize_block_quad<1, 2>(codes, scales, t, kplane, cbs, sbs, v); break;
    default: return;
  }
  uint8_t* dregion = p.dst_pool + (size_t)pid * p.dst_page_bytes + hd.off;
  const int cbd = kv ? hd.cbV : hd.cbK, sbd = kv ? hd.sbV : hd.sbK;
  uint8_t* dcodes = kv ? dregion + PAGE * (hd.cbK + hd.sbK) : dregion;
  uint8_t* dscales = dcodes + PAGE * cbd;
  quantize_row_quad(cd, v, dcodes, dscales, t, kplane, cbd, sbd, p.bf16);
}

cudaError_t launch_regrade(const RegradeParams& p, cudaStream_t s) {
  if (p.total_rows <= 0) return cudaSuccess;
  const long threads = 4L * p.total_rows * p.Hkv * 2;
  regrade_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
