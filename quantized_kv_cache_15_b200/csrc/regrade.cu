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

__global__ void __launch_bounds__(256) regrade_kernel(const __grid_constant__ RegradeParams p) {
  const int lane = threadIdx.x & 31;
  const long gw = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long row = gw / (p.Hkv * 2);
  if (row >= p.total_rows) return;
  const int rem = (int)(gw % (p.Hkv * 2));
  const int head = rem >> 1, kv = rem & 1;
  int si = 0;
  for (int i = 1; i < p.n_seqs; ++i)
    if (p.row0[i] <= row) si = i;
  const long pos = row - p.row0[si];
  const int pid = p.block_table[(size_t)p.seq[si] * p.max_pages_per_seq + pos / PAGE];
  if (pid < 0) {
    if (lane == 0) atomicOr(p.err, ERR_NO_PAGE);
    return;
  }
  const int t = (int)(pos % PAGE);
  const HeadInfo& hs = p.src[head];
  const HeadInfo& hd = p.dst[head];
  const int cs = kv ? hs.vcodec : hs.kcodec, bs = kv ? hs.vbits : hs.kbits;
  const int cd = kv ? hd.vcodec : hd.kcodec, bd = kv ? hd.vbits : hd.kbits;
  const int cbs = kv ? hs.cbV : hs.cbK, sbs = kv ? hs.sbV : hs.sbK;
  const uint8_t* region = p.src_pool + (size_t)pid * p.src_page_bytes + hs.off;
  const uint8_t* codes = kv ? region + PAGE * (hs.cbK + hs.sbK) : region;
  const uint8_t* scales = codes + PAGE * cbs;
  float x[4];
  if (cs == KVQ_F16) {
    const uint8_t* src = codes + (kv == 0 ? kplane_off(cbs, t, 8 * lane) : t * cbs + 8 * lane);
    const uint2 w = *reinterpret_cast<const uint2*>(src);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    transform_row(x, cd, p.rot, p.inv_s ? p.inv_s + ((size_t)head * 2 + kv) * D : nullptr);
  } else {
    // exact dequantization in the stored basis: _0 code * d, _1 u * d + m
    uint32_t u[4];
    lane_codes(codes, cbs, t, kv == 0, bs, D, lane, u);
    const int b = (4 * lane) / 32;
    float d, off;
    if (codec_is_asym(cs)) {
      const __half2 dm = *reinterpret_cast<const __half2*>(scales + t * sbs + 4 * b);
      d = __low2float(dm);
      off = __high2float(dm);
    } else {
      d = __half2float(*reinterpret_cast<const __half*>(scales + t * sbs + 2 * b));
      off = -(float)(1 << (bs - 1)) * d;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = fmaf((float)u[i], d, off);
  }
  uint8_t* dregion = p.dst_pool + (size_t)pid * p.dst_page_bytes + hd.off;
  const int cbd = kv ? hd.cbV : hd.cbK;
  uint8_t* dcodes = kv ? dregion + PAGE * (hd.cbK + hd.sbK) : dregion;
  uint8_t* dscales = dcodes + PAGE * cbd;
  quantize_store_row(x, cd, D, bd, dcodes, dscales, t, kv == 0);
}

cudaError_t launch_regrade(const RegradeParams& p, cudaStream_t s) {
  if (p.total_rows <= 0) return cudaSuccess;
  const long warps = p.total_rows * p.Hkv * 2;
  regrade_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
