// Reading the cache back: rows in the original basis (kvq_dequantize) and the
// canonical packed rows (kvq_read_rows).
//
// Dequantization in the stored basis is exact (each value is one correctly
// rounded operation): _0 code*d, _1 u*d + m, rank (2u - (2^b-1)) * d/2, all of
// which are what fmaf(u, d, off) returns because u*d and off are exact.  The
// inverse transform then applies the staged Hadamard transform (times the
// per-channel variance multiplier) or M_h^T for the projection path.
#include "kvq_internal.h"
#include "quant.cuh"

namespace kvq {

__global__ void __launch_bounds__(256) dequant_kernel(const __grid_constant__ DecodeParams p, int seq, int len,
                                                      long t0, long n_rows, float* k_out, float* v_out) {
  __shared__ __align__(16) float zs[8][D];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const long gw = (long)blockIdx.x * 8 + wib;
  const long row = gw / (p.Hkv * 2);
  if (row >= n_rows) return;
  const int rem = (int)(gw % (p.Hkv * 2));
  const int head = rem >> 1, kv = rem & 1;
  float* out = kv ? v_out : k_out;
  if (!out) return;
  const long pos = t0 + row;
  const int T = p.T;
  const long nq = len > T ? len - T : 0;
  const HeadInfo& h = p.heads[head];
  float x[4];
  if (pos >= nq) {
    // tail ring, raw fp16
    const uint8_t* ring = p.tail + (((size_t)seq * p.L + p.layer) * p.Hkv + head) * (size_t)T * (D * 2 * 2);
    const int slot = (int)(pos % T);
    const uint8_t* tp = ring + (size_t)(slot / TAIL_TOK) * TAIL_PAGE_BYTES;
    const int r = slot % TAIL_TOK;
    const uint8_t* src = kv == 0 ? tp + ((lane >> 1) * TAIL_TOK + r) * 16 + (lane & 1) * 8
                                 : tp + TAIL_TOK * D * 2 + r * (D * 2) + 8 * lane;
    const uint2 w = *reinterpret_cast<const uint2*>(src);
    const float2 a = raw2_to_float2(w.x, p.bf16), b = raw2_to_float2(w.y, p.bf16);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else {
    const int codec = kv ? h.vcodec : h.kcodec;
    const int bits = kv ? h.vbits : h.kbits;
    const int cb = kv ? h.cbV : h.cbK, sb = kv ? h.sbV : h.sbK;
    const int pid = p.block_table[(size_t)seq * p.max_pages_per_seq + pos / PAGE];
    if (pid < 0) { if (lane == 0) atomicOr(p.err, ERR_NO_PAGE); return; }
    const uint8_t* region = p.pool + (size_t)pid * p.page_bytes + h.off;
    const uint8_t* codes = kv ? region + PAGE * (h.cbK + h.sbK) : region;
    const uint8_t* scales = codes + PAGE * cb;
    const int t = (int)(pos % PAGE);
    const int n = codec == KVQ_RANK ? h.r : D;
    if (codec == KVQ_F16) {
      const int o = 8 * lane;
      const uint8_t* src = codes + (kv == 0 ? kplane_off(cb, t, o) : t * cb + o);
      const uint2 w = *reinterpret_cast<const uint2*>(src);
      const float2 a = raw2_to_float2(w.x, p.bf16), b = raw2_to_float2(w.y, p.bf16);
      x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
      uint32_t u[4];
      if (4 * lane < n) lane_codes(codes, cb, t, kv == 0, bits, n, lane, u);
      else u[0] = u[1] = u[2] = u[3] = 0;
      const int blk = n < 32 ? n : 32;
      const int b = (4 * lane < n) ? (4 * lane) / blk : 0;
      float d, m = 0.f;
      if (codec_is_asym(codec)) {
        __half2 dm = *reinterpret_cast<const __half2*>(scales + t * sb + 4 * b);
        d = __low2float(dm); m = __high2float(dm);
      } else {
        d = __half2float(*reinterpret_cast<const __half*>(scales + t * sb + 2 * b));
      }
      float off;
      if (codec == KVQ_RANK) off = -0.5f * (float)((1 << bits) - 1) * d;
      else if (codec_is_asym(codec)) off = m;
      else off = -(float)(1 << (bits - 1)) * d;
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = (4 * lane + i < n) ? fmaf((float)u[i], d, off) : 0.f;
      if (codec == KVQ_RANK) {
        if (p.rot == KVQ_ROT_PROJECTION) {
#pragma unroll
          for (int i = 0; i < 4; ++i) zs[wib][4 * lane + i] = x[i];
          __syncwarp();
          const float* M = p.M + h.m_off;
          float y[4] = {0.f, 0.f, 0.f, 0.f};
          for (int i = 0; i < h.r; ++i) {
            const float z = zs[wib][i];
            float4 mr = *reinterpret_cast<const float4*>(M + (size_t)i * D + 4 * lane);
            y[0] = fmaf(mr.x, z, y[0]); y[1] = fmaf(mr.y, z, y[1]);
            y[2] = fmaf(mr.z, z, y[2]); y[3] = fmaf(mr.w, z, y[3]);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) x[i] = y[i];
        }
      } else if (p.rot != KVQ_ROT_NONE) {
        fwht_row(x);
        const float* s = kv ? p.s_v : p.s_k;
        if (s) {
#pragma unroll
          for (int i = 0; i < 4; ++i) x[i] *= s[(size_t)head * D + 4 * lane + i];
        }
      }
    }
  }
  float4 o = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4*>(out + ((size_t)row * p.Hkv + head) * D + 4 * lane) = o;
}

cudaError_t launch_dequantize(const DecodeParams& p, int seq, int64_t t0, int64_t t1, float* k_out, float* v_out,
                              cudaStream_t s) {
  const long n_rows = (long)(t1 - t0);
  if (n_rows <= 0) return cudaSuccess;
  const long warps = n_rows * p.Hkv * 2;
  dequant_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(p, seq, p.len[0], (long)t0, n_rows, k_out, v_out);
  note_launches(1);
  return cudaGetLastError();
}

__global__ void read_rows_kernel(const __grid_constant__ DecodeParams p, int seq, long t0, long n_rows, int kv,
                                 uint8_t* codes_out, uint8_t* scales_out) {
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const long gw = (long)blockIdx.x * 8 + wib;
  const long row = gw / p.Hkv;
  if (row >= n_rows) return;
  const int head = (int)(gw % p.Hkv);
  size_t coff = 0, soff = 0;
  for (int hh = 0; hh < head; ++hh) {
    coff += (size_t)n_rows * (kv ? p.heads[hh].cbV : p.heads[hh].cbK);
    soff += (size_t)n_rows * (kv ? p.heads[hh].sbV : p.heads[hh].sbK);
  }
  const HeadInfo& h = p.heads[head];
  const int cb = kv ? h.cbV : h.cbK, sb = kv ? h.sbV : h.sbK;
  const long pos = t0 + row;
  const int pid = p.block_table[(size_t)seq * p.max_pages_per_seq + pos / PAGE];
  if (pid < 0) { if (lane == 0) atomicOr(p.err, ERR_NO_PAGE); return; }
  const uint8_t* region = p.pool + (size_t)pid * p.page_bytes + h.off;
  const uint8_t* codes = kv ? region + PAGE * (h.cbK + h.sbK) : region;
  const uint8_t* scales = codes + PAGE * cb;
  const int t = (int)(pos % PAGE);
  for (int i = lane; i < cb; i += 32)
    codes_out[coff + (size_t)row * cb + i] = codes[kv == 0 ? kplane_off(cb, t, i) : t * cb + i];
  for (int i = lane; i < sb; i += 32) scales_out[soff + (size_t)row * sb + i] = scales[t * sb + i];
}

cudaError_t launch_read_rows(const DecodeParams& p, int seq, int64_t t0, int64_t t1, int kv, uint8_t* codes,
                             uint8_t* scales, cudaStream_t s) {
  const long n_rows = (long)(t1 - t0);
  if (n_rows <= 0) return cudaSuccess;
  const long warps = n_rows * p.Hkv;
  read_rows_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(p, seq, (long)t0, n_rows, kv, codes, scales);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
