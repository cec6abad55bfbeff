// Decode attention over the paged, quantized cache: one new query token per
// sequence attends over every cached token of its kv head (grouped-query
// attention: G query heads share a kv head).
//
// Forum thread on KV compression (attention paragraph): dot the query with every
// prior key, softmax, weighted average of the values -- and (bandwidth
// paragraph) decode is bound by the bytes it must read, which is why the cache
// is read once, in its packed form, and dequantized in registers.
// BeeLlama v0.4.0 news, §KV cache 精度尾部: the tail segment is F16.
//
// Work split (split-K): a sequence's pages are cut into splits, first the
// quantized pages, pps per split, then the tail pages, pps_t per split (never
// mixed in one split).  One CTA per (split, kv head) in a 1-D grid ordered longest
// first (decode_item), so the CTAs the hardware starts last are the short ones and
// the launch ends evenly.  Each CTA:
//   * warp 4 (producer) streams one page-head region per tile into a ring of
//     shared-memory stages with cp.async.bulk (completion on mbarriers);
//   * warps 0-3 (consumers) take tiles round-robin, each keeping its own online
//     softmax state (max m, sum l, accumulator) for the G heads;
//   * the four states are merged, then either finalised (single split) or
//     written as a partial; the last CTA of the (sequence, kv head) -- found with
//     an atomic ticket, no waiting -- merges all partials in split order and
//     applies the inverse transform of the value basis.
// Scores are kept in log2 units: q' carries softmax_scale * log2(e).
//
// The key score uses the stored basis: q . khat = (R (s_k * q)) . yhat for the
// rotated paths (R symmetric orthogonal), (M_h q) . zhat for the projection, and
// the raw q for F16 rows.  Per block, yhat = d*u + off, so
//   q'.yhat_block = d * sum_j q'_j u_j + off * sum_j q'_j
// with sum_j q'_j precomputed per block (qsum).
#include <cfloat>
#include <map>
#include <mutex>
#include <tuple>

#include "decode_fast.cuh"
#include "kvq_internal.h"
#include "ptx.cuh"
#include "quant.cuh"

namespace kvq {

enum { BASIS_RAW = 0, BASIS_ROT = 1, BASIS_PROJ = 2 };

__host__ __device__ inline int basis_of(int codec, int rot) {
  if (codec == KVQ_F16 || rot == KVQ_ROT_NONE) return BASIS_RAW;
  if (codec == KVQ_RANK) return BASIS_PROJ;
  return BASIS_ROT;
}

// Warp-wide maximum of a float in one integer reduction: the map x -> key (the
// bits, with the magnitude bits flipped for negative x) is monotone from floats to
// int32, so the max of the keys is the key of the max (exact; no NaNs here).
__device__ __forceinline__ float warp_max(float v) {
  const int i = __float_as_int(v);
  const int m = __reduce_max_sync(0xffffffffu, i >= 0 ? i : (i ^ 0x7FFFFFFF));
  return __int_as_float(m >= 0 ? m : (m ^ 0x7FFFFFFF));
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// Offset term of a block: yhat = d*u + off.
__device__ __forceinline__ float block_off(int codec, int bits, float d, float m) {
  if (codec == KVQ_RANK) return -0.5f * (float)((1 << bits) - 1) * d;
  if (codec_is_asym(codec)) return m;
  return -(float)(1 << (bits - 1)) * d;
}

// Code j (0..n-1) of token t from an interleaved K plane (generic path).
__device__ __forceinline__ uint32_t kcode_generic(const uint8_t* kp, int cb, int t, int bits, int n, int j) {
  switch (bits) {
    case 8: return kp[kplane_off(cb, t, j)];
    case 4: return (kp[kplane_off(cb, t, j >> 1)] >> (4 * (j & 1))) & 15u;
    case 2: return (kp[kplane_off(cb, t, j >> 2)] >> (2 * (j & 3))) & 3u;
    case 1: return (kp[kplane_off(cb, t, j >> 3)] >> (j & 7)) & 1u;
    case 6: {
      uint32_t lo = (kp[kplane_off(cb, t, j >> 1)] >> (4 * (j & 1))) & 15u;
      uint32_t hi = (kp[kplane_off(cb, t, n / 2 + (j >> 2))] >> (2 * (j & 3))) & 3u;
      return lo | (hi << 4);
    }
    case 5: {
      uint32_t lo = (kp[kplane_off(cb, t, j >> 1)] >> (4 * (j & 1))) & 15u;
      uint32_t hi = (kp[kplane_off(cb, t, n / 2 + (j >> 3))] >> (j & 7)) & 1u;
      return lo | (hi << 4);
    }
    case 3: {
      uint32_t lo = (kp[kplane_off(cb, t, j >> 2)] >> (2 * (j & 3))) & 3u;
      uint32_t hi = (kp[kplane_off(cb, t, n / 4 + (j >> 3))] >> (j & 7)) & 1u;
      return lo | (hi << 2);
    }
    default: return 0;
  }
}

// Scores of token t for the G heads (log2 units).
template <int G>
__device__ __forceinline__ void score_token(int kc, int kbits, int n, int cb, int sb, const uint8_t* kp,
                                            const uint8_t* ks, int t, const float* __restrict__ qv,
                                            const float* __restrict__ qsum, float s[G], int rows, bool bf16) {
#pragma unroll
  for (int g = 0; g < G; ++g) s[g] = 0.f;
  if (kc == KVQ_F16) {
    if (t >= rows) return;                 // past the end of a tail tile (TAIL_TOK rows)
#pragma unroll 2
    for (int c = 0; c < 16; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(kp + (c * rows + t) * 16);
      float x[8];
      chunk_to_float(v, x, bf16);
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int j = 0; j < 8; ++j) s[g] = fmaf(qv[g * D + 8 * c + j], x[j], s[g]);
    }
    return;
  }
  const int blk = n < 32 ? n : 32;
  const int nb = n / blk;
  const bool asym = codec_is_asym(kc);
  for (int b = 0; b < nb; ++b) {
    float a[G];
#pragma unroll
    for (int g = 0; g < G; ++g) a[g] = 0.f;
    if (kc != KVQ_RANK && kbits == 8) {
      uint4 v0 = *reinterpret_cast<const uint4*>(kp + ((2 * b) * PAGE + t) * 16);
      uint4 v1 = *reinterpret_cast<const uint4*>(kp + ((2 * b + 1) * PAGE + t) * 16);
      uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float u = (float)((w[k] >> (8 * i)) & 0xffu);
#pragma unroll
          for (int g = 0; g < G; ++g) a[g] = fmaf(qv[g * D + 32 * b + 4 * k + i], u, a[g]);
        }
    } else if (kc != KVQ_RANK && kbits == 4) {
      uint4 v = *reinterpret_cast<const uint4*>(kp + (b * PAGE + t) * 16);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float u = (float)((w[k] >> (4 * i)) & 15u);
#pragma unroll
          for (int g = 0; g < G; ++g) a[g] = fmaf(qv[g * D + 32 * b + 8 * k + i], u, a[g]);
        }
    } else {
      for (int j = 0; j < blk; ++j) {
        const float u = (float)kcode_generic(kp, cb, t, kbits, n, b * blk + j);
#pragma unroll
        for (int g = 0; g < G; ++g) a[g] = fmaf(qv[g * D + b * blk + j], u, a[g]);
      }
    }
    float d, m = 0.f;
    if (asym) {
      __half2 dm = *reinterpret_cast<const __half2*>(ks + t * sb + 4 * b);
      d = __low2float(dm); m = __high2float(dm);
    } else {
      d = __half2float(*reinterpret_cast<const __half*>(ks + t * sb + 2 * b));
    }
    const float off = block_off(kc, kbits, d, m);
#pragma unroll
    for (int g = 0; g < G; ++g) s[g] = fmaf(d, a[g], fmaf(off, qsum[g * 4 + b], s[g]));
  }
}

// Dequantized values of the lane's 4 channels (4l..4l+3) of V row t (row-major plane).
__device__ __forceinline__ void v_lane(int vc, int vbits, int n, int cb, int sb, const uint8_t* vp, const uint8_t* vs,
                                       int t, int lane, float v[4], bool bf16) {
  if (4 * lane >= n) { v[0] = v[1] = v[2] = v[3] = 0.f; return; }
  const uint8_t* row = vp + t * cb;
  if (vc == KVQ_F16) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + 8 * lane);
    const float2 a = raw2_to_float2(w.x, bf16), b = raw2_to_float2(w.y, bf16);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    return;
  }
  uint32_t u[4];
  switch (vbits) {
    case 8: { uint32_t w = *reinterpret_cast<const uint32_t*>(row + 4 * lane);
      for (int i = 0; i < 4; ++i) u[i] = (w >> (8 * i)) & 0xffu; } break;
    case 4: { uint32_t w = *reinterpret_cast<const uint16_t*>(row + 2 * lane);
      for (int i = 0; i < 4; ++i) u[i] = (w >> (4 * i)) & 15u; } break;
    case 2: { uint32_t w = row[lane];
      for (int i = 0; i < 4; ++i) u[i] = (w >> (2 * i)) & 3u; } break;
    case 1: { uint32_t w = (row[lane >> 1] >> (4 * (lane & 1))) & 15u;
      for (int i = 0; i < 4; ++i) u[i] = (w >> i) & 1u; } break;
    case 6: { uint32_t lo = *reinterpret_cast<const uint16_t*>(row + 2 * lane); uint32_t hi = row[n / 2 + lane];
      for (int i = 0; i < 4; ++i) u[i] = ((lo >> (4 * i)) & 15u) | (((hi >> (2 * i)) & 3u) << 4); } break;
    case 3: { uint32_t lo = row[lane]; uint32_t hi = (row[n / 4 + (lane >> 1)] >> (4 * (lane & 1))) & 15u;
      for (int i = 0; i < 4; ++i) u[i] = ((lo >> (2 * i)) & 3u) | (((hi >> i) & 1u) << 2); } break;
    case 5: { uint32_t lo = *reinterpret_cast<const uint16_t*>(row + 2 * lane);
      uint32_t hi = (row[n / 2 + (lane >> 1)] >> (4 * (lane & 1))) & 15u;
      for (int i = 0; i < 4; ++i) u[i] = ((lo >> (4 * i)) & 15u) | (((hi >> i) & 1u) << 4); } break;
    default: u[0] = u[1] = u[2] = u[3] = 0;
  }
  const int blk = n < 32 ? n : 32;
  const int b = (4 * lane) / blk;
  float d, m = 0.f;
  if (codec_is_asym(vc)) {
    __half2 dm = *reinterpret_cast<const __half2*>(vs + t * sb + 4 * b);
    d = __low2float(dm); m = __high2float(dm);
  } else {
    d = __half2float(*reinterpret_cast<const __half*>(vs + t * sb + 2 * b));
  }
  const float off = block_off(vc, vbits, d, m);
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = fmaf((float)u[i], d, off);
}

// Shared memory of one CTA.  The stage ring is only read inside the tile loop;
// afterwards the same bytes hold the warps' merge area and the final
// accumulators ("post" region).
__host__ __device__ inline size_t post_bytes(int G) {
  return (size_t)NCW * G * (D + 4) * 4 + (size_t)2 * G * D * 4 + (size_t)2 * G * 4 + 16;
}
size_t decode_smem_bytes(int stage_bytes, int n_stages, int G, bool wtab_smem) {
  size_t ring = (size_t)stage_bytes * n_stages;
  // after the loop the ring's bytes hold the post region and at least one head's
  // staged partials (MAX_SPLITS of them) for the last CTA's merge
  const size_t post_and_stage = ((post_bytes(G) + 127) & ~(size_t)127) + (size_t)MAX_SPLITS * PARTIAL_FLOATS * 4;
  size_t a = ring > post_and_stage ? ring : post_and_stage;
  a = (a + 127) & ~(size_t)127;
  a += (size_t)G * D * 4;            // qv
  a += (size_t)G * 4 * 4;            // qsum
  a += (size_t)G * 4 * 4;            // qsi
  a += (size_t)8 * 4;                // sq
  a += (size_t)2 * G * 64 * 4;       // pair tables
  a = (a + 15) & ~(size_t)15;
  if (wtab_smem) a += (size_t)NCW * wtab_bytes(G);   // per-warp weight tables
  a += (size_t)(2 * 8 + 2) * 8;      // mbarriers: ring full / empty, merge staging
  return a;
}

// Apply the value-basis inverse transform and write out[g][:] =
// (T_v(aq) + at) / L for the CTA's G heads.  aq/at: smem [G][D].
template <int G>
__device__ void finalize(const DecodeParams& p, const HeadInfo& h, int vbasis, int head, float* aq, float* at,
                         const float* fl, float* out_base) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= 4) return;
  for (int g = warp; g < G; g += 4) {
    const float L = fl[g];
    const float invL = 1.0f / L;
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = aq[g * D + 4 * lane + i];
    if (vbasis == BASIS_ROT) {
      fwht_row(x);
      if (p.s_v) {
        const float* sv = p.s_v + (size_t)head * D;
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] *= sv[4 * lane + i];
      }
    } else if (vbasis == BASIS_PROJ) {
      const float* M = p.M + h.m_off;
      float y[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < h.r; ++i) {
        const float a = aq[g * D + i];
        float4 mrow = *reinterpret_cast<const float4*>(M + (size_t)i * D + 4 * lane);
        y[0] = fmaf(mrow.x, a, y[0]); y[1] = fmaf(mrow.y, a, y[1]);
        y[2] = fmaf(mrow.z, a, y[2]); y[3] = fmaf(mrow.w, a, y[3]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = y[i];
    }
    float4 o;
    o.x = (x[0] + at[g * D + 4 * lane + 0]) * invL;
    o.y = (x[1] + at[g * D + 4 * lane + 1]) * invL;
    o.z = (x[2] + at[g * D + 4 * lane + 2]) * invL;
    o.w = (x[3] + at[g * D + 4 * lane + 3]) * invL;
    *reinterpret_cast<float4*>(out_base + (size_t)g * D + 4 * lane) = o;
  }
}

// VA: some kv head of the layer stores V with a _1 codec (scale and minimum), whose
// offsets need per-block accumulators; layers without one compile those away.
template <int G, bool VA>
__global__ void __launch_bounds__(DECODE_THREADS, DECODE_MIN_CTAS(G)) decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  // launched as a programmatic dependent: the grid is set up while the previous
  // kernel drains, and waits for it before reading or writing any global data
  griddep_launch_dependents();
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DecodeItem it = decode_item(p, blockIdx.x);
  if (it.kind == 3) return;                        // a head whose pages divide evenly: no partial split
  const int si = it.si, head = it.head, split = it.split;
  const int seq = p.seq[si], len = p.len[si];
  const int T = p.T;
  const SplitCounts sc = split_counts(len, T, p.pps[head], p.pps_t, p.lim[si]);
  const int nq = sc.nq, nt = sc.nt, NQP = sc.nqp, NTP = sc.ntp, qsplits = sc.qsplits;
  const int S = sc.qsplits + sc.tsplits;
  float* out_base = p.out + ((size_t)si * p.Hq + (size_t)head * G) * D;
  if (it.kind == 2) {                              // nothing to attend to: zeros
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) out_base[i] = 0.f;
    return;
  }
  const bool is_tail = it.kind == 1;
  const int pps = is_tail ? p.pps_t : p.pps[head];
  const int pg0 = (is_tail ? split - qsplits : split) * pps;
  const int pg1 = min(pg0 + pps, is_tail ? NTP : NQP);
  const int n_tiles = pg1 - pg0;
  const int seg_tokens = is_tail ? nt : nq;
  const HeadInfo h = p.heads[head];
  const int kc = is_tail ? (int)KVQ_F16 : (int)h.kcodec;
  const int vc = is_tail ? (int)KVQ_F16 : (int)h.vcodec;
  const int kbits = is_tail ? 16 : h.kbits, vbits = is_tail ? 16 : h.vbits;
  const int kbasis = basis_of(kc, p.rot), vbasis = basis_of(vc, p.rot);
  const int nK = kc == KVQ_RANK ? h.r : D, nV = vc == KVQ_RANK ? h.r : D;
  const int cbK = is_tail ? 2 * D : h.cbK, sbK = is_tail ? 0 : h.sbK;
  const int cbV = is_tail ? 2 * D : h.cbV, sbV = is_tail ? 0 : h.sbV;
  const uint32_t tile_bytes = is_tail ? (uint32_t)TAIL_PAGE_BYTES : h.bytes;
  const int rows = is_tail ? TAIL_TOK : PAGE;              // token rows per tile
  const int NS = p.n_stages;

  // shared memory carve-up
  const size_t ring = (size_t)p.stage_bytes * NS;
  const size_t post_and_stage = ((post_bytes(G) + 127) & ~(size_t)127) + (size_t)MAX_SPLITS * PARTIAL_FLOATS * 4;
  size_t off = ((ring > post_and_stage ? ring : post_and_stage) + 127) & ~(size_t)127;
  uint8_t* stages = smem;
  // post-loop region (aliases the ring)
  float* mg = reinterpret_cast<float*>(smem);                      // [4 warps][G][D+4]
  float* aq = mg + (size_t)NCW * G * (D + 4);                      // [G][D] quantized-basis accumulator
  float* at = aq + (size_t)G * D;                                  // [G][D] tail accumulator
  float* fm = at + (size_t)G * D;
  float* fl = fm + G;
  int* flag = reinterpret_cast<int*>(fl + G);
  float* qv = reinterpret_cast<float*>(smem + off); off += (size_t)G * D * 4;
  float* qsum = reinterpret_cast<float*>(smem + off); off += (size_t)G * 4 * 4;
  int* qsi = reinterpret_cast<int*>(smem + off); off += (size_t)G * 4 * 4;
  float* sq = reinterpret_cast<float*>(smem + off); off += (size_t)8 * 4;
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + off); off += (size_t)2 * G * 64 * 4;
  off = (off + 15) & ~(size_t)15;
  uint64_t* pw2 = reinterpret_cast<uint64_t*>(smem + off);         // per-warp weight tables (p.wtab_smem)
  if (p.wtab_smem) off += (size_t)NCW * wtab_bytes(G);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + off);
  uint64_t* empty = full + 8;
  uint64_t* mmerge = full + 16;                                    // the merge's two staging buffers

  // The producer sets up the ring and starts the first NS page loads right away,
  // so they overlap the query preparation below.  Its 32 lanes read the
  // block-table entries of 32 tiles at once (lane j: tile i0 + j), so the first
  // loads do not wait on one another's table reads; lane 0 issues the copies.
  const uint8_t* tail_base =
      is_tail ? p.tail + (((size_t)seq * p.L + p.layer) * p.Hkv + head) * (size_t)T * (D * 2 * 2) : nullptr;
  auto load_pids = [&](int i0) -> int {
    int pid = 0;
    if (!is_tail && i0 + lane < n_tiles) {
      pid = p.block_table[(size_t)seq * p.max_pages_per_seq + pg0 + i0 + lane];
      if (pid < 0) { atomicOr(p.err, ERR_NO_PAGE); pid = 0; }
    }
    return pid;
  };
  auto issue_tile = [&](int i, int st, int pid) {  // lane 0 of the producer warp; st = i % NS
    const uint8_t* src = is_tail ? tail_base + (size_t)(pg0 + i) * TAIL_PAGE_BYTES
                                 : p.pool + (size_t)pid * p.page_bytes + h.off;
    // test-only fault injection: the last tile is never loaded, so its consumer's
    // bounded wait runs out (no later tile reuses the stage, no copy is left in flight)
    if (p.drop_last_tile && i == n_tiles - 1) return;
    mbar_arrive_expect_tx(&full[st], tile_bytes);
    bulk_g2s(stages + (size_t)st * p.stage_bytes, src, tile_bytes, &full[st]);
  };
  int pids = 0;                                     // producer: entries of tiles 32k .. 32k+31
  if (warp == NCW) {
    pids = load_pids(0);
    if (lane == 0) {
      for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
      mbar_init(&mmerge[0], 1);
      mbar_init(&mmerge[1], 1);
      fence_mbar_init();
    }
    for (int i = 0; i < NS && i < n_tiles; ++i) {  // NS <= 8: all in the first batch
      const int pid = __shfl_sync(0xffffffffu, pids, i);
      if (lane == 0) issue_tile(i, i, pid);
    }
  }

  const bool kfast = kc != KVQ_F16;                 // integer key scores (block and rank codecs)
  // ---- query preparation (consumer warps): q' in the K basis, scaled to log2 units
  if (warp < NCW) {
    for (int g = warp; g < G; g += NCW) {
      const __half* qsrc = p.q + ((size_t)si * p.Hq + (size_t)head * G + g) * D;
      const uint2 raw = *reinterpret_cast<const uint2*>(qsrc + 4 * lane);
      const float2 a = raw2_to_float2(raw.x, p.bf16), b = raw2_to_float2(raw.y, p.bf16);
      float x[4] = {a.x, a.y, b.x, b.y};
      if (kbasis == BASIS_ROT) {
        if (p.s_k) {
          const float* sk = p.s_k + (size_t)head * D;
#pragma unroll
          for (int i = 0; i < 4; ++i) x[i] *= sk[4 * lane + i];
        }
        fwht_row(x);
      } else if (kbasis == BASIS_PROJ) {
        // M_h q, computed once per (sequence, kv head) by project_query_kernel
        const float4 z = *reinterpret_cast<const float4*>(p.qproj + ((size_t)si * p.Hq + (size_t)head * G + g) * D +
                                                          4 * lane);
        x[0] = z.x; x[1] = z.y; x[2] = z.z; x[3] = z.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[i] = (4 * lane + i < nK) ? x[i] * p.qscale : 0.f;
        qv[g * D + 4 * lane + i] = x[i];
      }
      // per-block sums of q'
      const int blk = nK < 32 ? nK : 32;
      float ssum = (x[0] + x[1]) + (x[2] + x[3]);
      for (int m = 1; m < blk / 4; m <<= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, m);
      if (4 * lane < nK && ((4 * lane) % blk) == 0) qsum[g * 4 + (4 * lane) / blk] = ssum;
      if (kfast) {
        // integer query for the block codecs: int16 with one scale per head and
        // exact integer block sums
        const float amax = warp_max(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))));
        const float scale = amax > 0.f ? amax * (1.0f / 32767.0f) : 1.0f;
        const float inv = 1.0f / scale;
        // each value goes straight to its slots in the pair tables of the K codec's
        // code planes (tab_slot inverts the order the planes' masks produce)
        int tt0, tt1;
        codec_tables(kbits, &tt0, &tt1);
        uint16_t* tab16 = reinterpret_cast<uint16_t*>(tab);
        int bs = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          int v = __float2int_rn(x[i] * inv);
          v = max(-32767, min(32767, v));
          bs += v;
#pragma unroll
          for (int plane = 0; plane < 2; ++plane) {
            const int type = plane ? tt1 : tt0;
            if (type < 0) continue;
            int w, half;
            tab_slot(type, 4 * lane + i, w, half);
            tab16[((plane * G + g) * 64 + w) * 2 + half] = (uint16_t)(int16_t)v;
          }
        }
        bs += __shfl_xor_sync(0xffffffffu, bs, 1);
        bs += __shfl_xor_sync(0xffffffffu, bs, 2);
        bs += __shfl_xor_sync(0xffffffffu, bs, 4);
        if ((lane & 7) == 0) qsi[g * 4 + (lane >> 3)] = bs;
        if (lane == 0) sq[g] = scale;
      }
    }
  }
  __syncthreads();

  float m[G], l[G], acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY; l[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[g][i] = 0.f;
  }
  if (warp == NCW) {
    // ---- producer: refill each stage once its consumer warp has released it
    // stage and empty-barrier phase of tile i, kept incrementally (no division)
    int st = 0, ph = 0;
    for (int i = NS; i < n_tiles; ++i) {
      if ((i & 31) == 0) pids = load_pids(i);
      const int pid = __shfl_sync(0xffffffffu, pids, i & 31);
      if (lane == 0) {
        if (!mbar_wait(&empty[st], ph, p.wait_ns, 1024)) atomicOr(p.err, ERR_TIMEOUT);
        issue_tile(i, st, pid);
      }
      if (++st == NS) { st = 0; ph ^= 1; }
    }
  } else {
    // ---- consumers
    // Per warp: online-softmax state (m, l per head) and the fp32 value accumulators
    // of the lane's 4 channels 4*lane .. 4*lane+3, as two packed pairs per head.  On
    // the integer value path the block offsets of the lane's own tokens (weight x
    // (-2^(b-1) d) or weight x m) go into off[g][block] and are summed over the warp
    // after the last tile.
    uint64_t O2[G][2];
    float off[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      O2[g][0] = 0ull; O2[g][1] = 0ull;
#pragma unroll
      for (int b = 0; b < 4; ++b) off[g][b] = 0.f;
    }
    const bool vblock = vc != KVQ_F16 && vc != KVQ_RANK;
    // value path: centred integer (8/4/2-bit planes), two unsigned planes (LO*10 + HI),
    // or 0 = fp32 (F16)
    int vclass = 0;
    if (vblock) vclass = (vbits == 8 || vbits == 4 || vbits == 2) ? vbits : (vbits == 6) ? 42 : (vbits == 5) ? 41 : 21;
    else if (vc == KVQ_RANK) vclass = (vbits == 4) ? 40 : (vbits == 3) ? 21 : (vbits == 2) ? 20 : 10;
    const bool vasym = VA && codec_is_asym(vc);
    const bool kasym = codec_is_asym(kc);
    const float vhalf = vblock ? (float)(1 << (vbits - 1)) : 0.f;
    // the codes' centre on the plane path, the byte offset of the high plane, the
    // blocks per row and the lanes per token pair
    const float vcen = (vc == KVQ_RANK) ? 0.5f * (float)((1 << vbits) - 1) : vhalf;
    const int voffB = (vc == KVQ_RANK) ? nV / 4 : (vbits == 3 ? 32 : 64);
    const int blkV = nV < 32 ? nV : 32;
    const int nbV = nV / blkV;
    const int vcl = (nV == 16 || nV == 32 || nV == 64) ? nV / 4 : 32;
    const int blane = ((4 * lane) / (nV < 32 ? nV : 32)) & 3;
    const int kclass = !kfast ? 0 : (kc == KVQ_RANK) ? 10 + kbits : (kbits == 8 ? 8 : (kbits >= 4 ? 4 : 2));
    // This warp's weight table: (w, w) pairs per token on the fp32 path, int16 pairs
    // per token pair and block on the integer path (same bytes).
    constexpr int PWG = G + 1;                          // fp32 path row: G pairs + pad
    // The weight table goes into the K region of the warp's own stage once the
    // scores are taken (the stage is this warp's until it releases it), or into
    // the warp's slot of the separate table area when the K rows are too small.
    const bool wt_stage = (uint32_t)rows * (uint32_t)(cbK + sbK) >= wtab_bytes(G);
    // 0xF0F0F0F0 and 0x80808080 as run-time values (n_seqs >= 0, so rz == 0)
    const uint32_t rz = (uint32_t)p.n_seqs >> 31;
    const uint32_t kM = 0xF0F0F0F0u ^ rz, kC = 0x80808080u ^ rz;
    // stage and full-barrier phase of tile i, kept incrementally: tile i sits in stage
    // i % NS, phase (i / NS) & 1; warp w takes tiles w, w + NCW, ... and NCW <= NS
    int st = warp, ph = 0;
    for (int i = warp; i < n_tiles; i += NCW, st += NCW, ph ^= (st >= NS) ? 1 : 0, st -= (st >= NS) ? NS : 0) {
      if (!mbar_wait(&full[st], ph, p.wait_ns)) atomicOr(p.err, ERR_TIMEOUT);
      const uint8_t* sp = stages + (size_t)st * p.stage_bytes;
      const uint8_t* kp = sp;
      const uint8_t* ks = kp + rows * cbK;
      const uint8_t* vp = ks + rows * sbK;
      const uint8_t* vs = vp + rows * cbV;
      uint64_t* pw = wt_stage ? reinterpret_cast<uint64_t*>(stages + (size_t)st * p.stage_bytes)
                              : pw2 + (size_t)warp * (wtab_bytes(G) / 8);
      uint32_t* wq = reinterpret_cast<uint32_t*>(pw);
      const int tok0 = (pg0 + i) * rows;
      const int nvalid = min(rows, seg_tokens - tok0);
      // the lane's first token (the second one, lane + 32, lies past a 16-row tail
      // tile): inside the segment, and for a tail slot also visible to the query
      const bool vis0 = lane < nvalid && (!is_tail || tail_visible(sc, T, tok0 + lane));
      if (is_tail && !__any_sync(0xffffffffu, vis0)) {   // no visible token in this tile
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        continue;
      }
      float s0[G], s1[G];
      switch (kclass) {
#define KVQ_SCORE(KCL, ASYM) score2_block_codec<G, KCL, ASYM>(kc, kp, ks, sbK, lane, tab, tab + G * 64, qsi, s0, s1)
        case 8: if (kasym) KVQ_SCORE(8, true); else KVQ_SCORE(8, false); break;
        case 4: if (kasym) KVQ_SCORE(4, true); else KVQ_SCORE(4, false); break;
        case 2: if (kasym) KVQ_SCORE(2, true); else KVQ_SCORE(2, false); break;
#undef KVQ_SCORE
        case 11: score2_rank<G, 1>(nK, kp, ks, cbK, sbK, lane, tab, tab + G * 64, qsi, s0, s1); break;
        case 12: score2_rank<G, 2>(nK, kp, ks, cbK, sbK, lane, tab, tab + G * 64, qsi, s0, s1); break;
        case 13: score2_rank<G, 3>(nK, kp, ks, cbK, sbK, lane, tab, tab + G * 64, qsi, s0, s1); break;
        case 14: score2_rank<G, 4>(nK, kp, ks, cbK, sbK, lane, tab, tab + G * 64, qsi, s0, s1); break;
        default:
          score_token<G>(kc, kbits, nK, cbK, sbK, kp, ks, lane, qv, qsum, s0, rows, p.bf16);
          score_token<G>(kc, kbits, nK, cbK, sbK, kp, ks, lane + 32, qv, qsum, s1, rows, p.bf16);
      }
      if (kclass) {
#pragma unroll
        for (int g = 0; g < G; ++g) { s0[g] *= sq[g]; s1[g] *= sq[g]; }
      }
      float p0[G], p1[G], pm[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (!vis0) s0[g] = -INFINITY;
        if (lane + 32 >= nvalid) s1[g] = -INFINITY;
        const float tmax = warp_max(fmaxf(s0[g], s1[g]));
        const float mnew = fmaxf(m[g], tmax);
        const float alpha = ex2_approx(m[g] - mnew);
        p0[g] = ex2_approx(s0[g] - mnew);
        p1[g] = ex2_approx(s1[g] - mnew);
        pm[g] = ex2_approx(tmax - mnew);
        l[g] = l[g] * alpha + (p0[g] + p1[g]);
        const uint64_t a2 = pack2(alpha, alpha);
        O2[g][0] = mul2(O2[g][0], a2);
        O2[g][1] = mul2(O2[g][1], a2);
        if (vasym) {
#pragma unroll
          for (int b = 0; b < 4; ++b) off[g][b] *= alpha;
        }
        m[g] = mnew;
      }
      __syncwarp();                         // every lane's key reads are done: the K region may be reused
      switch (vclass) {
        case 8:
          if (vasym) value_tile_int<G, 8, true>(vhalf, vp, vs, sbV, nvalid, lane, blane, wq, kM, kC, p0, p1, pm, O2, off);
          else value_tile_int<G, 8, false>(vhalf, vp, vs, sbV, nvalid, lane, blane, wq, kM, kC, p0, p1, pm, O2, off);
          break;
        case 4:
          if (vasym) value_tile_int<G, 4, true>(vhalf, vp, vs, sbV, nvalid, lane, blane, wq, kM, kC, p0, p1, pm, O2, off);
          else value_tile_int<G, 4, false>(vhalf, vp, vs, sbV, nvalid, lane, blane, wq, kM, kC, p0, p1, pm, O2, off);
          break;
        case 2:
          if (vasym) value_tile_int<G, 2, true>(vhalf, vp, vs, sbV, nvalid, lane, blane, wq, kM, kC, p0, p1, pm, O2, off);
          else value_tile_int<G, 2, false>(vhalf, vp, vs, sbV, nvalid, lane, blane, wq, kM, kC, p0, p1, pm, O2, off);
          break;
#define KVQ_PLANES(LO, HI, ASYM)                                                                                      \
  value_tile_planes<G, LO, HI, ASYM>(nbV, blkV, vcl, vcen, voffB, vp, vs, cbV, sbV, nvalid, lane, wq, p0, p1, pm, O2, \
                                     off)
        case 42: if (vasym) KVQ_PLANES(4, 2, true); else KVQ_PLANES(4, 2, false); break;
        case 41: if (vasym) KVQ_PLANES(4, 1, true); else KVQ_PLANES(4, 1, false); break;
        case 21: if (vasym) KVQ_PLANES(2, 1, true); else KVQ_PLANES(2, 1, false); break;
        case 40: KVQ_PLANES(4, 0, false); break;
        case 20: KVQ_PLANES(2, 0, false); break;
        case 10: KVQ_PLANES(1, 0, false); break;
#undef KVQ_PLANES
        default:
          // fp32 path: dequantized values times the softmax numerator, packed FMAs
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float pg = half ? p1[g] : p0[g];
              pw[(size_t)lane * PWG + g] = pack2(pg, pg);
            }
            __syncwarp();
            const int ntok = min(32, nvalid - 32 * half);
            for (int tt = 0; tt < ntok; ++tt) {
              float v[4];
              v_lane(vc, vbits, nV, cbV, sbV, vp, vs, 32 * half + tt, lane, v, p.bf16);
              const uint64_t u01 = pack2(v[0], v[1]), u23 = pack2(v[2], v[3]);
              const uint64_t* wrow = pw + (size_t)tt * PWG;
#pragma unroll
              for (int g = 0; g < G; ++g) {
                const uint64_t w2 = wrow[g];
                O2[g][0] = fma2(w2, u01, O2[g][0]);
                O2[g][1] = fma2(w2, u23, O2[g][1]);
              }
            }
            __syncwarp();
          }
      }
      // the weight-table stores (generic proxy) must land before the stage's next
      // bulk copy (async proxy) overwrites it
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      l[g] = warp_sum(l[g]);
      float ob = 0.f;                     // the lane's block's offset sum, no dynamic register index
      if (vasym) {                        // only the _1 codecs accumulate offsets
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float sb = warp_sum(off[g][b]);
          ob = (b == blane) ? sb : ob;
        }
      }
      float a[4];
      unpack2(O2[g][0], a[0], a[1]);
      unpack2(O2[g][1], a[2], a[3]);
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[g][c] = a[c] + ob;
    }
  }
  __syncthreads();   // every stage consumed: the ring is reused as the merge area below
  if (warp < NCW) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* dst = mg + ((size_t)warp * G + g) * (D + 4);
      if (lane == 0) { dst[0] = m[g]; dst[1] = l[g]; }
#pragma unroll
      for (int c = 0; c < 4; ++c) dst[4 + 4 * lane + c] = acc[g][c];
    }
  }
  __syncthreads();

  // ---- merge the consumer warps' states in warp order: one pass over (head,
  // channel); a single split keeps the result for finalize, any other publishes it
  // straight to its partial.  Partials are laid out [sequence, kv head][G]
  // [MAX_SPLITS][PARTIAL_FLOATS], so one head's splits are one contiguous block for
  // the last CTA's merge below.
  float* pbase = p.ws + ((size_t)si * p.Hkv + head) * G * MAX_SPLITS * PARTIAL_FLOATS;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, c = idx % D;
    float mw[NCW];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
      mw[w] = mg[((size_t)w * G + g) * (D + 4)];
      M = fmaxf(M, mw[w]);
    }
    float A = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
      if (mw[w] == -INFINITY) continue;
      const float f = exp2f(mw[w] - M);
      L += f * mg[((size_t)w * G + g) * (D + 4) + 1];
      A += f * mg[((size_t)w * G + g) * (D + 4) + 4 + c];
    }
    if (S == 1) {
      aq[idx] = is_tail ? 0.f : A;
      at[idx] = is_tail ? A : 0.f;
      if (c == 0) { fm[g] = M; fl[g] = L; }
    } else {
      float* dst = pbase + ((size_t)g * MAX_SPLITS + split) * PARTIAL_FLOATS;
      dst[4 + c] = A;
      if (c == 0) { dst[0] = M; dst[1] = L; }
    }
  }
  __syncthreads();
  if (S == 1) {
    finalize<G>(p, h, vbasis, head, aq, at, fl, out_base);
    return;
  }
  if (threadIdx.x == 0) {
    // release: this CTA's partial (ordered before by the barrier) becomes visible
    // to whichever CTA draws the last ticket; acquire: that CTA sees all others'.
    const int old = atom_add_acq_rel_gpu(&p.tickets[si * p.Hkv + head], 1);
    flag[0] = (old == S - 1);
  }
  __syncthreads();
  if (!flag[0]) return;
  // ---- last CTA: merge every split in a fixed order (deterministic).  Each head's
  // S partials are pulled into shared memory with one bulk copy (double-buffered
  // over the heads when room allows); meanwhile every head's split maxima, factors
  // and sums are taken straight from L2, and then one thread per channel sums the
  // rescaled partials of a head as it lands.
  const uint32_t per_g = (uint32_t)S * PARTIAL_FLOATS * 4;
  const size_t stage_off = (post_bytes(G) + 127) & ~(size_t)127;
  const size_t stage_room = (size_t)(reinterpret_cast<uint8_t*>(full) - smem) - stage_off;   // all dead after the loop
  const int nbuf = min(min(G, 2), (int)(stage_room / per_g));      // >= 1: see decode_smem_bytes; 2 barriers
  float* fsc = mg;                                                  // [G][MAX_SPLITS] split factors
  if (threadIdx.x == 0) {
    fence_proxy_async_global();          // the acquired partials, read through the bulk-copy path
    fence_proxy_async_shared();          // the staging area was last used by ordinary loads and stores
    for (int b = 0; b < nbuf; ++b) {
      mbar_arrive_expect_tx(&mmerge[b], per_g);
      bulk_g2s(smem + stage_off + (size_t)b * per_g, pbase + (size_t)b * MAX_SPLITS * PARTIAL_FLOATS, per_g,
               &mmerge[b]);
    }
  }
  // every head's split maxima, factors and sums, read from L2 while the copies land
  // (the partials were published with release and acquired by the ticket above)
  for (int g = warp; g < G; g += blockDim.x / 32) {
    float ms[2], ls[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int s2 = lane + 32 * k;
      const float* src = pbase + ((size_t)g * MAX_SPLITS + s2) * PARTIAL_FLOATS;
      ms[k] = s2 < S ? __ldcg(src) : -INFINITY;
      ls[k] = s2 < S ? __ldcg(src + 1) : 0.f;
    }
    const float M = warp_max(fmaxf(ms[0], ms[1]));
    float part = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int s2 = lane + 32 * k;
      const float f = (ms[k] == -INFINITY) ? 0.f : exp2f(ms[k] - M);
      if (s2 < S) fsc[g * MAX_SPLITS + s2] = f;
      part += f * ls[k];
    }
    const float L = warp_sum(part);
    if (lane == 0) { fm[g] = M; fl[g] = L; }
  }
  __syncthreads();
  for (int g = 0; g < G; ++g) {
    const int b = g % nbuf;
    if (!mbar_wait(&mmerge[b], (g / nbuf) & 1, p.wait_ns)) atomicOr(p.err, ERR_TIMEOUT);
    const float* pg = reinterpret_cast<const float*>(smem + stage_off + (size_t)b * per_g);
    const float* fg = fsc + g * MAX_SPLITS;
    // two chains per sum (even and odd splits), added in that order: a fixed order
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      float A0 = 0.f, A1 = 0.f, B0 = 0.f, B1 = 0.f;
      int s2 = 0;
      for (; s2 + 1 < qsplits; s2 += 2) {
        A0 = fmaf(pg[(size_t)s2 * PARTIAL_FLOATS + 4 + c], fg[s2], A0);
        A1 = fmaf(pg[(size_t)(s2 + 1) * PARTIAL_FLOATS + 4 + c], fg[s2 + 1], A1);
      }
      if (s2 < qsplits) { A0 = fmaf(pg[(size_t)s2 * PARTIAL_FLOATS + 4 + c], fg[s2], A0); ++s2; }
      for (; s2 + 1 < S; s2 += 2) {
        B0 = fmaf(pg[(size_t)s2 * PARTIAL_FLOATS + 4 + c], fg[s2], B0);
        B1 = fmaf(pg[(size_t)(s2 + 1) * PARTIAL_FLOATS + 4 + c], fg[s2 + 1], B1);
      }
      if (s2 < S) B0 = fmaf(pg[(size_t)s2 * PARTIAL_FLOATS + 4 + c], fg[s2], B0);
      aq[g * D + c] = A0 + A1;
      at[g * D + c] = B0 + B1;
    }
    __syncthreads();
    if (threadIdx.x == 0 && g + nbuf < G) {
      fence_proxy_async_shared();
      mbar_arrive_expect_tx(&mmerge[b], per_g);
      bulk_g2s(smem + stage_off + (size_t)b * per_g, pbase + (size_t)(g + nbuf) * MAX_SPLITS * PARTIAL_FLOATS, per_g,
               &mmerge[b]);
    }
  }
  if (threadIdx.x == 0) p.tickets[si * p.Hkv + head] = 0;
  __syncthreads();
  const int vb_final = basis_of(h.vcodec, p.rot);
  finalize<G>(p, h, vb_final, head, aq, at, fl, out_base);
}

// Projected queries of the rank variant: z = M_h q for the G query heads of every
// (sequence, kv head), one thread per row of M_h (r <= 128), written to
// p.qproj[seq][q head][0..127] (zeros past r).  Runs before decode_kernel.
__global__ void __launch_bounds__(128) project_query_kernel(const __grid_constant__ DecodeParams p) {
  __shared__ __align__(16) float qs[MAX_G][D];
  const int head = blockIdx.x, si = blockIdx.y, i = threadIdx.x;
  const HeadInfo h = p.heads[head];
  for (int idx = threadIdx.x; idx < p.G * D; idx += blockDim.x) {
    const int g = idx / D, c = idx % D;
    qs[g][c] = __half2float(p.q[((size_t)si * p.Hq + (size_t)head * p.G + g) * D + c]);
  }
  __syncthreads();
  float z[MAX_G];
#pragma unroll
  for (int g = 0; g < MAX_G; ++g) z[g] = 0.f;
  if (h.kcodec == KVQ_RANK && i < h.r) {
    const float4* row = reinterpret_cast<const float4*>(p.M + h.m_off + (size_t)i * D);
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; ++c4) {
      const float4 m = __ldg(row + c4);
#pragma unroll
      for (int g = 0; g < MAX_G; ++g) {
        if (g < p.G) {
          z[g] = fmaf(m.x, qs[g][4 * c4 + 0], z[g]);
          z[g] = fmaf(m.y, qs[g][4 * c4 + 1], z[g]);
          z[g] = fmaf(m.z, qs[g][4 * c4 + 2], z[g]);
          z[g] = fmaf(m.w, qs[g][4 * c4 + 3], z[g]);
        }
      }
    }
  }
  for (int g = 0; g < p.G; ++g) p.qproj[((size_t)si * p.Hq + (size_t)head * p.G + g) * D + i] = z[g];
}

cudaError_t launch_project_query(const DecodeParams& p, cudaStream_t s) {
  project_query_kernel<<<dim3(p.Hkv, p.n_seqs), 128, 0, s>>>(p);
  note_launches(1);
  return cudaGetLastError();
}

int decode_max_smem() { return 227 * 1024; }

template <int G, bool VA>
static cudaError_t launch_gv(const DecodeParams& p, int grid_x, cudaStream_t s) {
  const size_t smem = decode_smem_bytes(p.stage_bytes, p.n_stages, G, p.wtab_smem != 0);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<G, VA>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_x, 1, 1);
  cfg.blockDim = dim3(DECODE_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<G, VA>, p);
  note_launches(1);
  return e;
}

template <int G>
static cudaError_t launch_g(const DecodeParams& p, int grid_x, cudaStream_t s) {
  bool va = false;
  for (int h = 0; h < p.Hkv; ++h) va = va || codec_is_asym(p.heads[h].vcodec);
  return va ? launch_gv<G, true>(p, grid_x, s) : launch_gv<G, false>(p, grid_x, s);
}

// Resident CTAs per SM of the kernel for G heads with `smem` dynamic bytes (registers,
// shared memory and the thread limit all counted), 0 on error.
template <int G>
static int blocks_per_sm_g(size_t smem) {
  // both variants have the same launch bounds (register cap) and shared memory
  if (cudaFuncSetAttribute(decode_kernel<G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<G, true>, DECODE_THREADS, smem) != cudaSuccess)
    return 0;
  return n;
}

static int blocks_per_sm_uncached(int G, size_t smem) {
  switch (G) {
    case 1: return blocks_per_sm_g<1>(smem);
    case 2: return blocks_per_sm_g<2>(smem);
    case 3: return blocks_per_sm_g<3>(smem);
    case 4: return blocks_per_sm_g<4>(smem);
    case 5: return blocks_per_sm_g<5>(smem);
    case 6: return blocks_per_sm_g<6>(smem);
    case 7: return blocks_per_sm_g<7>(smem);
    case 8: return blocks_per_sm_g<8>(smem);
    default: return 0;
  }
}

int decode_blocks_per_sm(int G, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, size_t>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, G, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  const int n = blocks_per_sm_uncached(G, smem);
  if (n > 0) cache[key] = n;
  return n;
}

cudaError_t launch_decode(const DecodeParams& p, int grid_x, cudaStream_t s) {
  switch (p.G) {
    case 1: return launch_g<1>(p, grid_x, s);
    case 2: return launch_g<2>(p, grid_x, s);
    case 3: return launch_g<3>(p, grid_x, s);
    case 4: return launch_g<4>(p, grid_x, s);
    case 5: return launch_g<5>(p, grid_x, s);
    case 6: return launch_g<6>(p, grid_x, s);
    case 7: return launch_g<7>(p, grid_x, s);
    case 8: return launch_g<8>(p, grid_x, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
