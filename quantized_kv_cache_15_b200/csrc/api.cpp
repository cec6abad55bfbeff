// Host side of the kvq C ABI: plan creation and validation, the paged cache
// layout, page allocation, split-K sizing and the launches.  Everything that
// touches data runs in the CUDA kernels of this directory; this file only moves
// host bookkeeping and enqueues work on the caller's stream.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include <cuda_fp16.h>

#include "kvq_internal.h"

using namespace kvq;

namespace {

thread_local std::string g_err;
std::atomic<unsigned long long> g_launches{0};

kvq_status fail(kvq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

kvq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool valid_codec(int c) { return c >= KVQ_F16 && c <= KVQ_Q5_1; }
bool valid_rank(int r) { return r == 16 || r == 32 || r == 64 || r == 96 || r == 128; }


}  // namespace

void kvq::note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

struct kvq_plan {
  int device = 0;
  int num_sms = 148;
  int L = 0, Hq = 0, Hkv = 0, G = 0, T = 0, max_seqs = 0;
  int64_t max_tokens = 0;
  int mpps = 0;            // max pages per sequence
  int64_t n_pages = 0;
  int rot = 0;
  bool bf16 = false;             // raw rows are bf16
  float scale = 0.f;
  std::vector<HeadInfo> heads;        // [L][Hkv]
  std::vector<uint64_t> layer_off;    // [L]
  std::vector<uint32_t> page_bytes;   // [L]
  std::vector<int> stage_bytes;       // [L] max region (and tail page) bytes
  uint64_t tail_off = 0, cache_bytes = 0;
  uint8_t* cache = nullptr;
  float* d_inv = nullptr;   // [L][Hkv][2][128] inverse RMS (append)
  float* d_sk = nullptr;    // [L][Hkv][128] 1/inv_rms of K (decode, dequantize)
  float* d_sv = nullptr;    // [L][Hkv][128] 1/inv_rms of V
  float* d_M = nullptr;     // fused projections M_h, fp32 [r][128] per head
  double* d_MT = nullptr;   // their transposes, widened to double [128][r] per head (append projection)
  int* d_bt = nullptr;      // block table [max_seqs][mpps]
  int* d_err = nullptr;
  std::vector<int64_t> len;           // [max_seqs][L]
  std::vector<int> bt;                // host mirror of the block table
  std::vector<int> npages;            // pages held per sequence
  std::vector<int> free_pages;        // stack of free page ids
  // test-only settings (kvq_debug_set_decode_split, kvq_debug_fault_injection)
  int debug_pps = 0;                          // fixed pages per split, 0 = chosen per call
  unsigned long long wait_ns = 2000000000ull; // give-up time of the kernels' bounded waits
  int drop_last_tile = 0;                     // decode producers skip their last tile
  int prefill_path = 0;                       // 0: tensor cores where the layer allows, 1: decode kernel

  ~kvq_plan() {
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(device);
    cudaFree(d_inv); cudaFree(d_sk); cudaFree(d_sv); cudaFree(d_M); cudaFree(d_MT); cudaFree(d_bt); cudaFree(d_err);
    cudaSetDevice(prev);
  }

  const HeadInfo& head(int l, int h) const { return heads[(size_t)l * Hkv + h]; }

  void reset_all() {
    std::fill(len.begin(), len.end(), 0);
    std::fill(bt.begin(), bt.end(), -1);
    std::fill(npages.begin(), npages.end(), 0);
    free_pages.clear();
    for (int64_t i = n_pages - 1; i >= 0; --i) free_pages.push_back((int)i);
  }

  DecodeParams base_params(int layer) const {
    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.pool = cache + layer_off[layer];
    p.page_bytes = page_bytes[layer];
    p.block_table = d_bt;
    p.max_pages_per_seq = mpps;
    p.tail = cache + tail_off;
    p.T = T; p.L = L; p.layer = layer; p.Hkv = Hkv; p.Hq = Hq; p.G = G;
    p.rot = rot;
    p.bf16 = bf16;
    p.s_k = (rot == KVQ_ROT_VARNORM_HADAMARD) ? d_sk + (size_t)layer * Hkv * D : nullptr;
    p.s_v = (rot == KVQ_ROT_VARNORM_HADAMARD) ? d_sv + (size_t)layer * Hkv * D : nullptr;
    p.M = d_M;
    p.qscale = scale * 1.4426950408889634f;
    p.err = d_err;
    p.wait_ns = wait_ns;
    p.drop_last_tile = drop_last_tile;
    for (int h = 0; h < Hkv; ++h) p.heads[h] = head(layer, h);
    return p;
  }
};

// Kernels are launched on the current device and read the plan's memory, so a call
// that enqueues work needs the plan's device current: on another device (through
// the legacy stream, say) they would reach that memory only by peer access, which
// this library never enables.  Checked before anything is enqueued.
static kvq_status require_plan_device(const kvq_plan* p) {
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != p->device) return fail(KVQ_ERR_STATE, "current device %d is not the plan's device %d", dev, p->device);
  return KVQ_OK;
}

extern "C" {

const char* kvq_last_error(void) { return g_err.c_str(); }

kvq_status kvq_launch_count(uint64_t* count) {
  if (!count) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  *count = (uint64_t)g_launches.load(std::memory_order_relaxed);
  return KVQ_OK;
}

kvq_status kvq_plan_create(const kvq_plan_desc* d, kvq_plan** out) {
  if (!d || !out) return fail(KVQ_ERR_INVALID_ARG, "null descriptor or output pointer");
  *out = nullptr;
  if (d->head_dim != D) return fail(KVQ_ERR_UNSUPPORTED, "head_dim must be 128 (got %d)", d->head_dim);
  if (d->n_layers < 1 || d->n_kv_heads < 1 || d->n_q_heads < 1)
    return fail(KVQ_ERR_INVALID_ARG, "n_layers, n_q_heads and n_kv_heads must be >= 1");
  if (d->n_kv_heads > MAX_HKV) return fail(KVQ_ERR_UNSUPPORTED, "n_kv_heads > %d", MAX_HKV);
  if (d->n_q_heads % d->n_kv_heads) return fail(KVQ_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  if (d->n_q_heads / d->n_kv_heads > MAX_G) return fail(KVQ_ERR_UNSUPPORTED, "GQA ratio above %d", MAX_G);
  if (d->max_seqs < 1 || d->max_tokens_per_seq < 1) return fail(KVQ_ERR_INVALID_ARG, "max_seqs and max_tokens_per_seq must be >= 1");
  if (d->max_tokens_per_seq > (int64_t)1 << 30) return fail(KVQ_ERR_UNSUPPORTED, "max_tokens_per_seq above 2^30");
  if (d->tail_tokens < 0 || d->tail_tokens % PAGE) return fail(KVQ_ERR_INVALID_ARG, "tail_tokens must be 0 or a multiple of 64");
  if (d->rot < KVQ_ROT_NONE || d->rot > KVQ_ROT_PROJECTION) return fail(KVQ_ERR_INVALID_ARG, "bad rot %d", d->rot);
  if (!d->k_codec || !d->v_codec) return fail(KVQ_ERR_INVALID_ARG, "k_codec and v_codec tables are required");
  if (d->rot == KVQ_ROT_VARNORM_HADAMARD && !d->inv_rms) return fail(KVQ_ERR_INVALID_ARG, "VARNORM_HADAMARD needs inv_rms");
  if (d->rot == KVQ_ROT_PROJECTION && (!d->rank || !d->k_bits || !d->v_bits || !d->proj_basis))
    return fail(KVQ_ERR_INVALID_ARG, "PROJECTION needs rank, k_bits, v_bits and proj_basis");
  if (d->kv_dtype != KVQ_KV_F16 && d->kv_dtype != KVQ_KV_BF16) return fail(KVQ_ERR_INVALID_ARG, "bad kv_dtype %d", d->kv_dtype);
  if (d->kv_dtype == KVQ_KV_BF16 && d->rot == KVQ_ROT_PROJECTION)
    return fail(KVQ_ERR_UNSUPPORTED, "bf16 rows are not supported with the projection path");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  kvq_plan* p = new kvq_plan();
  p->device = dev;
  cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, dev);
  p->L = d->n_layers; p->Hq = d->n_q_heads; p->Hkv = d->n_kv_heads; p->G = p->Hq / p->Hkv;
  p->T = d->tail_tokens; p->max_seqs = d->max_seqs; p->max_tokens = d->max_tokens_per_seq;
  p->mpps = (int)((p->max_tokens + PAGE - 1) / PAGE);
  p->n_pages = d->max_pages > 0 ? d->max_pages : (int64_t)p->max_seqs * p->mpps;
  p->rot = d->rot;
  p->bf16 = d->kv_dtype == KVQ_KV_BF16;
  p->scale = d->softmax_scale > 0.f ? d->softmax_scale : (float)(1.0 / std::sqrt((double)D));

  // per-head codec info and page layout
  std::vector<float> Mhost;
  std::vector<double> MT;        // per head: M_h^T widened to double, [128][r]
  const double* pb = d->proj_basis;
  p->heads.resize((size_t)p->L * p->Hkv);
  p->layer_off.resize(p->L);
  p->page_bytes.resize(p->L);
  p->stage_bytes.resize(p->L);
  uint64_t off = 0;
  for (int l = 0; l < p->L; ++l) {
    uint32_t poff = 0;
    int stage = 0;
    for (int h = 0; h < p->Hkv; ++h) {
      const size_t i = (size_t)l * p->Hkv + h;
      HeadInfo hi;
      std::memset(&hi, 0, sizeof(hi));
      const int kc = d->k_codec[i], vc = d->v_codec[i];
      if (!valid_codec(kc) || !valid_codec(vc)) { delete p; return fail(KVQ_ERR_UNSUPPORTED, "bad codec at layer %d head %d", l, h); }
      if (p->bf16 && (kc == KVQ_F16 || vc == KVQ_F16)) {
        delete p;
        return fail(KVQ_ERR_UNSUPPORTED, "bf16 plans keep raw rows in the tail only: no KVQ_F16 pages (layer %d head %d)", l, h);
      }
      const bool rank = (kc == KVQ_RANK || vc == KVQ_RANK);
      if (rank != (d->rot == KVQ_ROT_PROJECTION) && !(d->rot == KVQ_ROT_PROJECTION && kc == KVQ_F16 && vc == KVQ_F16)) {
        delete p;
        return fail(KVQ_ERR_UNSUPPORTED, "KVQ_RANK codecs need rot = PROJECTION and vice versa (layer %d head %d)", l, h);
      }
      int r = D, kb = 0, vb = 0;
      if (d->rot == KVQ_ROT_PROJECTION) {
        r = d->rank[i]; kb = d->k_bits[i]; vb = d->v_bits[i];
        if (!valid_rank(r) || kb < 1 || kb > 4 || vb < 1 || vb > 4) {
          delete p;
          return fail(KVQ_ERR_UNSUPPORTED, "rank must be 16/32/64/96/128 and bits 1..4 (layer %d head %d)", l, h);
        }
      }
      hi.kcodec = (uint8_t)kc; hi.vcodec = (uint8_t)vc; hi.r = (uint8_t)r;
      hi.kbits = (uint8_t)(kc == KVQ_RANK ? kb : codec_bits(kc));
      hi.vbits = (uint8_t)(vc == KVQ_RANK ? vb : codec_bits(vc));
      int cbK, sbK, cbV, sbV;
      row_bytes(kc, r, kb, &cbK, &sbK);
      row_bytes(vc, r, vb, &cbV, &sbV);
      hi.cbK = (uint16_t)cbK; hi.sbK = (uint16_t)sbK; hi.cbV = (uint16_t)cbV; hi.sbV = (uint16_t)sbV;
      hi.off = poff;
      hi.bytes = (uint32_t)(PAGE * (cbK + sbK + cbV + sbV));
      poff += hi.bytes;
      stage = std::max(stage, (int)hi.bytes);
      if (d->rot == KVQ_ROT_PROJECTION) {
        // M_h = R_r P_h^T with R_r = H_r / sqrt(r) (Sylvester H; block-diagonal H_32 for
        // r = 96): entry (i, c) is the sum over k of H[i][k] P[c][k] within the block of
        // row i, taken in k order in double (every product is exact: H is +-1), times
        // 1/sqrt(block), rounded once to fp32.
        hi.m_off = (uint32_t)Mhost.size();
        const int blk = (r == 96) ? 32 : r;
        const double s = 1.0 / std::sqrt((double)blk);
        std::vector<float> M((size_t)r * D);
        for (int row = 0; row < r; ++row) {
          const int b0 = (row / blk) * blk, ii = row % blk;
          for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int k = 0; k < blk; ++k) {
              const double h = (__builtin_popcount((unsigned)(ii & k)) & 1) ? -1.0 : 1.0;
              acc += h * pb[(size_t)c * r + b0 + k];
            }
            M[(size_t)row * D + c] = (float)(acc * s);
          }
        }
        Mhost.insert(Mhost.end(), M.begin(), M.end());
        while (Mhost.size() % 4) Mhost.push_back(0.f);
        hi.mt_off = (uint32_t)MT.size();
        for (int c = 0; c < D; ++c)
          for (int row = 0; row < r; ++row) MT.push_back((double)M[(size_t)row * D + c]);
        pb += (size_t)D * r;
      }
      p->heads[i] = hi;
    }
    if (p->T > 0) stage = std::max(stage, TAIL_PAGE_BYTES);
    p->stage_bytes[l] = (stage + 127) & ~127;
    p->page_bytes[l] = poff;
    p->layer_off[l] = off;
    off += (uint64_t)poff * (uint64_t)p->n_pages;
    off = (off + 255) & ~(uint64_t)255;
  }
  p->tail_off = off;
  off += (uint64_t)p->max_seqs * p->L * p->Hkv * (uint64_t)p->T * (D * 2 * 2);
  p->cache_bytes = off;

  // device tables
  auto dmalloc = [&](void** ptr, size_t bytes) -> bool {
    if (std::getenv("KVQ_TEST_FAIL_ALLOC")) return false;
    return cudaMalloc(ptr, bytes) == cudaSuccess;
  };
  if (!dmalloc((void**)&p->d_err, sizeof(int)) ||
      !dmalloc((void**)&p->d_bt, sizeof(int) * (size_t)p->max_seqs * p->mpps)) {
    delete p;
    return fail(KVQ_ERR_OOM, "device allocation for the plan tables failed");
  }
  cudaMemset(p->d_err, 0, sizeof(int));
  if (d->rot == KVQ_ROT_VARNORM_HADAMARD) {
    const size_t n = (size_t)p->L * p->Hkv * 2 * D;
    std::vector<float> sk((size_t)p->L * p->Hkv * D), sv((size_t)p->L * p->Hkv * D);
    for (int l = 0; l < p->L; ++l)
      for (int h = 0; h < p->Hkv; ++h)
        for (int c = 0; c < D; ++c) {
          const float ik = d->inv_rms[(((size_t)l * p->Hkv + h) * 2 + 0) * D + c];
          const float iv = d->inv_rms[(((size_t)l * p->Hkv + h) * 2 + 1) * D + c];
          if (!(ik > 0.f) || !(iv > 0.f) || !std::isfinite(ik) || !std::isfinite(iv)) {
            delete p;
            return fail(KVQ_ERR_INVALID_ARG, "inv_rms must be finite and positive");
          }
          sk[((size_t)l * p->Hkv + h) * D + c] = (float)(1.0 / (double)ik);
          sv[((size_t)l * p->Hkv + h) * D + c] = (float)(1.0 / (double)iv);
        }
    if (!dmalloc((void**)&p->d_inv, n * 4) || !dmalloc((void**)&p->d_sk, sk.size() * 4) ||
        !dmalloc((void**)&p->d_sv, sv.size() * 4)) {
      delete p;
      return fail(KVQ_ERR_OOM, "device allocation for the variance tables failed");
    }
    cudaMemcpy(p->d_inv, d->inv_rms, n * 4, cudaMemcpyHostToDevice);
    cudaMemcpy(p->d_sk, sk.data(), sk.size() * 4, cudaMemcpyHostToDevice);
    cudaMemcpy(p->d_sv, sv.data(), sv.size() * 4, cudaMemcpyHostToDevice);
  }
  if (!Mhost.empty()) {
    if (!dmalloc((void**)&p->d_M, Mhost.size() * 4)) {
      delete p;
      return fail(KVQ_ERR_OOM, "device allocation for the projections failed");
    }
    cudaMemcpy(p->d_M, Mhost.data(), Mhost.size() * 4, cudaMemcpyHostToDevice);
    if (!dmalloc((void**)&p->d_MT, MT.size() * sizeof(double))) {
      delete p;
      return fail(KVQ_ERR_OOM, "device allocation for the projection transposes failed");
    }
    cudaMemcpy(p->d_MT, MT.data(), MT.size() * sizeof(double), cudaMemcpyHostToDevice);
  }
  p->len.assign((size_t)p->max_seqs * p->L, 0);
  p->bt.assign((size_t)p->max_seqs * p->mpps, -1);
  p->npages.assign(p->max_seqs, 0);
  std::vector<int> neg(p->bt.size(), -1);
  e = cudaMemcpy(p->d_bt, neg.data(), neg.size() * sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) { delete p; return cuda_fail(e, "block table init"); }
  p->reset_all();
  *out = p;
  return KVQ_OK;
}

void kvq_plan_destroy(kvq_plan* plan) { delete plan; }

kvq_status kvq_plan_cache_bytes(const kvq_plan* p, size_t* bytes) {
  if (!p || !bytes) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  *bytes = (size_t)p->cache_bytes;
  return KVQ_OK;
}

// Decode workspace: [split partials][projected queries (projection plans)][merge counters]
static size_t partial_bytes(const kvq_plan* p, int n_seqs) {
  return (size_t)n_seqs * p->Hkv * MAX_SPLITS * p->G * PARTIAL_FLOATS * sizeof(float);
}
static size_t qproj_bytes(const kvq_plan* p, int n_seqs) {
  return p->rot == KVQ_ROT_PROJECTION ? (size_t)n_seqs * p->Hq * D * sizeof(float) : 0;
}
// Workspace layout: [merge tickets for KVQ_MAX_BATCH entries][partials][projected
// queries].  The tickets sit at a fixed place whatever the call's entry count, so a
// workspace zeroed once serves every later call with at most as many entries.
static size_t ticket_bytes(const kvq_plan* p) { return ((size_t)MAX_BATCH * p->Hkv * sizeof(int) + 255) & ~(size_t)255; }
static size_t workspace_bytes(const kvq_plan* p, int n_seqs) {
  return ticket_bytes(p) + partial_bytes(p, n_seqs) + qproj_bytes(p, n_seqs);
}

kvq_status kvq_plan_workspace_bytes(const kvq_plan* p, int n_seqs, size_t* bytes) {
  if (!p || !bytes) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (n_seqs < 0 || n_seqs > MAX_BATCH) return fail(KVQ_ERR_INVALID_ARG, "n_seqs must be in [0, %d]", MAX_BATCH);
  *bytes = workspace_bytes(p, n_seqs);
  return KVQ_OK;
}

kvq_status kvq_cache_bind(kvq_plan* p, void* dev, size_t bytes) {
  if (!p || !dev) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if ((uintptr_t)dev % 256) return fail(KVQ_ERR_INVALID_ARG, "cache must be 256-byte aligned");
  if (bytes < p->cache_bytes) return fail(KVQ_ERR_INVALID_ARG, "cache has %zu bytes, plan needs %llu", bytes,
                                         (unsigned long long)p->cache_bytes);
  p->cache = (uint8_t*)dev;
  p->reset_all();
  std::vector<int> neg(p->bt.size(), -1);
  cudaError_t e = cudaMemcpy(p->d_bt, neg.data(), neg.size() * sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "block table reset");
  return KVQ_OK;
}

kvq_status kvq_append_quantize(kvq_plan* p, int layer, int n_seqs, const int* seq_ids, const int* n_new,
                               const void* k_new, const void* v_new, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (const kvq_status st = require_plan_device(p); st != KVQ_OK) return st;
  if (!p->cache) return fail(KVQ_ERR_STATE, "no cache bound");
  if (layer < 0 || layer >= p->L) return fail(KVQ_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (n_seqs < 0 || n_seqs > MAX_BATCH) return fail(KVQ_ERR_INVALID_ARG, "n_seqs must be in [0, %d]", MAX_BATCH);
  if (n_seqs == 0) return KVQ_OK;
  if (!seq_ids || !n_new) return fail(KVQ_ERR_INVALID_ARG, "null seq_ids or n_new");
  int64_t total = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    if (s < 0 || s >= p->max_seqs) return fail(KVQ_ERR_INVALID_ARG, "sequence id %d out of range", s);
    for (int j = 0; j < i; ++j)
      if (seq_ids[j] == s) return fail(KVQ_ERR_INVALID_ARG, "sequence id %d repeated", s);
    if (n_new[i] < 0) return fail(KVQ_ERR_INVALID_ARG, "negative n_new");
    if (p->len[(size_t)s * p->L + layer] + n_new[i] > p->max_tokens)
      return fail(KVQ_ERR_CAPACITY, "sequence %d would exceed max_tokens_per_seq", s);
    total += n_new[i];
  }
  if (total == 0) return KVQ_OK;
  if (!k_new || !v_new) return fail(KVQ_ERR_INVALID_ARG, "null k_new or v_new");
  if (((uintptr_t)k_new | (uintptr_t)v_new) % 16) return fail(KVQ_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  // pages: check capacity first, then allocate
  int64_t need = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    const int64_t nl = p->len[(size_t)s * p->L + layer] + n_new[i];
    const int64_t nq = nl > p->T ? nl - p->T : 0;
    const int pages = (int)((nq + PAGE - 1) / PAGE);
    need += std::max(0, pages - p->npages[s]);
  }
  if (need > (int64_t)p->free_pages.size()) return fail(KVQ_ERR_CAPACITY, "page pool exhausted (%lld pages needed, %zu free)",
                                                        (long long)need, p->free_pages.size());
  cudaStream_t st = (cudaStream_t)stream;
  std::vector<int> idx, val;
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    const int64_t nl = p->len[(size_t)s * p->L + layer] + n_new[i];
    const int64_t nq = nl > p->T ? nl - p->T : 0;
    const int pages = (int)((nq + PAGE - 1) / PAGE);
    while (p->npages[s] < pages) {
      const int pid = p->free_pages.back();
      p->free_pages.pop_back();
      const int j = p->npages[s]++;
      p->bt[(size_t)s * p->mpps + j] = pid;
      idx.push_back(s * p->mpps + j);
      val.push_back(pid);
    }
  }
  if (!idx.empty()) {
    cudaError_t e = launch_block_table_update(p->d_bt, (int)idx.size(), idx.data(), val.data(), st);
    if (e != cudaSuccess) return cuda_fail(e, "block table update");
  }
  // work items, in chunks of MAX_APPEND_SEQS sequences
  const int T = p->T;
  int row0 = 0;
  for (int c0 = 0; c0 < n_seqs; c0 += MAX_APPEND_SEQS) {
    const int cn = std::min(MAX_APPEND_SEQS, n_seqs - c0);
    AppendParams ap;
    std::memset(&ap, 0, sizeof(ap));
    ap.pool = p->cache + p->layer_off[layer];
    ap.page_bytes = p->page_bytes[layer];
    ap.block_table = p->d_bt;
    ap.max_pages_per_seq = p->mpps;
    ap.tail = p->cache + p->tail_off;
    ap.T = T; ap.L = p->L; ap.layer = layer; ap.Hkv = p->Hkv; ap.rot = p->rot; ap.bf16 = p->bf16;
    ap.k_in = (const __half*)k_new;
    ap.v_in = (const __half*)v_new;
    ap.inv_s = p->d_inv ? p->d_inv + (size_t)layer * p->Hkv * 2 * D : nullptr;
    ap.M = p->d_M;
    ap.err = p->d_err;
    for (int h = 0; h < p->Hkv; ++h) ap.heads[h] = p->head(layer, h);
    int items = 0, qitems = 0;
    for (int k = 0; k < cn; ++k) {
      const int i = c0 + k;
      const int s = seq_ids[i];
      const int64_t lo = p->len[(size_t)s * p->L + layer];
      const int64_t ln = lo + n_new[i];
      AppendSeq& q = ap.seqs[k];
      q.seq = s; q.len_old = (int)lo; q.in_row0 = row0; q.item0 = items;
      if (T == 0) {
        q.nE = 0; q.nP = n_new[i]; q.nF = 0; q.e0 = 0; q.f0 = (int)ln;
      } else {
        const int64_t e0 = std::max<int64_t>(0, lo - T);
        const int64_t e1 = std::min<int64_t>(lo, ln - T);
        q.e0 = (int)e0;
        q.nE = (int)std::max<int64_t>(0, e1 - e0);
        q.nP = (int)std::max<int64_t>(0, ln - T - lo);
        const int64_t f0 = std::max<int64_t>(lo, ln - T);
        q.f0 = (int)f0;
        q.nF = (int)(ln - f0);
      }
      q.qitem0 = qitems;
      items += q.nE + q.nP + q.nF;
      qitems += q.nE + q.nP;
      row0 += n_new[i];
    }
    ap.n_seqs = cn;
    ap.total_items = items;
    if (p->rot == KVQ_ROT_PROJECTION && qitems > 0) {
      // projection + quantization of the rows leaving (or bypassing) the tail; it
      // reads evicted rows from the ring, so it runs before the ring writes
      ProjParams pp;
      std::memset(&pp, 0, sizeof(pp));
      pp.pool = ap.pool; pp.page_bytes = ap.page_bytes; pp.block_table = ap.block_table;
      pp.max_pages_per_seq = ap.max_pages_per_seq; pp.tail = ap.tail;
      pp.T = T; pp.L = p->L; pp.layer = layer; pp.Hkv = p->Hkv;
      pp.k_in = ap.k_in; pp.v_in = ap.v_in; pp.in_stride = p->Hkv * D;
      pp.mt = p->d_MT; pp.err = p->d_err;
      pp.n_seqs = cn; pp.total_q = qitems;
      std::memcpy(pp.heads, ap.heads, sizeof(pp.heads));
      std::memcpy(pp.seqs, ap.seqs, sizeof(pp.seqs));
      cudaError_t e = launch_project(pp, qitems, p->Hkv, st);
      if (e != cudaSuccess) return cuda_fail(e, "projection launch");
    }
    cudaError_t e = launch_append(ap, st);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
  }
  for (int i = 0; i < n_seqs; ++i) p->len[(size_t)seq_ids[i] * p->L + layer] += n_new[i];
  return KVQ_OK;
}

}  // extern "C"

// A validated decode launch: parameters, grid and whether it uses the workspace.
struct DecodeLaunch {
  DecodeParams dp;
  int grid_x = 1;
  bool uses_ws = false;     // split-K partials / merge counters / projected queries live in the workspace
  bool proj = false;        // the projected-query kernel runs first
};

// Validate one decode launch over n_seqs entries (entry i attends sequence
// seq_ids[i] over its first lims[i] tokens, all of them when lims is null) and
// size it.  Nothing is enqueued; on failure the plan is unchanged.
static kvq_status decode_prepare(const kvq_plan* p, int layer, int n_seqs, const int* seq_ids, const int* lims,
                                 const void* q, float* out, void* workspace, size_t workspace_bytes_given,
                                 DecodeLaunch& L) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (!p->cache) return fail(KVQ_ERR_STATE, "no cache bound");
  if (layer < 0 || layer >= p->L) return fail(KVQ_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (n_seqs < 0 || n_seqs > MAX_BATCH) return fail(KVQ_ERR_INVALID_ARG, "n_seqs must be in [0, %d]", MAX_BATCH);
  if (n_seqs > 0 && (!seq_ids || !q || !out)) return fail(KVQ_ERR_INVALID_ARG, "null seq_ids, q or out");
  if (((uintptr_t)q % 16) || ((uintptr_t)out % 16)) return fail(KVQ_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  DecodeParams& dp = L.dp;
  dp = p->base_params(layer);
  dp.q = (const __half*)q;
  dp.out = out;
  dp.n_seqs = n_seqs;
  int maxq = 0, maxt = 0;         // most quantized / tail pages of one entry
  for (int i = 0; i < n_seqs; ++i) {
    const int s = seq_ids[i];
    if (s < 0 || s >= p->max_seqs) return fail(KVQ_ERR_INVALID_ARG, "sequence id %d out of range", s);
    const int64_t len = p->len[(size_t)s * p->L + layer];
    dp.seq[i] = s;
    dp.len[i] = (int)len;
    dp.lim[i] = lims ? lims[i] : (int)len;
    if (dp.lim[i] < 0 || dp.lim[i] > len) return fail(KVQ_ERR_INVALID_ARG, "visible length %d outside [0, %lld]",
                                                       dp.lim[i], (long long)len);
    const SplitCounts c = split_counts((int)len, (int)p->T, 1, 1, dp.lim[i]);
    maxq = std::max(maxq, c.nqp);
    maxt = std::max(maxt, c.ntp);
  }
  L.grid_x = 1;
  L.uses_ws = false;
  L.proj = p->rot == KVQ_ROT_PROJECTION;
  if (n_seqs == 0) return KVQ_OK;
  dp.stage_bytes = p->stage_bytes[layer];
  // The consumer warps keep their weight tables in the K region of their current
  // stage unless some head's (or the tail's) K rows are smaller than a table.
  dp.wtab_smem = 0;
  for (int h = 0; h < p->Hkv; ++h) {
    const HeadInfo& hi = p->head(layer, h);
    if ((uint32_t)PAGE * (uint32_t)(hi.cbK + hi.sbK) < wtab_bytes(p->G)) dp.wtab_smem = 1;
  }
  if (p->T > 0 && (uint32_t)TAIL_TOK * (uint32_t)(2 * D) < wtab_bytes(p->G)) dp.wtab_smem = 1;
  // Stage ring: one stage per consumer warp at least, deeper while the CTAs per SM
  // that the register allocation aims at still fit in shared memory.
  const int want_ctas = DECODE_MIN_CTAS(p->G);
  dp.n_stages = NCW;
  for (int ns = 8; ns > NCW; --ns)
    if (decode_smem_bytes(dp.stage_bytes, ns, p->G, dp.wtab_smem) + 1024 <= (size_t)((228 * 1024) / want_ctas)) {
      dp.n_stages = ns;
      break;
    }
  const size_t smem = decode_smem_bytes(dp.stage_bytes, dp.n_stages, p->G, dp.wtab_smem);
  // Split sizes, per kv head.  A quantized page counts as one unit of work for
  // the block codecs (a layer's heads share a codec in the workloads) and a
  // 16-row tail tile as half a unit.  For the rank codec the measured per-tile
  // time of a CTA grows with the head's bit width and hardly with its rank (the
  // loops' fixed work per tile dominates): 0.86, 0.95, 1.35 and 1.45 us per tile
  // at 1 .. 4 bits (config-4 layer, one wave), modelled as 0.7 + 0.18 b units.
  // Each head's split size is P / cost, so full splits of every head cost about
  // the same.  P is the candidate with the smallest estimated makespan: the
  // largest of (the costliest split) and (the average split cost x the waves of
  // resident CTAs, registers and shared memory both counted), where a split of n
  // tiles costs ceil(n / consumer warps) rounds of its tiles plus a fixed cost of
  // three units (query preparation, publishing the partial).  Candidates cover the
  // sizes just above one full wave of CTAs one by one, so a sequence whose pages
  // would spill a few CTAs into a second wave gets a slightly larger split.
  const int per_sm = std::max(1, decode_blocks_per_sm(p->G, smem));
  const int64_t target = (int64_t)p->num_sms * per_sm;
  std::vector<double> cq(p->Hkv, 1.0);
  for (int h = 0; h < p->Hkv; ++h) {
    const HeadInfo& hi = p->head(layer, h);
    if (hi.kcodec == KVQ_RANK) cq[h] = 0.7 + 0.18 * std::max(hi.kbits, hi.vbits);
  }
  const double cmin = *std::min_element(cq.begin(), cq.end());
  const double ct = 0.5 * cmin;
  const int min_q = std::max(1, (maxq + MAX_SPLITS - 3) / (MAX_SPLITS - 2));
  const int min_t = std::max(1, (maxt + 1) / 2);
  auto sizes = [&](int P, std::vector<int>& ppq, int& ppt) {
    ppq.resize(p->Hkv);
    for (int h = 0; h < p->Hkv; ++h)
      ppq[h] = std::max(min_q, (int)std::lround((double)P * cmin / cq[h]));
    ppt = std::max(min_t, (int)std::lround((double)P * cmin / ct));
    if (p->debug_pps > 0) {                                   // fixed split size (tests)
      for (int h = 0; h < p->Hkv; ++h) ppq[h] = std::max(min_q, p->debug_pps);
      ppt = std::max(min_t, p->debug_pps);
    }
  };
  auto makespan = [&](int P) {
    std::vector<int> ppq;
    int ppt;
    sizes(P, ppq, ppt);
    int64_t ctas = 0;
    double total = 0.0, worst = 0.0;
    // splits of n pages of size pp, each costing rounds of tiles of cost c
    auto add = [&](int n, int pp, double c) {
      if (n <= 0) return;
      const int full = n / pp, rest = n - full * pp;
      const double cf = (double)((pp + NCW - 1) / NCW) * NCW * c + 3.0 * cmin;
      total += full * cf;
      ctas += full;
      if (full) worst = std::max(worst, cf);
      if (rest) {
        const double cr = (double)((rest + NCW - 1) / NCW) * NCW * c + 3.0 * cmin;
        total += cr;
        ++ctas;
        worst = std::max(worst, cr);
      }
    };
    for (int i = 0; i < n_seqs; ++i) {
      const SplitCounts c = split_counts(dp.len[i], (int)p->T, 1, 1, dp.lim[i]);
      for (int h = 0; h < p->Hkv; ++h) {
        add(c.nqp, ppq[h], cq[h]);
        add(c.ntp, ppt, ct);
      }
    }
    const int64_t waves = (ctas + target - 1) / target;
    return std::max(worst, (double)waves * total / (double)std::max<int64_t>(ctas, 1));
  };
  int64_t unit_pages = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const SplitCounts c = split_counts(dp.len[i], (int)p->T, 1, 1, dp.lim[i]);
    for (int h = 0; h < p->Hkv; ++h) unit_pages += (int64_t)std::lround(c.nqp * cq[h] / cmin + c.ntp * ct / cmin);
  }
  const int P0 = std::max<int>(1, (int)((unit_pages + target - 1) / target));
  int best_P = P0;
  double best = makespan(P0);
  std::vector<int> cands = {4, 6, 8, 10, 12, 16, 24, 32, 48, 64, 96, 128};
  for (int P = P0 + 1; P <= P0 + std::min(P0 / 2 + 1, 24); ++P) cands.push_back(P);
  for (int cand : cands) {
    if (cand == P0) continue;
    const double m = makespan(cand);
    if (m < best * 0.999) { best = m; best_P = cand; }
  }
  std::vector<int> ppq;
  int ppt = 1;
  sizes(best_P, ppq, ppt);
  for (int h = 0; h < p->Hkv; ++h) dp.pps[h] = (uint16_t)ppq[h];
  dp.pps_t = ppt;
  // CTA order of the launch (decode_item): full quantized splits, partial ones
  // largest first, tail splits, zero-writing items
  int max_splits = 0;
  L.grid_x = build_decode_order(dp, &max_splits);
  if (max_splits > 1 || L.proj) {
    const size_t need = workspace_bytes(p, n_seqs);
    if (!workspace || workspace_bytes_given < need)
      return fail(KVQ_ERR_INVALID_ARG, "workspace of %zu bytes needed (got %zu)", need, workspace_bytes_given);
    if ((uintptr_t)workspace % 16) return fail(KVQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    dp.tickets = (int*)workspace;
    dp.ws = (float*)((char*)workspace + ticket_bytes(p));
    dp.qproj = (float*)((char*)workspace + ticket_bytes(p) + partial_bytes(p, n_seqs));
    L.uses_ws = true;
  }
  return KVQ_OK;
}

static kvq_status decode_enqueue(const DecodeLaunch& L, void* stream) {
  if (L.dp.n_seqs == 0) return KVQ_OK;
  if (L.proj) {
    cudaError_t e = launch_project_query(L.dp, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "query projection launch");
  }
  cudaError_t e = launch_decode(L.dp, L.grid_x, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return KVQ_OK;
}

static kvq_status decode_launch(kvq_plan* p, int layer, int n_seqs, const int* seq_ids, const int* lims,
                                const void* q, float* out, void* workspace, size_t workspace_bytes_given,
                                void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (const kvq_status st = require_plan_device(p); st != KVQ_OK) return st;
  DecodeLaunch L;
  const kvq_status st = decode_prepare(p, layer, n_seqs, seq_ids, lims, q, out, workspace, workspace_bytes_given, L);
  if (st != KVQ_OK) return st;
  return decode_enqueue(L, stream);
}

extern "C" {

kvq_status kvq_decode_attention(kvq_plan* p, int layer, int n_seqs, const int* seq_ids, const void* q, float* out,
                                void* workspace, size_t workspace_bytes_given, void* stream) {
  return decode_launch(p, layer, n_seqs, seq_ids, nullptr, q, out, workspace, workspace_bytes_given, stream);
}

// The tensor-core prefill takes a layer whose heads all store block codecs (the
// kernel dequantizes 32-value blocks; F16 pages and the rank codec go through the
// decode kernel) under a rotation other than the projection, when two raw stages
// of the largest page-head fit beside its operand buffers.
static bool prefill_tc_layout(const kvq_plan* p, int layer, int* stage_bytes, int* n_raw) {
  if (p->rot == KVQ_ROT_PROJECTION) return false;
  int sb = 0;
  for (int h = 0; h < p->Hkv; ++h) {
    const HeadInfo& hi = p->head(layer, h);
    for (int c : {(int)hi.kcodec, (int)hi.vcodec})
      if (c == KVQ_F16 || c == KVQ_RANK) return false;
    if (hi.cbK % 16 || hi.cbV % 16 || hi.off % 16 || hi.bytes % 16) return false;
    sb = std::max(sb, (int)hi.bytes);
  }
  sb = (sb + 127) & ~127;
  const int n = prefill_raw_stages(sb);
  if (n < 2) return false;
  *stage_bytes = sb;
  *n_raw = n;
  return true;
}

kvq_status kvq_prefill_attention(kvq_plan* p, int layer, int seq_id, int n_q, const void* q, float* out,
                                 void* workspace, size_t workspace_bytes_given, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (const kvq_status st = require_plan_device(p); st != KVQ_OK) return st;
  if (!p->cache) return fail(KVQ_ERR_STATE, "no cache bound");
  if (layer < 0 || layer >= p->L) return fail(KVQ_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (seq_id < 0 || seq_id >= p->max_seqs) return fail(KVQ_ERR_INVALID_ARG, "sequence id %d out of range", seq_id);
  const int64_t len = p->len[(size_t)seq_id * p->L + layer];
  if (n_q < 0 || n_q > len) return fail(KVQ_ERR_INVALID_ARG, "n_q %d outside [0, %lld]", n_q, (long long)len);
  if (n_q == 0) return KVQ_OK;
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "null q or out");
  int stage_bytes = 0, n_raw = 0;
  if (p->prefill_path == 0 && prefill_tc_layout(p, layer, &stage_bytes, &n_raw)) {
    if (((uintptr_t)q % 16) || ((uintptr_t)out % 16)) return fail(KVQ_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
    const DecodeParams dp = p->base_params(layer);
    PrefillParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.pool = dp.pool;
    pp.page_bytes = dp.page_bytes;
    pp.bt = p->d_bt + (size_t)seq_id * p->mpps;
    pp.ring = dp.tail + ((size_t)seq_id * p->L + layer) * p->Hkv * (size_t)p->T * (D * 2 * 2);
    pp.T = (int)p->T;
    pp.len = (int)len;
    pp.nq_all = len > p->T ? (int)(len - p->T) : 0;
    pp.n_q = n_q;
    pp.Hq = p->Hq;
    pp.Hkv = p->Hkv;
    pp.G = p->G;
    pp.QB = 128 / p->G;
    pp.rot = p->rot;
    pp.bf16 = p->bf16;
    pp.q = (const __half*)q;
    pp.out = out;
    pp.s_k = dp.s_k;
    pp.s_v = dp.s_v;
    pp.inv_s = (p->rot == KVQ_ROT_VARNORM_HADAMARD && p->d_inv) ? p->d_inv + (size_t)layer * p->Hkv * 2 * D : nullptr;
    pp.qscale = dp.qscale;
    pp.stage_bytes = stage_bytes;
    pp.n_raw = n_raw;
    pp.err = dp.err;
    pp.wait_ns = dp.wait_ns;
    for (int h = 0; h < p->Hkv; ++h) pp.heads[h] = dp.heads[h];
    cudaError_t e = launch_prefill(pp, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
    return KVQ_OK;
  }
  int ids[MAX_BATCH], lims[MAX_BATCH];
  for (int c0 = 0; c0 < n_q; c0 += MAX_BATCH) {
    const int n = std::min(MAX_BATCH, n_q - c0);
    for (int i = 0; i < n; ++i) {
      ids[i] = seq_id;
      lims[i] = (int)(len - n_q + c0 + i + 1);          // query c0 + i sits at position len - n_q + c0 + i
    }
    const kvq_status st = decode_launch(p, layer, n, ids, lims, (const char*)q + (size_t)c0 * p->Hq * D * 2,
                                        out + (size_t)c0 * p->Hq * D, workspace, workspace_bytes_given, stream);
    if (st != KVQ_OK) return st;
  }
  return KVQ_OK;
}

kvq_status kvq_decode_attention_noalloc(kvq_plan* p, int layer, int n_seqs, const int* seq_ids, const void* q,
                                        float* out, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (n_seqs < 0 || n_seqs > MAX_BATCH) return fail(KVQ_ERR_INVALID_ARG, "n_seqs must be in [0, %d]", MAX_BATCH);
  // the scratch array is looked up on the current device: it must be the plan's
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != p->device)
    return fail(KVQ_ERR_STATE, "current device %d is not the plan's device %d", dev, p->device);
  const size_t need = workspace_bytes(p, n_seqs);
  if (need > NOALLOC_SCRATCH_BYTES)
    return fail(KVQ_ERR_CAPACITY, "decode of %d sequences needs %zu bytes of scratch; the built-in array holds %zu "
                "(use kvq_decode_attention with a workspace)", n_seqs, need, NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  e = noalloc_scratch(p->device, &scratch);
  if (e != cudaSuccess) return cuda_fail(e, "scratch address lookup");
  // every argument is checked before anything is enqueued
  DecodeLaunch L;
  const kvq_status st = decode_prepare(p, layer, n_seqs, seq_ids, nullptr, q, out, scratch, NOALLOC_SCRATCH_BYTES, L);
  if (st != KVQ_OK) return st;
  // merge counters must start at zero (partials are written before they are read)
  const size_t tickets = (size_t)n_seqs * p->Hkv * sizeof(int);
  if (L.uses_ws && tickets) {
    e = cudaMemsetAsync(scratch, 0, tickets, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "scratch counter reset");
  }
  return decode_enqueue(L, stream);
}

kvq_status kvq_dequantize(const kvq_plan* p, int layer, int seq_id, int64_t t0, int64_t t1, float* k_out,
                          float* v_out, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (const kvq_status st = require_plan_device(p); st != KVQ_OK) return st;
  if (!p->cache) return fail(KVQ_ERR_STATE, "no cache bound");
  if (layer < 0 || layer >= p->L) return fail(KVQ_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (seq_id < 0 || seq_id >= p->max_seqs) return fail(KVQ_ERR_INVALID_ARG, "sequence id out of range");
  const int64_t len = p->len[(size_t)seq_id * p->L + layer];
  if (t0 < 0 || t1 < t0 || t1 > len) return fail(KVQ_ERR_INVALID_ARG, "rows [%lld, %lld) outside [0, %lld)",
                                                 (long long)t0, (long long)t1, (long long)len);
  if (((uintptr_t)k_out | (uintptr_t)v_out) % 16) return fail(KVQ_ERR_INVALID_ARG, "outputs must be 16-byte aligned");
  DecodeParams dp = p->base_params(layer);
  dp.len[0] = (int)len;
  cudaError_t e = launch_dequantize(dp, seq_id, t0, t1, k_out, v_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return KVQ_OK;
}

kvq_status kvq_row_bytes(const kvq_plan* p, int layer, int head, int kv, int* cb, int* sb) {
  if (!p || !cb || !sb) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (layer < 0 || layer >= p->L || head < 0 || head >= p->Hkv || (kv != 0 && kv != 1))
    return fail(KVQ_ERR_INVALID_ARG, "layer, head or kv out of range");
  const HeadInfo& h = p->head(layer, head);
  *cb = kv ? h.cbV : h.cbK;
  *sb = kv ? h.sbV : h.sbK;
  return KVQ_OK;
}

kvq_status kvq_read_rows(const kvq_plan* p, int layer, int seq_id, int64_t t0, int64_t t1, int kv, void* codes,
                         void* scales, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (const kvq_status st = require_plan_device(p); st != KVQ_OK) return st;
  if (!p->cache) return fail(KVQ_ERR_STATE, "no cache bound");
  if (layer < 0 || layer >= p->L || (kv != 0 && kv != 1)) return fail(KVQ_ERR_INVALID_ARG, "layer or kv out of range");
  if (seq_id < 0 || seq_id >= p->max_seqs) return fail(KVQ_ERR_INVALID_ARG, "sequence id out of range");
  const int64_t len = p->len[(size_t)seq_id * p->L + layer];
  const int64_t nq = len > p->T ? len - p->T : 0;
  if (t0 < 0 || t1 < t0 || t1 > nq) return fail(KVQ_ERR_INVALID_ARG, "rows must lie in the quantized range [0, %lld)", (long long)nq);
  if (!codes || !scales) return fail(KVQ_ERR_INVALID_ARG, "null output");
  DecodeParams dp = p->base_params(layer);
  cudaError_t e = launch_read_rows(dp, seq_id, t0, t1, kv, (uint8_t*)codes, (uint8_t*)scales, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "read_rows launch");
  return KVQ_OK;
}

// New layout of one layer for the codecs kc[h], vc[h] (block codecs or F16, not the
// rank codec): head infos with region offsets, the page bytes and the stage bytes.
static kvq_status regrade_layout(const kvq_plan* p, int layer, const int* kc, const int* vc,
                                 std::vector<HeadInfo>& heads, uint32_t& page_bytes, int& stage) {
  if (p->bf16)
    for (int h = 0; h < p->Hkv; ++h)
      if (kc[h] == KVQ_F16 || vc[h] == KVQ_F16)
        return fail(KVQ_ERR_UNSUPPORTED, "bf16 plans keep raw rows in the tail only: no KVQ_F16 pages");
  if (p->rot == KVQ_ROT_PROJECTION) return fail(KVQ_ERR_UNSUPPORTED, "regrade of projection plans is not supported");
  heads.assign(p->Hkv, HeadInfo{});
  uint32_t poff = 0;
  stage = 0;
  for (int h = 0; h < p->Hkv; ++h) {
    const HeadInfo& old = p->head(layer, h);
    const int nk = kc[h], nv = vc[h];
    if (!valid_codec(nk) || !valid_codec(nv) || nk == KVQ_RANK || nv == KVQ_RANK)
      return fail(KVQ_ERR_UNSUPPORTED, "head %d: regrade targets must be block codecs or F16", h);
    if ((nk == KVQ_F16 && old.kcodec != KVQ_F16) || (nv == KVQ_F16 && old.vcodec != KVQ_F16))
      return fail(KVQ_ERR_UNSUPPORTED, "head %d: a quantized row cannot be regraded to F16", h);
    HeadInfo hi;
    std::memset(&hi, 0, sizeof(hi));
    hi.kcodec = (uint8_t)nk; hi.vcodec = (uint8_t)nv; hi.r = (uint8_t)D;
    hi.kbits = (uint8_t)codec_bits(nk); hi.vbits = (uint8_t)codec_bits(nv);
    int cbK, sbK, cbV, sbV;
    row_bytes(nk, D, 0, &cbK, &sbK);
    row_bytes(nv, D, 0, &cbV, &sbV);
    hi.cbK = (uint16_t)cbK; hi.sbK = (uint16_t)sbK; hi.cbV = (uint16_t)cbV; hi.sbV = (uint16_t)sbV;
    hi.off = poff;
    hi.bytes = (uint32_t)(PAGE * (cbK + sbK + cbV + sbV));
    poff += hi.bytes;
    stage = std::max(stage, (int)hi.bytes);
    heads[h] = hi;
  }
  if (p->T > 0) stage = std::max(stage, TAIL_PAGE_BYTES);
  stage = (stage + 127) & ~127;
  page_bytes = poff;
  if (page_bytes > p->page_bytes[layer])
    return fail(KVQ_ERR_CAPACITY, "regrade must not grow the layer's pages (%u -> %u bytes)", p->page_bytes[layer],
                page_bytes);
  return KVQ_OK;
}

kvq_status kvq_plan_regrade_bytes(const kvq_plan* p, int layer, const int* k_codec, const int* v_codec, size_t* bytes) {
  if (!p || !k_codec || !v_codec || !bytes) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (layer < 0 || layer >= p->L) return fail(KVQ_ERR_INVALID_ARG, "layer %d out of range", layer);
  std::vector<HeadInfo> heads;
  uint32_t pb = 0;
  int stage = 0;
  const kvq_status st = regrade_layout(p, layer, k_codec, v_codec, heads, pb, stage);
  if (st != KVQ_OK) return st;
  *bytes = (size_t)pb * (size_t)p->n_pages;
  return KVQ_OK;
}

kvq_status kvq_regrade_layer(kvq_plan* p, int layer, const int* k_codec, const int* v_codec, void* scratch,
                             size_t scratch_bytes, void* stream) {
  if (!p || !k_codec || !v_codec) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (const kvq_status st = require_plan_device(p); st != KVQ_OK) return st;
  if (!p->cache) return fail(KVQ_ERR_STATE, "no cache bound");
  if (layer < 0 || layer >= p->L) return fail(KVQ_ERR_INVALID_ARG, "layer %d out of range", layer);
  std::vector<HeadInfo> heads;
  uint32_t pb = 0;
  int stage = 0;
  kvq_status st = regrade_layout(p, layer, k_codec, v_codec, heads, pb, stage);
  if (st != KVQ_OK) return st;
  const size_t need = (size_t)pb * (size_t)p->n_pages;
  if (need && (!scratch || scratch_bytes < need))
    return fail(KVQ_ERR_INVALID_ARG, "scratch of %zu bytes needed (got %zu)", need, scratch_bytes);
  if ((uintptr_t)scratch % 16) return fail(KVQ_ERR_INVALID_ARG, "scratch must be 16-byte aligned");
  const cudaStream_t s = (cudaStream_t)stream;
  RegradeParams rp;
  std::memset(&rp, 0, sizeof(rp));
  rp.src_pool = p->cache + p->layer_off[layer];
  rp.src_page_bytes = p->page_bytes[layer];
  rp.dst_pool = (uint8_t*)scratch;
  rp.dst_page_bytes = pb;
  rp.block_table = p->d_bt;
  rp.max_pages_per_seq = p->mpps;
  rp.Hkv = p->Hkv;
  rp.rot = p->rot;
  rp.bf16 = p->bf16;
  rp.inv_s = p->d_inv ? p->d_inv + (size_t)layer * p->Hkv * 2 * D : nullptr;
  rp.err = p->d_err;
  for (int h = 0; h < p->Hkv; ++h) { rp.src[h] = p->head(layer, h); rp.dst[h] = heads[h]; }
  // every sequence's quantized rows, MAX_REGRADE_SEQS sequences per launch
  for (int s0 = 0; s0 < p->max_seqs; s0 += MAX_REGRADE_SEQS) {
    rp.n_seqs = 0;
    rp.total_rows = 0;
    for (int sq = s0; sq < std::min(p->max_seqs, s0 + MAX_REGRADE_SEQS); ++sq) {
      const int64_t len = p->len[(size_t)sq * p->L + layer];
      const int64_t nq = len > p->T ? len - p->T : 0;
      if (nq <= 0) continue;
      rp.seq[rp.n_seqs] = sq;
      rp.row0[rp.n_seqs] = rp.total_rows;
      rp.total_rows += nq;
      ++rp.n_seqs;
    }
    rp.row0[rp.n_seqs] = rp.total_rows;
    const cudaError_t e = launch_regrade(rp, s);
    if (e != cudaSuccess) return cuda_fail(e, "regrade launch");
  }
  if (need) {
    const cudaError_t e = cudaMemcpyAsync(p->cache + p->layer_off[layer], scratch, need, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "regrade copy-back");
  }
  for (int h = 0; h < p->Hkv; ++h) p->heads[(size_t)layer * p->Hkv + h] = heads[h];
  p->page_bytes[layer] = pb;
  p->stage_bytes[layer] = stage;
  return KVQ_OK;
}

kvq_status kvq_plan_bytes_in_use(const kvq_plan* p, int64_t* bytes) {
  if (!p || !bytes) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  int64_t pages = 0;
  for (int s = 0; s < p->max_seqs; ++s) pages += p->npages[s];
  int64_t b = 0;
  for (int l = 0; l < p->L; ++l) b += pages * (int64_t)p->page_bytes[l];
  *bytes = b + (int64_t)(p->cache_bytes - p->tail_off);
  return KVQ_OK;
}

kvq_status kvq_seq_length(const kvq_plan* p, int seq_id, int layer, int64_t* len) {
  if (!p || !len) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (seq_id < 0 || seq_id >= p->max_seqs || layer < 0 || layer >= p->L)
    return fail(KVQ_ERR_INVALID_ARG, "sequence or layer out of range");
  *len = p->len[(size_t)seq_id * p->L + layer];
  return KVQ_OK;
}

kvq_status kvq_seq_reset(kvq_plan* p, int seq_id) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (seq_id < 0 || seq_id >= p->max_seqs) return fail(KVQ_ERR_INVALID_ARG, "sequence id out of range");
  for (int l = 0; l < p->L; ++l) p->len[(size_t)seq_id * p->L + l] = 0;
  for (int j = 0; j < p->npages[seq_id]; ++j) {
    int& slot = p->bt[(size_t)seq_id * p->mpps + j];
    p->free_pages.push_back(slot);
    slot = -1;
  }
  p->npages[seq_id] = 0;
  // the device table keeps stale ids for this sequence; they are overwritten
  // before any read because reads are bounded by the (now zero) lengths.
  return KVQ_OK;
}

kvq_status kvq_calibrate_varnorm(int64_t n_tokens, int n_channels, int64_t row_stride, const void* x, float* inv_rms,
                                 void* stream) {
  if (n_tokens < 1 || n_channels < 1 || row_stride < n_channels) return fail(KVQ_ERR_INVALID_ARG, "bad sizes");
  if (!x || !inv_rms) return fail(KVQ_ERR_INVALID_ARG, "null pointer");
  cudaError_t e = launch_calibrate(n_tokens, n_channels, row_stride, (const __half*)x, inv_rms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "calibrate launch");
  return KVQ_OK;
}

kvq_status kvq_check_device_error(kvq_plan* p, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpy(&v, p->d_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "error word read");
  if (v == 0) return KVQ_OK;
  cudaMemset(p->d_err, 0, sizeof(int));
  if (v & ERR_TIMEOUT) return fail(KVQ_ERR_TIMEOUT, "a bounded wait inside a kernel ran out (error word 0x%x)", v);
  return fail(KVQ_ERR_DEVICE, "a kernel latched device error word 0x%x (1 = missing page)", v);
}

kvq_status kvq_microbench(int kind, int iters, int ctas, const void* buf, size_t buf_bytes, void* sink, double* work,
                          void* stream) {
  if (kind < KVQ_UB_FFMA || kind > KVQ_UB_READ) return fail(KVQ_ERR_INVALID_ARG, "bad micro-benchmark kind %d", kind);
  if (iters < 1 || iters > (1 << 20)) return fail(KVQ_ERR_INVALID_ARG, "iters must be in [1, 2^20]");
  if (ctas < 1 || ctas > 65536) return fail(KVQ_ERR_INVALID_ARG, "ctas must be in [1, 65536]");
  if (!sink || !work) return fail(KVQ_ERR_INVALID_ARG, "null sink or work");
  if (kind == KVQ_UB_READ && (!buf || buf_bytes < 16 || (uintptr_t)buf % 16))
    return fail(KVQ_ERR_INVALID_ARG, "the streaming read needs a 16-byte aligned buffer of at least 16 bytes");
  const cudaError_t e = launch_microbench(kind, iters, buf, buf_bytes, (unsigned long long*)sink, ctas,
                                          (cudaStream_t)stream, work);
  if (e != cudaSuccess) return cuda_fail(e, "micro-benchmark launch");
  return KVQ_OK;
}

kvq_status kvq_debug_set_prefill_path(kvq_plan* p, int path) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (path != 0 && path != 1) return fail(KVQ_ERR_INVALID_ARG, "path must be 0 or 1");
  p->prefill_path = path;
  return KVQ_OK;
}

kvq_status kvq_debug_set_decode_split(kvq_plan* p, int pages_per_split) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (pages_per_split < 0) return fail(KVQ_ERR_INVALID_ARG, "pages_per_split must be >= 0");
  p->debug_pps = pages_per_split;
  return KVQ_OK;
}

kvq_status kvq_debug_fault_injection(kvq_plan* p, int64_t wait_limit_ns, int drop_last_tile) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "null plan");
  if (wait_limit_ns < 1000 || wait_limit_ns > 2000000000ll)
    return fail(KVQ_ERR_INVALID_ARG, "wait_limit_ns must be in [1e3, 2e9]");
  if (drop_last_tile != 0 && drop_last_tile != 1) return fail(KVQ_ERR_INVALID_ARG, "drop_last_tile must be 0 or 1");
  p->wait_ns = (unsigned long long)wait_limit_ns;
  p->drop_last_tile = drop_last_tile;
  return KVQ_OK;
}

kvq_status kvq_debug_rotate(const kvq_plan* p, int layer, int head, int kv, int n, const void* x, float* y,
                            int layout, void* stream) {
  if (!p || !x || !y) return fail(KVQ_ERR_INVALID_ARG, "null argument");
  if (const kvq_status st = require_plan_device(p); st != KVQ_OK) return st;
  if (layout != KVQ_ROWS_WARP && layout != KVQ_ROWS_QUAD) return fail(KVQ_ERR_INVALID_ARG, "bad row layout");
  if (layer < 0 || layer >= p->L || head < 0 || head >= p->Hkv || (kv != 0 && kv != 1) || n < 0)
    return fail(KVQ_ERR_INVALID_ARG, "argument out of range");
  const HeadInfo& h = p->head(layer, head);
  if ((kv ? h.vcodec : h.kcodec) == KVQ_RANK) {
    ProjParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.k_in = (const __half*)x; pp.in_stride = D;
    pp.mt = p->d_MT; pp.err = p->d_err;
    pp.z_out = y; pp.head_override = head; pp.kv_override = kv;
    pp.total_q = n; pp.Hkv = p->Hkv;
    for (int hh = 0; hh < p->Hkv; ++hh) pp.heads[hh] = p->head(layer, hh);
    cudaError_t e = launch_project(pp, n, 1, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "projection launch");
    return KVQ_OK;
  }
  const float* inv = p->d_inv ? p->d_inv + (((size_t)layer * p->Hkv + head) * 2 + kv) * D : nullptr;
  cudaError_t e = launch_debug_rotate(h, p->rot, kv, inv, n, (const __half*)x, y, layout == KVQ_ROWS_QUAD, p->bf16,
                                      (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "debug_rotate launch");
  return KVQ_OK;
}

kvq_status kvq_debug_quantize_f32(int codec, int r, int b, int n_rows, const float* y, void* codes, void* scales,
                                  int layout, void* stream) {
  if (!valid_codec(codec)) return fail(KVQ_ERR_UNSUPPORTED, "bad codec");
  if (layout != KVQ_ROWS_WARP && layout != KVQ_ROWS_QUAD) return fail(KVQ_ERR_INVALID_ARG, "bad row layout");
  if (layout == KVQ_ROWS_QUAD && codec == KVQ_RANK) return fail(KVQ_ERR_UNSUPPORTED, "rank rows are warp rows");
  if (codec == KVQ_RANK && (!valid_rank(r) || b < 1 || b > 4)) return fail(KVQ_ERR_UNSUPPORTED, "bad rank or bits");
  if (n_rows < 0 || !y || !codes || (!scales && codec != KVQ_F16)) return fail(KVQ_ERR_INVALID_ARG, "bad argument");
  if (codec != KVQ_RANK) r = D;
  cudaError_t e = launch_debug_quantize(codec, r, b, n_rows, y, (uint8_t*)codes, (uint8_t*)scales,
                                        layout == KVQ_ROWS_QUAD, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "debug_quantize launch");
  return KVQ_OK;
}

}  // extern "C"
