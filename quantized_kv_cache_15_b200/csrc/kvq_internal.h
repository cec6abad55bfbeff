// Internal declarations of the kvq library (not part of the public ABI).
//
// Cache layout (all offsets in bytes, every region 128-byte aligned):
//   [layer 0 pool][layer 1 pool]...[layer L-1 pool][tail rings]
// A layer pool is n_pages pages; a page holds 64 consecutive token positions of
// one sequence for every kv head of that layer.  Inside a page, head h owns a
// contiguous region [K codes][K scales][V codes][V scales]:
//   K codes : 64 rows of cbK bytes, "interleaved": byte i of token t sits at
//             ((i / w) * 64 + t) * w + i % w, with w the largest of 16, 8, 4, 2
//             that divides cbK -- lane t of a warp reads its token's w-byte piece
//             next to lane t+1's (conflict-free, coalesced).
//   K scales: 64 rows of sbK bytes, row-major.
//   V codes : 64 rows of cbV bytes, row-major (lanes split one row's channels).
//   V scales: 64 rows of sbV bytes, row-major.
// Canonical packed rows (codes then scales) are defined by the quantizer: see
// quant.cuh.  The tail ring of (seq, layer, kv head) is T/TAIL_TOK tail pages of
// 8 KiB, each TAIL_TOK = 16 token slots: [K fp16, interleaved as above but with
// 16 rows: byte i of slot t at ((i / 16) * 16 + t) * 16 + i % 16][V fp16
// row-major]; token position p lives in ring slot p % T.  A tail page is one
// decode tile no larger than a quantized page-head of the common codecs, so a
// tail does not enlarge the decode kernel's stage ring.
#pragma once

#include <algorithm>
#include <cstdint>
#include <utility>
#include <vector>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/kvq.h"

namespace kvq {

constexpr int D = KVQ_HEAD_DIM;
constexpr int PAGE = KVQ_PAGE_TOKENS;
constexpr int MAX_HKV = KVQ_MAX_KV_HEADS;
constexpr int MAX_G = KVQ_MAX_GQA;
constexpr int MAX_BATCH = KVQ_MAX_BATCH;
constexpr int MAX_SPLITS = 64;            // split-K pieces per (sequence, kv head)
constexpr int TAIL_TOK = 16;                 // token slots per tail page
constexpr int TAIL_PAGE_BYTES = TAIL_TOK * D * 2 * 2;   // 8 KiB: K fp16 (interleaved) then V fp16
constexpr int PARTIAL_FLOATS = 4 + D;     // m, l, kind, pad, acc[128]
// Decode CTA shape: NCW consumer warps and one producer warp.
#ifndef KVQ_DECODE_CONSUMER_WARPS
#define KVQ_DECODE_CONSUMER_WARPS 4
#endif
constexpr int NCW = KVQ_DECODE_CONSUMER_WARPS;
constexpr int DECODE_THREADS = 32 * (NCW + 1);
// resident CTAs per SM the register allocation aims at (a build may fix it)
#ifdef KVQ_DECODE_MIN_CTAS
#define DECODE_MIN_CTAS(G) (KVQ_DECODE_MIN_CTAS)
#else
#define DECODE_MIN_CTAS(G) ((NCW <= 4) ? ((G) <= 4 ? 3 : 2) : ((G) <= 4 ? 2 : 1))
#endif
// unroll factors of the decode inner loops (score blocks, value token pairs)
#ifndef KVQ_SCORE_UNROLL
#define KVQ_SCORE_UNROLL 1
#endif
#ifndef KVQ_VDOT_UNROLL
#define KVQ_VDOT_UNROLL 4
#endif
#define KVQ_STR_(x) #x
#define KVQ_UNROLL(n) _Pragma(KVQ_STR_(unroll n))

// Split-K layout of one sequence of `len` tokens, shared by the host (grid size)
// and the decode kernel: the quantized segment in 64-token pages cut into splits
// of pps_q pages, then the tail segment in TAIL_TOK-token tail pages cut into
// splits of pps_t tail pages (a split never mixes the two).
// Splits of one (sequence, kv head) of length len whose query sees the first lim
// tokens (lim = len for decode; lim < len for the earlier queries of a prefill
// chunk).  nq: visible quantized tokens (pages in position order); nt: tail slots
// to visit.  While len <= T the tail holds positions 0 .. len-1 in slots 0 .. len-1,
// so the visible ones are the first lim slots.  Past that every slot is occupied
// and the visible positions nq_all .. lim-1 sit in a cyclic run of slots starting
// at nq_all mod T: all T slots are visited and the others are masked (tail_visible).
struct SplitCounts { int nq, nt, nqp, ntp, qsplits, tsplits, nq_all, nt_vis; };
__host__ __device__ inline SplitCounts split_counts(int len, int T, int pps_q, int pps_t, int lim) {
  SplitCounts c;
  c.nq_all = len > T ? len - T : 0;
  c.nq = c.nq_all < lim ? c.nq_all : lim;
  c.nt_vis = lim > c.nq_all ? lim - c.nq_all : 0;
  c.nt = len <= T ? c.nt_vis : (c.nt_vis > 0 ? T : 0);
  c.nqp = (c.nq + PAGE - 1) / PAGE;
  c.ntp = (c.nt + TAIL_TOK - 1) / TAIL_TOK;
  c.qsplits = (c.nqp + pps_q - 1) / pps_q;
  c.tsplits = (c.ntp + pps_t - 1) / pps_t;
  return c;
}
// Whether tail slot s holds a visible position (see split_counts).
__host__ __device__ inline bool tail_visible(const SplitCounts& c, int T, int s) {
  return ((s - c.nq_all % T) % T + T) % T < c.nt_vis;
}

// Device error word bits.
constexpr int ERR_NO_PAGE = 1;
constexpr int ERR_TIMEOUT = 2;
constexpr int ERR_BAD_ARG = 4;

struct HeadInfo {                // one (layer, kv head); 32 bytes
  uint8_t kcodec, vcodec;        // kvq_codec
  uint8_t r;                     // rank (KVQ_RANK), else 128
  uint8_t kbits, vbits;          // code bits of K / V (16 for F16)
  uint8_t pad[3];
  uint16_t cbK, sbK, cbV, sbV;   // canonical row bytes (codes, scales)
  uint32_t off;                  // region offset inside a page
  uint32_t bytes;                // region bytes = 64 * (cbK + sbK + cbV + sbV)
  uint32_t m_off;                // float offset of M_h (r x 128) in the projection table
  uint32_t mt_off;               // double offset of M_h^T (128 x r, exact widening) in the projection's table
};

__host__ __device__ inline int codec_bits(int c) {
  switch (c) {
    case KVQ_Q8_0: case KVQ_Q8_1: return 8;
    case KVQ_Q6_0: case KVQ_Q6_1: return 6;
    case KVQ_Q5_0: case KVQ_Q5_1: return 5;
    case KVQ_Q4_0: case KVQ_Q4_1: return 4;
    case KVQ_Q3_0: case KVQ_Q3_1: return 3;
    case KVQ_Q2_0: case KVQ_Q2_1: return 2;
    default: return 16;
  }
}
__host__ __device__ inline bool codec_is_asym(int c) { return (c >= KVQ_Q8_1 && c <= KVQ_Q2_1) || c == KVQ_Q5_1; }
__host__ __device__ inline int interleave_w(int cb) {
  return (cb % 16 == 0) ? 16 : (cb % 8 == 0) ? 8 : (cb % 4 == 0) ? 4 : 2;
}
// Canonical row bytes of a codec (n = 128, or r for KVQ_RANK).
__host__ __device__ inline void row_bytes(int codec, int r, int b, int* cb, int* sb) {
  int n = codec == KVQ_RANK ? r : D;
  int bits = codec == KVQ_RANK ? b : codec_bits(codec);
  int blk = n < 32 ? n : 32;
  int nb = n / blk;
  *cb = n * bits / 8;
  if (codec == KVQ_F16) *sb = 0;
  else if (codec == KVQ_RANK) *sb = 2 * nb;
  else *sb = codec_is_asym(codec) ? 4 * nb : 2 * nb;
}

// ---------------------------------------------------------------- append
struct AppendSeq {
  int seq;        // sequence id
  int len_old;    // tokens in this layer before the call
  int in_row0;    // first input row of this sequence
  int item0;      // first work item of this sequence
  int qitem0;     // first quantize item (E or P) of this sequence, over all sequences
  int nE, nP, nF; // evicted-from-tail, pass-through, final-tail-occupant counts
  int e0, f0;     // first evicted position, first final tail position
};
constexpr int MAX_APPEND_SEQS = 64;

struct AppendParams {
  uint8_t* pool;                 // this layer's page pool
  uint32_t page_bytes;
  const int* block_table;        // device [max_seqs][max_pages_per_seq]
  int max_pages_per_seq;
  uint8_t* tail;                 // tail region base (all sequences and layers)
  int T, L, layer, Hkv;
  int rot;
  int bf16;                      // raw rows (input, ring, F16 pages) are bf16, else fp16
  const __half* k_in;            // raw 16-bit rows (see bf16)
  const __half* v_in;
  const float* inv_s;            // [Hkv][2][128] of this layer, or null
  const float* M;                // projection table (floats), or null
  int* err;
  int n_seqs;
  int total_items;
  HeadInfo heads[MAX_HKV];
  AppendSeq seqs[MAX_APPEND_SEQS];
};

// Projection path: quantize items E and P of an append, or (z_out set) export
// z = M_h x for rows of k_in.
struct ProjParams {
  uint8_t* pool;
  uint32_t page_bytes;
  const int* block_table;
  int max_pages_per_seq;
  uint8_t* tail;
  int T, L, layer, Hkv;
  const __half* k_in;
  const __half* v_in;
  int in_stride;                 // halves between consecutive input rows
  const double* mt;              // M_h^T of every head, double [128][r] at heads[h].mt_off
  int* err;
  float* z_out;                  // inspection: z rows [total_q][r] (one head, one kv)
  int head_override, kv_override;
  int n_seqs;
  int total_q;                   // quantize items over all sequences
  HeadInfo heads[MAX_HKV];
  AppendSeq seqs[MAX_APPEND_SEQS];
};

// ---------------------------------------------------------------- decode
struct DecodeParams {
  const uint8_t* pool;
  uint32_t page_bytes;
  const int* block_table;
  int max_pages_per_seq;
  const uint8_t* tail;
  int T, L, layer, Hkv, Hq, G;
  int rot;
  int bf16;                      // raw rows (q, tail, F16 pages) are bf16, else fp16
  const __half* q;               // [n_seqs][Hq][128], raw 16-bit (see bf16)
  float* out;                    // [n_seqs][Hq][128]
  const float* s_k;              // [Hkv][128] per-channel K dequant multiplier (varnorm) or null
  const float* s_v;              // [Hkv][128] per-channel V multiplier or null
  const float* M;                // projection table (floats), or null
  float qscale;                  // softmax scale * log2(e)
  uint16_t pps[MAX_HKV];         // quantized pages per split, per kv head
  int pps_t;                     // tail pages per split
  // CTA order of the 1-D grid (see decode_item): every split of every entry, one CTA
  // per (split, kv head), longest first.
  int n_full, n_part, n_tail, n_zero;   // items of each kind
  int full0[MAX_BATCH + 1];      // prefix sums over entries of their full quantized splits (all heads)
  int tail0[MAX_BATCH + 1];      // prefix sums over entries of their tail splits
  uint8_t part_order[MAX_BATCH]; // entries with a partial quantized split, largest first
  uint8_t zero_order[MAX_BATCH]; // entries with nothing to attend to
  int stage_bytes;               // bytes of one pipeline stage
  int n_stages;                  // 4 or 8
  int wtab_smem;                 // 1: the weight tables get their own shared memory (some head's K rows are too small)
  float* ws;                     // partials [n_seqs*Hkv][G][MAX_SPLITS][PARTIAL_FLOATS]
  float* qproj;                  // projected queries M_h q [n_seqs][Hq][128] (projection plans)
  int* tickets;                  // [n_seqs*Hkv]
  int* err;
  unsigned long long wait_ns;    // bounded waits give up after this long (latching ERR_TIMEOUT)
  int drop_last_tile;            // test-only fault injection: producers skip their last tile
  int n_seqs;
  HeadInfo heads[MAX_HKV];
  int seq[MAX_BATCH];
  int len[MAX_BATCH];
  int lim[MAX_BATCH];            // tokens the entry's query sees (len, or fewer for prefill queries)
};

// The splits of a decode launch in CTA order.  The hardware hands out CTAs in
// grid order as slots free up, so the order is longest first: all full quantized
// splits (pps[head] pages each, the split sizes chosen so that full splits of
// every head cost about the same; entry by entry, kv head by kv head, splits in
// order), then, per entry that has any, one item per kv head for the entry's
// partial last quantized split (entries largest first; a head whose pages divide
// evenly gets an item that does nothing), then the tail splits (tail pages are
// 16-row tiles), and last one zero-writing item per entry with nothing to attend
// to; after the full splits, the kv head varies fastest.  kind: 0 quantized split,
// 1 tail split (split = index among the entry's splits, quantized first), 2
// nothing to attend (write zeros), 3 no work.
struct DecodeItem { int si, head, split, kind; };
__host__ __device__ inline int prefix_find(const int* pre, int n, int q) {
  // the entry e with pre[e] <= q < pre[e + 1] (pre non-decreasing, pre[0] = 0)
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= q) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__host__ __device__ inline DecodeItem decode_item(const DecodeParams& p, int b) {
  DecodeItem it;
  if (b < p.n_full) {
    it.si = prefix_find(p.full0, p.n_seqs, b);
    const int nqp = split_counts(p.len[it.si], p.T, 1, 1, p.lim[it.si]).nqp;
    int j = b - p.full0[it.si];
    int h = 0;
    for (; h < p.Hkv - 1; ++h) {                // the entry's full splits, head by head
      const int f = nqp / p.pps[h];
      if (j < f) break;
      j -= f;
    }
    it.head = h;
    it.split = j;
    it.kind = 0;
    return it;
  }
  it.head = (b - p.n_full) % p.Hkv;
  int q = (b - p.n_full) / p.Hkv;
  if (q < p.n_part) {
    it.si = p.part_order[q];
    const int nqp = split_counts(p.len[it.si], p.T, 1, 1, p.lim[it.si]).nqp;
    it.split = nqp / p.pps[it.head];
    it.kind = (nqp % p.pps[it.head]) ? 0 : 3;
    return it;
  }
  q -= p.n_part;
  if (q < p.n_tail) {
    it.si = prefix_find(p.tail0, p.n_seqs, q);
    const SplitCounts c = split_counts(p.len[it.si], p.T, p.pps[it.head], p.pps_t, p.lim[it.si]);
    it.split = c.qsplits + (q - p.tail0[it.si]);
    it.kind = 1;
    return it;
  }
  q -= p.n_tail;
  it.si = p.zero_order[q];
  it.split = 0;
  it.kind = 2;
  return it;
}

// Fill the CTA order of a decode launch (the fields decode_item reads) from the
// entries' lengths, visible lengths and split sizes; returns the grid size (items
// x kv heads) and the largest split count of one (entry, kv head) in *max_splits.
inline int build_decode_order(DecodeParams& dp, int* max_splits) {
  std::vector<std::pair<int, int>> parts;             // (pages of the largest partial split, entry)
  int nzero = 0, most = 0;
  dp.full0[0] = 0;
  dp.tail0[0] = 0;
  for (int i = 0; i < dp.n_seqs; ++i) {
    const SplitCounts c1 = split_counts(dp.len[i], dp.T, 1, dp.pps_t, dp.lim[i]);
    int full = 0, rest = 0;
    for (int h = 0; h < dp.Hkv; ++h) {
      full += c1.nqp / dp.pps[h];
      rest = std::max(rest, c1.nqp % (int)dp.pps[h]);
      const SplitCounts c = split_counts(dp.len[i], dp.T, dp.pps[h], dp.pps_t, dp.lim[i]);
      most = std::max(most, c.qsplits + c.tsplits);
    }
    dp.full0[i + 1] = dp.full0[i] + full;
    dp.tail0[i + 1] = dp.tail0[i] + c1.tsplits;
    if (rest) parts.emplace_back(rest, i);
    if (c1.nqp + c1.ntp == 0) dp.zero_order[nzero++] = (uint8_t)i;
  }
  std::stable_sort(parts.begin(), parts.end(),
                   [](const std::pair<int, int>& a, const std::pair<int, int>& b) { return a.first > b.first; });
  for (size_t k = 0; k < parts.size(); ++k) dp.part_order[k] = (uint8_t)parts[k].second;
  dp.n_full = dp.full0[dp.n_seqs];
  dp.n_part = (int)parts.size();
  dp.n_tail = dp.tail0[dp.n_seqs];
  dp.n_zero = nzero;
  *max_splits = most;
  return dp.n_full + (dp.n_part + dp.n_tail + dp.n_zero) * dp.Hkv;
}

// ---------------------------------------------------------------- launchers (host)
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
cudaError_t launch_block_table_update(int* table, int n, const int* idx_host, const int* val_host, cudaStream_t s);
int decode_blocks_per_sm(int G, size_t smem_bytes);
cudaError_t launch_decode(const DecodeParams& p, int grid_x, cudaStream_t s);
cudaError_t launch_project_query(const DecodeParams& p, cudaStream_t s);
// ---------------------------------------------------------------- VBR regrade
constexpr int MAX_REGRADE_SEQS = 128;
struct RegradeParams {
  const uint8_t* src_pool;       // the layer's page pool in its current layout
  uint32_t src_page_bytes;
  uint8_t* dst_pool;             // scratch: every page of the layer in the new layout
  uint32_t dst_page_bytes;
  const int* block_table;
  int max_pages_per_seq;
  int Hkv, rot;
  int bf16;                      // F16-codec rows are bf16
  const float* inv_s;            // [Hkv][2][128] of this layer, or null
  int* err;
  int n_seqs;
  long total_rows;
  int seq[MAX_REGRADE_SEQS];
  long row0[MAX_REGRADE_SEQS + 1];   // prefix sums of the sequences' quantized rows
  HeadInfo src[MAX_HKV];
  HeadInfo dst[MAX_HKV];
};
cudaError_t launch_regrade(const RegradeParams& p, cudaStream_t s);

cudaError_t launch_dequantize(const DecodeParams& p, int seq, int64_t t0, int64_t t1, float* k_out, float* v_out,
                              cudaStream_t s);
cudaError_t launch_read_rows(const DecodeParams& p, int seq, int64_t t0, int64_t t1, int kv, uint8_t* codes,
                             uint8_t* scales, cudaStream_t s);
cudaError_t launch_project(const ProjParams& p, int n_items, int n_heads, cudaStream_t s);
cudaError_t launch_calibrate(int64_t n_tok, int n_ch, int64_t stride, const __half* x, float* inv, cudaStream_t s);
cudaError_t launch_debug_rotate(const HeadInfo& h, int rot, int kv, const float* inv_s, int n, const __half* x,
                                float* y, bool quad, bool bf16, cudaStream_t s);
cudaError_t launch_debug_quantize(int codec, int r, int b, int n, const float* y, uint8_t* codes, uint8_t* scales,
                                  bool quad, cudaStream_t s);
size_t decode_smem_bytes(int stage_bytes, int n_stages, int G, bool wtab_smem);
// Bytes of one consumer warp's softmax-weight table: 32 token-pair rows of
// [4 blocks][G] int16 pairs plus a pad word per block (the fp32 path's (w, w)
// pairs of 32 tokens take half of it).  It lives in the dead K-code region of the
// warp's current stage whenever that region is large enough.
__host__ __device__ constexpr uint32_t wtab_bytes(int G) { return 32u * (4u * (uint32_t)G + 4u) * 4u; }
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)16 << 20;   // = KVQ_NOALLOC_SCRATCH_BYTES
cudaError_t noalloc_scratch(int device, void** out);
void note_launches(int n);   // counts kernel launches made by the library
cudaError_t launch_microbench(int kind, int iters, const void* buf, size_t buf_bytes, unsigned long long* sink,
                              int ctas, cudaStream_t s, double* work);
int decode_max_smem();

// ---------------------------------------------------------------- prefill (tensor cores)
// Causal attention of the last n_q tokens of one sequence over one layer's cache:
// a CTA takes QB = 128 / G consecutive queries of one kv head (rows j*G + g), and
// every key/value tile of 64 positions is dequantized once per CTA into fp16
// operands for tcgen05.mma.  Layers whose heads all use block codecs (not F16,
// not the rank codec) and a rotation other than the projection take this path.
struct PrefillParams {
  const uint8_t* pool;           // the layer's page pool
  uint32_t page_bytes;
  const int* bt;                 // the sequence's block-table row
  const uint8_t* ring;           // tail ring of (sequence, layer, kv head 0); heads T*512 bytes apart
  int T;                         // tail length (ring slots)
  int nq_all;                    // quantized rows of the sequence (len - T, or 0)
  int len, n_q, Hq, Hkv, G, QB;
  int rot, bf16;
  const __half* q;               // [n_q][Hq][128] raw 16-bit
  float* out;                    // [n_q][Hq][128]
  const float* s_k;              // [Hkv][128] or null (variance normalisation)
  const float* s_v;
  const float* inv_s;            // [Hkv][2][128] or null: the append's multipliers (tail rows)
  float qscale;                  // softmax scale * log2(e)
  int stage_bytes;               // raw page-head stage (multiple of 128)
  int n_raw;                     // raw stages (2..4)
  int* err;
  unsigned long long wait_ns;
  HeadInfo heads[MAX_HKV];
};
size_t prefill_smem_bytes(int stage_bytes, int n_raw);
int prefill_raw_stages(int stage_bytes);     // stages that fit, 0 if fewer than two
cudaError_t launch_prefill(const PrefillParams& p, cudaStream_t s);

}  // namespace kvq
