/*
 * kvq.h -- C ABI of the B200 quantized KV cache: append-quantize and decode
 * attention over packed q8/q6/q4/q3/q2 (_0 and _1), F16 and per-head rank/bit
 * codecs, with a Hadamard rotation (optionally variance-normalised, or fused
 * into a per-head projection), an F16 (or BF16) precision tail for the newest
 * tokens, a per-layer / per-head codec map, grouped-query decode attention and
 * chunked-prefill attention over the cache.
 *
 * Sources (web pages, cited by title and section):
 *  - "BeeLlama.cpp v0.4.0 发布：聚焦 KV cache 量化，新增 KVarN 与精度尾部机制":
 *    §核心新特性：KVarN (variance-normalised quantization), §KV cache 精度尾部
 *    (newest tokens kept in F16), §新增标准 KV cache 类型 (q6_0/q6_1,
 *    q3_0/q3_1, q2_0/q2_1 next to q8_0 and q5/q4).
 *  - "KV-COBRA splits the KV-cache budget per head -- Rank vs bit-width
 *    allocation": §Jargon (Hadamard rotation, scalar quantization to 2^b
 *    levels, rank / low-rank projection), §The news (per-head rank and bits,
 *    rotation fused into the projection matrix, frozen per-head settings at
 *    inference).
 *  - "Introducing a new KV format: VBR (Variable Bit Rate)": per-layer codec
 *    mixes and asymmetric K/V codecs.
 *  - Forum thread on KV compression (swe-vps, maurelius2): decode attention is
 *    a dot product of the query with every prior key, a softmax and a weighted
 *    average of the values; decode is bound by memory bandwidth.
 *
 * Conventions (every entry point):
 *  - Pointers marked "device" are CUDA device pointers on the plan's device;
 *    pointers marked "host" are ordinary host memory read before the call
 *    returns.  The caller owns every buffer it passes (cache, inputs, outputs,
 *    workspace).  A plan owns only its own copies of the host tables it was
 *    given (small device allocations) and host bookkeeping.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued asynchronously on it; argument errors are reported synchronously,
 *    before anything is enqueued, and leave the plan unchanged.
 *  - A call that enqueues work on a plan (append, decode, prefill, dequantize,
 *    row reads, regrade, the debug transforms) needs the plan's device (the one
 *    current at kvq_plan_create) to be current: otherwise it returns
 *    KVQ_ERR_STATE and enqueues nothing.
 *  - Errors never throw across the ABI.  Every call returns a kvq_status;
 *    kvq_last_error() gives a thread-local message for the last failure.
 *    Conditions that only a kernel can see (a missing page, an exhausted wait)
 *    are latched in the plan's device error word and reported by
 *    kvq_check_device_error().
 *  - head_dim is 128.  Positions, lengths and capacities count tokens.
 *  - A plan is not thread-safe; calls on one plan must be serialised.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_HEAD_DIM 128
#define KVQ_PAGE_TOKENS 64      /* tokens per cache page */
#define KVQ_MAX_KV_HEADS 32
#define KVQ_MAX_GQA 8           /* query heads per kv head */
#define KVQ_MAX_BATCH 256       /* sequences per decode / append call */

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size, layer or sequence out of range */
  KVQ_ERR_UNSUPPORTED = 2,   /* codec, rank/bits, head_dim or GQA ratio this build does not handle */
  KVQ_ERR_CAPACITY = 3,      /* sequence longer than max_tokens_per_seq, or the page pool is exhausted */
  KVQ_ERR_OOM = 4,           /* a plan-owned device allocation failed */
  KVQ_ERR_CUDA = 5,          /* a CUDA runtime call or a launch failed */
  KVQ_ERR_DEVICE = 6,        /* a kernel latched an error (see kvq_check_device_error) */
  KVQ_ERR_TIMEOUT = 7,       /* a bounded wait inside a kernel ran out */
  KVQ_ERR_STATE = 8          /* call out of order (e.g. no cache bound) */
} kvq_status;

/* Codecs.  Block = 32 consecutive values of a row in the stored basis.
 *  _0 (symmetric): d = max|x| / (2^(b-1) - 1) stored fp16 (round to nearest
 *     even); codes round-half-even(x / d) clamped to [-2^(b-1), 2^(b-1) - 1]
 *     (the tiny workload's q4_0: d = max|x|/7, codes in [-8, 7]).
 *  _1 (scale + minimum): m = fp16 round-down of the block minimum,
 *     d = (max - m) / (2^b - 1) fp16; codes round-half-even((x - m)/d) in
 *     [0, 2^b - 1].
 *  KVQ_RANK: the KV-COBRA per-head path: the row is projected to r
 *     coordinates (rotation fused into the projection) and each block of
 *     min(32, r) coordinates is quantized mid-rise with all 2^b levels
 *     (levels (k + 1/2) d, d = max|z| / (2^(b-1) - 1/2)); r and b per head.
 *  KVQ_F16: raw fp16 rows (unrotated).
 * Codes are stored offset-binary (u = code + 2^(b-1) for _0).  A canonical
 * packed row (what kvq_read_rows returns) is the code planes, then the block
 * scales.  Planes hold b-bit fields, lowest field in the lowest bits of each
 * byte, in value order; 6 bits = 4-bit plane then 2-bit plane, 5 bits = 4-bit
 * plane then 1-bit plane, 3 bits = 2-bit plane then 1-bit plane (a value's low
 * bits in the first plane).  Scales: fp16 d per block (_0, KVQ_RANK), or fp16
 * (d, m) pairs per block (_1).  Row bytes for 128 values: 16 b of codes plus 8
 * (_0) or 16 (_1) of scales; F16 rows are the 256 bytes of raw values.  In the
 * cache, a page's K code rows are interleaved in 16-byte chunks across its 64
 * token rows and every other plane is row-major. */
typedef enum {
  KVQ_F16 = 0, KVQ_Q8_0 = 1, KVQ_Q6_0 = 2, KVQ_Q4_0 = 3, KVQ_Q3_0 = 4, KVQ_Q2_0 = 5,
  KVQ_Q8_1 = 6, KVQ_Q6_1 = 7, KVQ_Q4_1 = 8, KVQ_Q3_1 = 9, KVQ_Q2_1 = 10, KVQ_RANK = 11,
  KVQ_Q5_0 = 12, KVQ_Q5_1 = 13
} kvq_codec;

/* Transform applied to rows before quantization (F16 rows are never
 * transformed).  HADAMARD: y = H x / sqrt(128) (Sylvester H, computed as the
 * staged fast transform in fp32).  VARNORM_HADAMARD: y = H (x * inv_rms) /
 * sqrt(128) with a per-(layer, kv-head, K|V, channel) inverse RMS from a
 * calibration prefix (KVarN).  PROJECTION: z = M_h x with M_h = R_r P_h^T,
 * P_h the head's 128 x r orthonormal basis and R_r the order-r rotation
 * (codec must be KVQ_RANK or KVQ_F16). */
typedef enum {
  KVQ_ROT_NONE = 0, KVQ_ROT_HADAMARD = 1, KVQ_ROT_VARNORM_HADAMARD = 2, KVQ_ROT_PROJECTION = 3
} kvq_rot;

/* Dtype of the plan's raw 16-bit rows: the appended K/V rows (k_new, v_new), the
 * decode queries q, the precision tail and the pages of the KVQ_F16 codec
 * [BeeLlama v0.4.0 news, §KV cache 精度尾部: the newest tokens are kept in BF16 or
 * F16].  KVQ_KV_BF16 plans take bf16 rows throughout (exactly widened to fp32 before
 * the transform and the quantizer) and keep a bf16 tail; they support neither
 * KVQ_ROT_PROJECTION nor KVQ_F16 pages (KVQ_ERR_UNSUPPORTED at plan creation or
 * regrade).  kvq_calibrate_varnorm always reads fp16 rows. */
typedef enum { KVQ_KV_F16 = 0, KVQ_KV_BF16 = 1 } kvq_kv_dtype;

typedef struct kvq_plan kvq_plan;

typedef struct {
  int n_layers;                 /* >= 1 */
  int n_q_heads;                /* query heads per layer */
  int n_kv_heads;               /* kv heads per layer (<= KVQ_MAX_KV_HEADS); n_q_heads / n_kv_heads <= KVQ_MAX_GQA */
  int head_dim;                 /* must be 128 */
  int max_seqs;                 /* sequence ids are 0 .. max_seqs-1 */
  int64_t max_tokens_per_seq;   /* capacity of one sequence (every layer) */
  int64_t max_pages;            /* pages in the pool (each page: 64 tokens x all kv heads of a layer, in
                                   every layer); 0 = max_seqs * ceil(max_tokens_per_seq / 64) */
  int tail_tokens;              /* precision tail length per (seq, layer, kv-head), raw rows in kv_dtype;
                                   0 or a multiple of 64 */
  const int* k_codec;           /* host [n_layers][n_kv_heads] kvq_codec of K */
  const int* v_codec;           /* host [n_layers][n_kv_heads] kvq_codec of V */
  int rot;                      /* kvq_rot */
  const float* inv_rms;         /* host [n_layers][n_kv_heads][2 (K,V)][128], VARNORM_HADAMARD only, else NULL */
  const int* rank;              /* host [n_layers][n_kv_heads] r in {16,32,64,96,128}, PROJECTION only */
  const int* k_bits;            /* host [n_layers][n_kv_heads] b in {1,2,3,4} for K, PROJECTION only */
  const int* v_bits;            /* host [n_layers][n_kv_heads] b in {1,2,3,4} for V, PROJECTION only */
  const double* proj_basis;     /* host, PROJECTION only: for each (layer, head) in order, P_h as a
                                   row-major [128][r] matrix with orthonormal columns; concatenated */
  float softmax_scale;          /* 0 => 1/sqrt(128) */
  int kv_dtype;                 /* kvq_kv_dtype of the raw 16-bit rows; 0 = KVQ_KV_F16 */
} kvq_plan_desc;

/* Create a plan on the current CUDA device: validates the descriptor, lays out
 * the paged cache, copies the host tables (and fuses the rotation into the
 * projections: M_h = R_r P_h^T) into plan-owned device memory.
 * [KV-COBRA explainer, §The news: frozen per-head settings, rotation fused]. */
kvq_status kvq_plan_create(const kvq_plan_desc* desc, kvq_plan** out);
void kvq_plan_destroy(kvq_plan* plan);

/* Bytes of device memory the caller must allocate for the cache. */
kvq_status kvq_plan_cache_bytes(const kvq_plan* plan, size_t* bytes);

/* Bytes of device workspace kvq_decode_attention needs for n_seqs sequences.
 * The workspace must be zero-filled once before its first use; every call
 * leaves its counters back at zero, and a workspace sized for n sequences serves
 * every later call (decode or prefill) with at most n entries. */
kvq_status kvq_plan_workspace_bytes(const kvq_plan* plan, int n_seqs, size_t* bytes);

/* Attach caller-owned device memory of at least kvq_plan_cache_bytes(), 256-byte
 * aligned.  Its contents need not be initialised.  Resets every sequence. */
kvq_status kvq_cache_bind(kvq_plan* plan, void* dev_cache, size_t bytes);

/* Append n_new[i] new tokens to sequence seq_ids[i] in one layer
 * [BeeLlama v0.4.0 news §KV cache 精度尾部 and §KVarN; KV-COBRA §The news].
 *  k_new, v_new: device fp16 (bf16 for KVQ_KV_BF16 plans)
 *  [sum(n_new)][n_kv_heads][128], the sequences' rows concatenated in call order.
 * New rows enter the layer's F16 tail; rows pushed out of the tail (or every
 * row, when tail_tokens = 0) are transformed and quantized into the paged
 * cache.  seq_ids must be distinct.  Lengths advance at enqueue time (per
 * sequence and layer).  KVQ_ERR_CAPACITY if a sequence would exceed
 * max_tokens_per_seq or the page pool runs out (nothing is enqueued then). */
kvq_status kvq_append_quantize(kvq_plan* plan, int layer, int n_seqs, const int* seq_ids /*host*/,
                               const int* n_new /*host*/, const void* k_new, const void* v_new, void* stream);

/* Decode attention for one new query token per sequence
 * [forum thread on KV compression: dot, softmax, weighted average of values].
 *  q:   device fp16 (bf16 for KVQ_KV_BF16 plans) [n_seqs][n_q_heads][128]
 *  out: device fp32 [n_seqs][n_q_heads][128]
 *  workspace: device, kvq_plan_workspace_bytes(plan, n_seqs), zeroed before first use;
 *    may be NULL when no sequence needs more than one split and the plan has no
 *    projection (KVQ_ROT_PROJECTION plans keep their projected queries there).
 * Query head h attends with kv head h / (n_q_heads / n_kv_heads) over every
 * cached token of the sequence in this layer (quantized rows dequantized in
 * registers, tail rows in F16).  Split-K over pages; partial softmax states
 * are merged in a fixed order (deterministic). */
kvq_status kvq_decode_attention(kvq_plan* plan, int layer, int n_seqs, const int* seq_ids /*host*/,
                                const void* q, float* out, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Chunked-prefill attention over the quantized cache [forum thread on KV
 * compression: dot, softmax, weighted average; BeeLlama v0.4.0 news §KV cache
 * 精度尾部 for the tail]: the last n_q tokens of sequence seq_id in this layer,
 * already appended, attend causally to the cache, so query i (position
 * len - n_q + i) sees positions 0 .. len - n_q + i, quantized rows dequantized in
 * registers and tail rows raw, with the same GQA grouping as decode.
 *  q:   device raw dtype [n_q][n_q_heads][128];  out: device fp32 [n_q][n_q_heads][128]
 *  workspace: kvq_plan_workspace_bytes(plan, min(n_q, KVQ_MAX_BATCH)), zeroed before
 *    first use (the calls leave it ready for reuse).
 * Layers whose heads all use block codecs (no F16 pages, no rank codec) under a
 * rotation other than the projection run on the tensor cores: a CTA takes
 * 128 / G consecutive queries of one kv head and dequantizes each 64-token
 * key/value tile once for all of them (keys and the query as fp16 hi + lo pairs,
 * values and softmax weights as fp16, fp32 accumulation; q and out 16-byte
 * aligned; the workspace is not used).  Other layers run each query through the
 * split-K decode kernel over its visible prefix, KVQ_MAX_BATCH queries per launch.
 * KVQ_ERR_INVALID_ARG if n_q exceeds the length. */
kvq_status kvq_prefill_attention(kvq_plan* plan, int layer, int seq_id, int n_q, const void* q, float* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Decode attention without any allocation, for callers that cannot allocate
 * device memory (no counterpart in the pages: this is a deployment variant of
 * kvq_decode_attention).  Some callers cannot supply a workspace: runtimes
 * without an allocator, hosts whose memory pool owns every byte of device
 * memory and cannot lend a slice to a library, and loops that must never call
 * cudaMalloc because it can synchronise the device.  This entry point computes
 * exactly what kvq_decode_attention computes, with the same arguments except the
 * workspace: its split-K scratch is a fixed device array of
 * KVQ_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.
 *  - Calls needing more scratch than that (kvq_plan_workspace_bytes(plan, n_seqs)
 *    above the limit) return KVQ_ERR_CAPACITY before enqueueing anything.
 *  - The first call on a device looks the array's device address up (with that
 *    device current); make that first call before any stream capture.
 *  - The entry point allocates nothing (no cudaMalloc/cudaFree, no allocating
 *    library routine); it zeroes the array's merge counters with an async
 *    memset on `stream` at every call.
 *  - Every call shares the one array: calls that may overlap on the GPU (other
 *    streams, other threads, other plans on the same device) race and must be
 *    serialised by the caller. */
#define KVQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
kvq_status kvq_decode_attention_noalloc(kvq_plan* plan, int layer, int n_seqs, const int* seq_ids /*host*/,
                                        const void* q, float* out, void* stream);

/* VBR regrade ["Introducing a new KV format: VBR (Variable Bit Rate)", first post:
 * the cache is quantized layer by layer as the session grows, within a VRAM
 * budget and above a quality floor].  Requantize every cached row of one layer
 * below the F16 tail, for every sequence, to new per-kv-head codecs:
 *  k_codec, v_codec: host [n_kv_heads]; block codecs (q8_0 .. q5_1) or F16 where
 *    the head's rows are F16 already.  Rows are brought to the stored basis
 *    (F16 rows through the layer's variance normalisation and Hadamard rotation,
 *    block rows dequantized exactly) and quantized with the new codec; the tail
 *    stays raw.  Later appends and decodes of the layer use the new codecs.
 *  scratch: device, kvq_plan_regrade_bytes() bytes, 16-byte aligned: the layer's
 *    pages are written there in the new layout and then copied over the layer's
 *    pool on `stream`.
 * KVQ_ERR_UNSUPPORTED for projection plans, rank targets, or a quantized row
 * regraded to F16; KVQ_ERR_CAPACITY if the new pages would be larger than the
 * layer's current pages (a regrade only moves to poorer codecs overall). */
kvq_status kvq_plan_regrade_bytes(const kvq_plan* plan, int layer, const int* k_codec /*host*/,
                                  const int* v_codec /*host*/, size_t* bytes);
kvq_status kvq_regrade_layer(kvq_plan* plan, int layer, const int* k_codec /*host*/, const int* v_codec /*host*/,
                             void* scratch, size_t scratch_bytes, void* stream);

/* VBR policy step (host only) ["Introducing a new KV format: VBR (Variable Bit
 * Rate)": quantize layer by layer as the session grows, within --vbr-vram and
 * above --vbr-floor].  The pages fix no ladder or order; this reading uses the
 * rungs F16 > q8_0 > q6_0 > q4_1 > q2_1 with V on a rung and K one rung richer.
 * If bytes_in_use > budget, *layer is the deepest layer on the richest rung above
 * floor_codec (a rung of the ladder) and new_k_codec / new_v_codec (host
 * [n_kv_heads]) its codecs one rung down; else, or when every layer sits at the
 * floor, *layer = -1.  k_codec, v_codec: host [n_layers][n_kv_heads], every head
 * of a layer on the same V rung.  KVQ_ERR_UNSUPPORTED for codecs off the ladder. */
kvq_status kvq_vbr_next(int n_layers, int n_kv_heads, const int* k_codec, const int* v_codec, int64_t bytes_in_use,
                        int64_t budget, int floor_codec, int* layer, int* new_k_codec, int* new_v_codec);

/* Device bytes the plan's cache uses now: every layer's pages held by sequences at
 * the layer's current page size, plus the F16 tail rings. */
kvq_status kvq_plan_bytes_in_use(const kvq_plan* plan, int64_t* bytes);

/* Reconstruct cached rows t0 .. t1-1 of one sequence and layer in the ORIGINAL
 * basis (inverse rotation / projection applied; tail rows copied).
 *  k_out, v_out: device fp32 [t1-t0][n_kv_heads][128] (either may be NULL). */
kvq_status kvq_dequantize(const kvq_plan* plan, int layer, int seq_id, int64_t t0, int64_t t1,
                          float* k_out, float* v_out, void* stream);

/* Packed row sizes of one (layer, kv head, K=0|V=1): code bytes and scale bytes
 * of one canonical row (F16: 256 and 0). */
kvq_status kvq_row_bytes(const kvq_plan* plan, int layer, int head, int kv, int* code_bytes,
                         int* scale_bytes);

/* Copy quantized rows t0 .. t1-1 (all below the tail) of one sequence, layer and
 * K|V out of the paged cache into canonical packed rows, head after head:
 * head h's rows start at sum_{h'<h} (t1-t0) * code_bytes(h') in codes_out and
 * likewise in scales_out.  Device buffers. */
kvq_status kvq_read_rows(const kvq_plan* plan, int layer, int seq_id, int64_t t0, int64_t t1, int kv,
                         void* codes_out, void* scales_out, void* stream);

/* Host mirror of a sequence's length in one layer. */
kvq_status kvq_seq_length(const kvq_plan* plan, int seq_id, int layer, int64_t* len);

/* Forget a sequence (all layers) and return its pages to the pool. */
kvq_status kvq_seq_reset(kvq_plan* plan, int seq_id);

/* Per-channel inverse RMS of a calibration prefix [BeeLlama v0.4.0 news
 * §KVarN: variance normalisation]: inv_rms[c] = fp32(1 / sqrt(mean_t x[t][c]^2))
 * with the sum taken in double in token order (1 where the RMS is < 1e-6).
 *  x: device fp16 [n_tokens][row_stride] (channels 0 .. n_channels-1 used)
 *  inv_rms: device fp32 [n_channels] */
kvq_status kvq_calibrate_varnorm(int64_t n_tokens, int n_channels, int64_t row_stride, const void* x,
                                 float* inv_rms, void* stream);

/* KV-COBRA rank/bit allocation, run once at calibration [KV-COBRA explainer,
 * §The news: steps C1 and C2; §Where the bits actually go].  For each head the
 * error of keeping rank r at b bits is the variance of the dropped directions
 * plus eps[b-1] times the variance of the kept ones (eps: relative rounding
 * noise of the b-bit rank quantizer, b = 1..4, measured by the caller).  Every
 * head starts at (16, 1); the budget of round(bpd * 128 * n_heads) bits is then
 * handed out one upgrade at a time to the head whose affordable upgrade removes
 * the most error per extra bit (ties: lower head index, then fewer bits).
 *  lambdas: host [n_heads][128] direction variances, each row non-increasing.
 *  ranks, bits: host [n_heads] outputs (r in {16,32,64,96,128}, b in 1..4).
 *  bits_used: host, may be NULL.  Host-only: touches no device.
 * KVQ_ERR_CAPACITY if the budget is below 16 bits per head. */
kvq_status kvq_cobra_allocate(int n_heads, const double* lambdas, double bpd, const double* eps, int* ranks,
                              int* bits, int* bits_used);

/* Synchronise `stream`, read and clear the plan's device error word. */
kvq_status kvq_check_device_error(kvq_plan* plan, void* stream);

/* Thread-local description of the last failure ("" if none). */
const char* kvq_last_error(void);

/* Total number of CUDA kernels this library has launched in the process
 * (every entry point that enqueues work adds its launches). */
kvq_status kvq_launch_count(uint64_t* count);

/* --- inspection entry points (used by the parity tests) ------------------ */

/* Row layouts of the append and regrade kernels (the inspection entry points
 * below run either): KVQ_ROWS_WARP one warp per row (4 values per lane; small
 * appends, the projection path), KVQ_ROWS_QUAD four threads per row (one
 * 32-value block each; chunk appends, regrade).  Both must produce the same
 * bytes. */
enum kvq_row_layout { KVQ_ROWS_WARP = 0, KVQ_ROWS_QUAD = 1 };

/* Rows in the stored basis, fp32, exactly as the append path computes them
 * before quantization: the staged Hadamard transform (after variance
 * normalisation) for rotated codecs, z = M_h x for the projection path (the
 * exact products summed over the channels in order in double, rounded once to
 * fp32), the raw values for F16.
 *  x: device raw rows in the plan's kv dtype [n][128];  y: device fp32 [n][128] (or [n][r]).
 *  layout: kvq_row_layout (ignored for the projection path). */
kvq_status kvq_debug_rotate(const kvq_plan* plan, int layer, int head, int kv, int n, const void* x,
                            float* y, int layout, void* stream);

/* The block quantizer alone: fp32 rows in the stored basis -> canonical packed
 * rows.  codec: kvq_codec; r, b: rank and bits (KVQ_RANK only, else ignored).
 *  y: device fp32 [n_rows][128 or r]; codes: device [n_rows][code_bytes];
 *  scales: device [n_rows][scale_bytes].
 *  layout: kvq_row_layout (KVQ_RANK: KVQ_ROWS_WARP only, else
 *  KVQ_ERR_UNSUPPORTED). */
kvq_status kvq_debug_quantize_f32(int codec, int r, int b, int n_rows, const float* y, void* codes,
                                  void* scales, int layout, void* stream);

/* Micro-benchmarks of the CUDA-core issue pipes and of a streaming read (no
 * counterpart in the pages: they measure the ceilings that decode attention on
 * CUDA cores runs against).  One bounded launch of `ctas` CTAs of 256 threads on
 * `stream`; the caller times it (events on the same stream) and divides *work by
 * the time.
 *  kind: KVQ_UB_FFMA (fp32 fma, work = multiply-adds), KVQ_UB_DP2A (dp2a: 2 per
 *    instruction), KVQ_UB_DP4A (dp4a: 4), KVQ_UB_FMA2 (fma.rn.f32x2: 2), KVQ_UB_MIX
 *    (dp2a and fp32 fma one to one: 3 per pair), each thread running `iters`
 *    rounds of 8 independent chains; KVQ_UB_READ: `iters` passes of 16-byte
 *    streaming loads over buf (work = bytes read).
 *  buf: device, 16-byte aligned, buf_bytes >= 16 (KVQ_UB_READ only; else ignored).
 *  sink: device [ctas * 256] 64-bit words, written (keeps the work alive).
 *  work: host, the launch's work count.
 * KVQ_ERR_INVALID_ARG for a bad kind, iters outside [1, 2^20], ctas outside
 * [1, 65536], or missing buffers; nothing is enqueued then. */
enum kvq_microbench_kind {
  KVQ_UB_FFMA = 0, KVQ_UB_DP2A = 1, KVQ_UB_DP4A = 2, KVQ_UB_FMA2 = 3, KVQ_UB_MIX = 4, KVQ_UB_READ = 5
};
kvq_status kvq_microbench(int kind, int iters, int ctas, const void* buf, size_t buf_bytes, void* sink,
                          double* work, void* stream);

/* Fixed split-K size for this plan's decode and prefill calls (test-only; no
 * counterpart in the pages): pages_per_split > 0 cuts every sequence into splits of
 * that many pages (at least as many as the split limit needs); 0 restores the
 * automatic choice.  The merge order is fixed either way, so results differ only
 * by the rounding of the merge.  KVQ_ERR_INVALID_ARG for a negative count. */
kvq_status kvq_debug_set_decode_split(kvq_plan* plan, int pages_per_split);

/* Prefill path selection (test-only; no counterpart in the pages): path 0 (the
 * default) uses the tensor-core prefill wherever the layer allows it, path 1
 * always runs the decode kernel per query.  KVQ_ERR_INVALID_ARG for other values. */
kvq_status kvq_debug_set_prefill_path(kvq_plan* plan, int path);

/* Failure injection for the failure-path tests (test-only; no counterpart in the
 * pages).  wait_limit_ns: every bounded wait inside this plan's decode kernels
 * gives up after this long (default 2e9; accepted range [1e3, 2e9]) and latches
 * KVQ_ERR_TIMEOUT in the plan's error word.  drop_last_tile = 1 makes every decode
 * CTA's producer skip loading its last tile, so the consumer waiting for it runs
 * out its wait, finishes the launch on stale shared memory (the output of that
 * call is garbage) and the next kvq_check_device_error() returns KVQ_ERR_TIMEOUT;
 * the context stays usable.  No bulk copy is left in flight: the skipped tile is
 * the last use of its stage.  (2e9, 0) restores normal operation. */
kvq_status kvq_debug_fault_injection(kvq_plan* plan, int64_t wait_limit_ns, int drop_last_tile);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H_ */
