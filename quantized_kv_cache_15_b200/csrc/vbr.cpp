// VBR policy: which layer to requantize next.
//
// "Introducing a new KV format: VBR (Variable Bit Rate)": the cache starts F16 and
// is quantized layer by layer as the session grows (F16, then F16 / 8-bit mixes,
// and so on), so that it fits the VRAM given to it (--vbr-vram) without going
// below a quality floor (--vbr-floor).  The pages give no ladder or order; this
// library reads them as the VBR-mix workload's map does: rungs F16 > q8_0 > q6_0 >
// q4_1 > q2_1 with V on a rung and K one rung richer, and, while the bytes in use
// exceed the budget, the deepest layer on the richest rung moves down one rung.
#include "kvq_internal.h"

namespace {

const int kLadder[] = {KVQ_F16, KVQ_Q8_0, KVQ_Q6_0, KVQ_Q4_1, KVQ_Q2_1};
constexpr int kRungs = 5;

int rung_of(int codec) {
  for (int i = 0; i < kRungs; ++i)
    if (kLadder[i] == codec) return i;
  return -1;
}

}  // namespace

extern "C" kvq_status kvq_vbr_next(int n_layers, int n_kv_heads, const int* k_codec, const int* v_codec,
                                   int64_t bytes_in_use, int64_t budget, int floor_codec, int* layer,
                                   int* new_k_codec, int* new_v_codec) {
  if (n_layers <= 0 || n_kv_heads <= 0 || !k_codec || !v_codec || !layer || !new_k_codec || !new_v_codec)
    return KVQ_ERR_INVALID_ARG;
  const int floor_rung = rung_of(floor_codec);
  if (floor_rung < 0) return KVQ_ERR_UNSUPPORTED;
  *layer = -1;
  if (bytes_in_use <= budget) return KVQ_OK;
  // a layer's rung is its V codec's rung (every head of a layer moves together)
  int best = -1, best_rung = kRungs;
  for (int l = 0; l < n_layers; ++l) {
    const int r = rung_of(v_codec[(size_t)l * n_kv_heads]);
    if (r < 0) return KVQ_ERR_UNSUPPORTED;
    for (int h = 1; h < n_kv_heads; ++h)
      if (rung_of(v_codec[(size_t)l * n_kv_heads + h]) != r) return KVQ_ERR_UNSUPPORTED;
    if (r >= floor_rung) continue;                   // at (or below) the floor already
    if (r < best_rung || (r == best_rung && l > best)) { best = l; best_rung = r; }
  }
  if (best < 0) return KVQ_OK;                       // every layer sits at the floor
  const int nv = kLadder[best_rung + 1];
  const int nk = kLadder[best_rung];                 // K one rung richer than V
  for (int h = 0; h < n_kv_heads; ++h) {
    const int ok = k_codec[(size_t)best * n_kv_heads + h];
    // K never moves to a richer rung than it holds
    new_k_codec[h] = (rung_of(ok) >= 0 && rung_of(ok) > best_rung) ? ok : nk;
    new_v_codec[h] = nv;
  }
  *layer = best;
  return KVQ_OK;
}
