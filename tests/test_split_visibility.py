"""Host-side checks of the decode kernel's index arithmetic, compiled with the host
compiler and run on the CPU: the split and causal-visibility arithmetic that
decode and chunked prefill share (split_counts / tail_visible in the library's
internal header), and the pair-table layout of the integer key scores
(pair_tables.h: tab_slot must invert tab_channels).

For every (len, tail T, visible length lim) the tiles the kernel visits and the
slots it keeps must cover exactly positions 0 .. lim-1: the quantized pages in
position order, then the tail ring, where position p lives in slot p % T.
"""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_kv_cache_15_b200", "csrc")
CUDA_INC = "/usr/local/cuda/include"

PROGRAM = r'''
#include <cstdio>
#include <vector>
#include "kvq_internal.h"
using namespace kvq;
int main() {
  long checked = 0;
  const int tails[] = {0, 16, 64, 256, 1024};
  for (int T : tails)
    for (int len = 0; len <= 1300; len += (len < 200 ? 1 : 37))
      for (int lim = 0; lim <= len; lim += (len < 200 ? 1 : 13)) {
        for (int pps : {1, 3, 8})
        for (int ppt : {1, 2, 5}) {
          const SplitCounts c = split_counts(len, T, pps, ppt, lim);
          const int nq_all = len > T ? len - T : 0;
          std::vector<int> seen(len > 0 ? len : 1, 0);
          // quantized pages: splits of pps pages, 64 rows each, first nq tokens
          if (c.qsplits * pps < c.nqp || (c.qsplits - 1) * pps >= c.nqp + (c.nqp == 0)) { printf("bad qsplits\n"); return 1; }
          for (int t = 0; t < c.nq; ++t) seen[t]++;
          // tail: ntp tiles of TAIL_TOK slots, slots < nt visited, then masked
          if (c.tsplits * ppt < c.ntp || (c.tsplits - 1) * ppt >= c.ntp + (c.ntp == 0)) { printf("bad tsplits\n"); return 1; }
          for (int s = 0; s < c.ntp * TAIL_TOK; ++s) {
            if (s >= c.nt) continue;
            if (!tail_visible(c, T, s)) continue;
            const int p = len <= T ? s : nq_all + ((s - nq_all) % T + T) % T;
            if (p < nq_all || p >= len) { printf("slot %d maps outside the tail\n", s); return 1; }
            seen[p]++;
          }
          for (int p = 0; p < len; ++p)
            if (seen[p] != (p < lim ? 1 : 0)) {
              printf("len %d T %d lim %d pps %d: position %d seen %d times\n", len, T, lim, pps, p, seen[p]);
              return 1;
            }
          ++checked;
        }
      }
  printf("ok %ld\n", checked);
  return 0;
}
'''


def test_visited_tiles_cover_exactly_the_visible_prefix(tmp_path):
    if not os.path.isdir(CUDA_INC):
        pytest.skip("CUDA headers not installed")
    src = tmp_path / "vis.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "vis"
    r = subprocess.run(["g++", "-O1", "-std=c++17", "-I", CSRC, "-I", CUDA_INC, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout[-500:]


TAB_PROGRAM = r'''
#include <cstdio>
#include <cuda_runtime.h>
#include "pair_tables.h"
using namespace kvq;
int main() {
  for (int type = 0; type < 4; ++type) {
    int seen[128] = {0};
    for (int w = 0; w < 64; ++w) {
      int c0, c1, w0, h0, w1, h1;
      tab_channels(type, w, c0, c1);
      tab_slot(type, c0, w0, h0);
      tab_slot(type, c1, w1, h1);
      if (w0 != w || h0 != 0 || w1 != w || h1 != 1) { printf("type %d word %d\\n", type, w); return 1; }
      seen[c0]++; seen[c1]++;
    }
    for (int c = 0; c < 128; ++c)
      if (seen[c] != 1) { printf("type %d channel %d seen %d times\\n", type, c, seen[c]); return 1; }
  }
  printf("ok\\n");
  return 0;
}
'''


def test_pair_table_slots_invert_the_channel_order(tmp_path):
    """The decode prologue writes each quantized query value straight to the word and
    half that tab_slot names; the score loop reads word w as the two channels
    tab_channels names.  Every channel must land in exactly one slot, and the slot
    must be the one the score loop reads it from, for every plane layout."""
    if not os.path.isdir(CUDA_INC):
        pytest.skip("CUDA headers not installed")
    src = tmp_path / "tab.cpp"
    src.write_text(TAB_PROGRAM)
    exe = tmp_path / "tab"
    r = subprocess.run(["g++", "-O1", "-std=c++17", "-I", CSRC, "-I", CUDA_INC, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout[-500:]


ORDER_PROGRAM = r'''
#include <cstdio>
#include <cstdlib>
#include <vector>
#include "kvq_internal.h"
using namespace kvq;
int main() {
  unsigned rng = 12345u;
  auto rnd = [&](int n) { rng = rng * 1103515245u + 12345u; return (int)((rng >> 8) % (unsigned)n); };
  long checked = 0;
  for (int trial = 0; trial < 400; ++trial) {
    static DecodeParams dp;
    dp.n_seqs = 1 + rnd(trial < 200 ? 8 : MAX_BATCH);
    dp.Hkv = 1 + rnd(trial < 100 ? 4 : 12);
    const int tails[] = {0, 64, 256, 1024};
    dp.T = tails[rnd(4)];
    const int base = 1 + rnd(40);
    for (int h = 0; h < dp.Hkv; ++h) dp.pps[h] = (uint16_t)(trial % 3 == 0 ? base : 1 + rnd(40));
    dp.pps_t = 1 + rnd(8);
    for (int i = 0; i < dp.n_seqs; ++i) {
      dp.len[i] = rnd(5) == 0 ? 0 : rnd(6000);
      dp.lim[i] = rnd(3) == 0 ? rnd(dp.len[i] + 1) : dp.len[i];
    }
    int most = 0;
    const int grid = build_decode_order(dp, &most);
    std::vector<std::vector<int>> seen(dp.n_seqs * dp.Hkv);
    int prev_kind = 0;
    for (int b = 0; b < grid; ++b) {
      const DecodeItem it = decode_item(dp, b);
      const int head = it.head;
      if (head < 0 || head >= dp.Hkv) { printf("head out of range\\n"); return 1; }
      if (it.si < 0 || it.si >= dp.n_seqs) { printf("entry out of range\\n"); return 1; }
      const SplitCounts c = split_counts(dp.len[it.si], dp.T, dp.pps[head], dp.pps_t, dp.lim[it.si]);
      const int S = c.qsplits + c.tsplits;
      if (it.kind == 3) {                       // no-op item: only for a head without a partial split
        if (b < dp.n_full || c.nqp % dp.pps[head] != 0) { printf("misplaced no-op item\\n"); return 1; }
        continue;
      }
      // kinds in order: quantized splits, tail splits, zero items
      if (it.kind < prev_kind) { printf("item kinds out of order\\n"); return 1; }
      prev_kind = it.kind;
      if (it.kind == 2) {
        if (S != 0) { printf("zero item for an entry with splits\\n"); return 1; }
        seen[it.si * dp.Hkv + head].push_back(-1);
        continue;
      }
      if (it.split < 0 || it.split >= S || (it.kind == 1) != (it.split >= c.qsplits)) {
        printf("bad split %d of %d (kind %d)\\n", it.split, S, it.kind); return 1;
      }
      // full splits first (every one of pps[head] pages), then the partial ones
      const bool full = it.kind == 0 && (it.split + 1) * dp.pps[head] <= c.nqp;
      if ((b < dp.n_full) != full) { printf("full/partial split misplaced\\n"); return 1; }
      seen[it.si * dp.Hkv + head].push_back(it.split);
    }
    for (int i = 0; i < dp.n_seqs; ++i)
      for (int h = 0; h < dp.Hkv; ++h) {
        const SplitCounts c = split_counts(dp.len[i], dp.T, dp.pps[h], dp.pps_t, dp.lim[i]);
        const int S = c.qsplits + c.tsplits;
        std::vector<int>& v = seen[i * dp.Hkv + h];
        std::sort(v.begin(), v.end());
        if (S == 0) { if (v.size() != 1 || v[0] != -1) { printf("empty entry not zeroed once\\n"); return 1; } continue; }
        if ((int)v.size() != S) { printf("entry %d head %d: %zu of %d splits\\n", i, h, v.size(), S); return 1; }
        for (int k = 0; k < S; ++k) if (v[k] != k) { printf("split %d missing\\n", k); return 1; }
        if (S > most) { printf("max splits wrong\\n"); return 1; }
        ++checked;
      }
  }
  printf("ok %ld\\n", checked);
  return 0;
}
'''


def test_cta_order_covers_every_split_once_longest_first(tmp_path):
    """The decode launch's 1-D grid (build_decode_order / decode_item) gives every
    (entry, kv head, split) exactly one CTA -- full quantized splits first, then the
    partial ones (no-op items only for heads without one), then the tail splits --
    and exactly one zero-writing CTA per (entry, kv head) with nothing to attend to,
    for random batches of lengths and per-head split sizes."""
    if not os.path.isdir(CUDA_INC):
        pytest.skip("CUDA headers not installed")
    src = tmp_path / "order.cpp"
    src.write_text(ORDER_PROGRAM)
    exe = tmp_path / "order"
    r = subprocess.run(["g++", "-O1", "-std=c++17", "-I", CSRC, "-I", CUDA_INC, str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout[-500:]
