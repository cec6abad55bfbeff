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
