// Pair tables of the decode kernel's integer key scores.
//
// Word w of a table packs two int16 query values (low half, high half) in the
// order that the code-plane masks of the score loop produce the codes, so that one
// dp2a multiplies two query values by two codes.  tab_channels gives the two
// channels of a word, tab_slot the word and half of a channel (its inverse); both
// are plain index arithmetic, shared with the host for the CPU check.
#pragma once

namespace kvq {

enum { TAB_NAT = 0, TAB_Q4 = 1, TAB_Q2 = 2, TAB_Q1 = 3 };
__host__ __device__ inline void tab_channels(int type, int w, int& c0, int& c1) {
  switch (type) {
    case TAB_NAT: c0 = 2 * w; c1 = c0 + 1; break;                              // bytes in order
    case TAB_Q4: {                                                              // masks 0x0F0F0F0F, >>4
      const int k = w >> 2, j = w & 3;
      c0 = 8 * k + ((j == 0) ? 0 : (j == 1) ? 4 : (j == 2) ? 1 : 5);
      c1 = c0 + 2;
    } break;
    case TAB_Q2: {                                                              // masks 0x03030303, >>2s
      const int k = w >> 3, j = w & 7, s = j >> 1;
      c0 = 16 * k + s + ((j & 1) ? 8 : 0);
      c1 = c0 + 4;
    } break;
    default: {                                                                  // masks 0x01010101, >>s
      const int k = w >> 4, j = w & 15, s = j >> 1;
      c0 = 32 * k + s + ((j & 1) ? 16 : 0);
      c1 = c0 + 8;
    } break;
  }
}

// Inverse of tab_channels: the word of the table and the half (0 low, 1 high) that
// hold query channel c.
__host__ __device__ inline void tab_slot(int type, int c, int& w, int& half) {
  switch (type) {
    case TAB_NAT: w = c >> 1; half = c & 1; break;
    case TAB_Q4: {
      const int k = c >> 3, o = c & 7;
      half = (o >> 1) & 1;                          // o in {2, 3, 6, 7}: c = c0 + 2
      const int o0 = half ? o - 2 : o;              // in {0, 4, 1, 5}
      w = 4 * k + ((o0 == 0) ? 0 : (o0 == 4) ? 1 : (o0 == 1) ? 2 : 3);
    } break;
    case TAB_Q2: {
      const int k = c >> 4, o = c & 15;
      half = (o >> 2) & 1;
      w = 8 * k + 2 * (o & 3) + ((o >> 3) & 1);
    } break;
    default: {
      const int k = c >> 5, o = c & 31;
      half = (o >> 3) & 1;
      w = 16 * k + 2 * (o & 7) + ((o >> 4) & 1);
    } break;
  }
}

// Pair-table layouts of a key codec with `bits` code bits (plane 0, plane 1; -1 = none).
__host__ __device__ inline void codec_tables(int bits, int* t0, int* t1) {
  switch (bits) {
    case 8: *t0 = TAB_NAT; *t1 = -1; break;
    case 6: *t0 = TAB_Q4; *t1 = TAB_Q2; break;
    case 5: *t0 = TAB_Q4; *t1 = TAB_Q1; break;
    case 4: *t0 = TAB_Q4; *t1 = -1; break;
    case 3: *t0 = TAB_Q2; *t1 = TAB_Q1; break;
    case 2: *t0 = TAB_Q2; *t1 = -1; break;
    case 1: *t0 = TAB_Q1; *t1 = -1; break;
    default: *t0 = -1; *t1 = -1; break;
  }
}

}  // namespace kvq
