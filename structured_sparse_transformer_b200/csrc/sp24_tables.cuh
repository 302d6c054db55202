// Pattern tables of the transposable 2:4 mask search, generated at compile time.
//
// "Accelerating Transformer Pre-training with 2:4 Sparsity", reproducibility
// table, Pseudocode row, Algorithm 1: the filter set m of the stride-4
// convolution is every 4x4 0/1 pattern with two ones in each row and column.
// Index order: lexicographic on the per-row column pairs, pair ranks
// (0,1)<(0,2)<(0,3)<(1,2)<(1,3)<(2,3), row 0 most significant.
//
// The search kernel does not loop over the 90 patterns.  It splits a pattern
// into a "top" half (rows 0-1, a choice of two column pairs, 36 combos) and a
// "bottom" half (rows 2-3, 36 combos).  A top and a bottom combo form a pattern
// iff their column counts add up to (2,2,2,2); the top combo's count vector is
// its "state" (19 of them).  The tables below give, per combo, the state it
// produces (top) or needs (bottom), and the pattern index of every compatible
// (top, bottom) pair.  Since pattern order is (top rank, bottom rank) order,
// the lowest-index optimum is the lexicographically smallest (top, bottom).
#pragma once
#include <stdint.h>

namespace sp24 {

constexpr int kNumPatterns = 90;
constexpr int kNumStates = 19;
constexpr uint8_t kPadIndex = 255;  // marks blocks outside the matrix in shared tiles

// Column pair of pair rank q.
__host__ __device__ constexpr int pair_lo(int q) { return q < 3 ? 0 : (q < 5 ? 1 : 2); }
__host__ __device__ constexpr int pair_hi(int q) {
  return q == 0 ? 1 : (q == 1 ? 2 : (q == 2 ? 3 : (q == 3 ? 2 : 3)));
}
// 2-bit position code of a kept pair (lo, hi): lo | hi << 2.
__host__ __device__ constexpr int pair_code(int q) { return pair_lo(q) | (pair_hi(q) << 2); }

struct PatternTables {
  uint16_t bits[256];      // bit 4*i+j: row i, column j kept (pad entries: 0)
  uint16_t rowcode[256];   // nibble i: code of row i's kept column pair (pad: 0x4444)
  uint16_t colcode[256];   // nibble j: code of column j's kept row pair (pad: 0x4444)
  uint8_t top_state[36];   // state produced by top combo 6*q0 + q1
  uint8_t bot_state[36];   // state a bottom combo 6*q2 + q3 needs from the top
  uint8_t index[36 * 36];  // pattern index of (top, bottom), or kPadIndex
  int count;
};

__host__ __device__ constexpr int counts_code(int q0, int q1) {
  int c[4] = {0, 0, 0, 0};
  c[pair_lo(q0)] += 1; c[pair_hi(q0)] += 1;
  c[pair_lo(q1)] += 1; c[pair_hi(q1)] += 1;
  return c[0] + 3 * c[1] + 9 * c[2] + 27 * c[3];
}

__host__ __device__ constexpr int complement_code(int code) {
  int out = 0, scale = 1;
  for (int j = 0; j < 4; ++j) { out += (2 - code % 3) * scale; code /= 3; scale *= 3; }
  return out;
}

__host__ __device__ constexpr PatternTables make_pattern_tables() {
  PatternTables t{};
  int state_code[kNumStates] = {};
  int nstates = 0;
  for (int tc = 0; tc < 36; ++tc) {
    int code = counts_code(tc / 6, tc % 6);
    int s = -1;
    for (int k = 0; k < nstates; ++k) if (state_code[k] == code) s = k;
    if (s < 0) { s = nstates; state_code[nstates++] = code; }
    t.top_state[tc] = (uint8_t)s;
  }
  for (int bc = 0; bc < 36; ++bc) {
    int need = complement_code(counts_code(bc / 6, bc % 6));
    int s = 0;
    for (int k = 0; k < nstates; ++k) if (state_code[k] == need) s = k;
    t.bot_state[bc] = (uint8_t)s;
  }
  for (int i = 0; i < 256; ++i) { t.bits[i] = 0; t.rowcode[i] = 0x4444; t.colcode[i] = 0x4444; }
  int n = 0;
  for (int tc = 0; tc < 36; ++tc)
    for (int bc = 0; bc < 36; ++bc) {
      t.index[tc * 36 + bc] = kPadIndex;
      if (t.top_state[tc] != t.bot_state[bc]) continue;
      int q[4] = {tc / 6, tc % 6, bc / 6, bc % 6};
      uint16_t bits = 0, rc = 0;
      for (int i = 0; i < 4; ++i) {
        bits |= (uint16_t)((1u << (4 * i + pair_lo(q[i]))) | (1u << (4 * i + pair_hi(q[i]))));
        rc |= (uint16_t)(pair_code(q[i]) << (4 * i));
      }
      uint16_t cc = 0;
      for (int j = 0; j < 4; ++j) {
        int lo = -1, hi = -1;
        for (int i = 0; i < 4; ++i)
          if (bits >> (4 * i + j) & 1u) { if (lo < 0) lo = i; else hi = i; }
        cc |= (uint16_t)((lo | (hi << 2)) << (4 * j));
      }
      t.bits[n] = bits;
      t.rowcode[n] = rc;
      t.colcode[n] = cc;
      t.index[tc * 36 + bc] = (uint8_t)n;
      ++n;
    }
  t.count = n;
  return t;
}

#ifdef __CUDACC__
// The pattern tables in global memory: threads index them with per-thread
// pattern numbers, which the L1 cache serves without the serialisation that
// divergent reads of __constant__ memory would take, and without a per-CTA copy.
__device__ const PatternTables g_tables = make_pattern_tables();
#endif

// Tables of the packed-key search (mask_kernels.cuh, search_block_packed).
// A pattern's key is (exact sum of its |w|) << 8 plus an 8-bit tie field
//   tie = (35 - top rank) * 6 + (5 - q2),
// q2 the pair rank of row 2.  Within one column-count state the bottom combos
// that fit have distinct q2, in the order of their rank, so among patterns with
// equal sums the larger tie field is the smaller (top rank, bottom rank), i.e.
// the lower pattern index.  The field is linear in the row pair ranks,
//   tie = 36 (5 - q0) + 6 (5 - q1) + (5 - q2),
// so each row's share rides on that row's pair sums (pair_tie).  decode maps a
// tie field back to the pattern index.
struct PackedTables {
  uint8_t ntop[kNumStates];      // top combos producing each state
  uint8_t top[kNumStates][6];    // their ranks, ascending
  uint8_t nbot[kNumStates];      // bottom combos needing each state
  uint8_t bot[kNumStates][6];    // their ranks, ascending
  uint8_t decode[256];           // tie field -> pattern index (kPadIndex where unused)
};

// Row i's share of the tie field for pair rank q.
__host__ __device__ constexpr uint32_t pair_tie(int i, int q) {
  return i == 0 ? 36u * (5 - q) : (i == 1 ? 6u * (5 - q) : (i == 2 ? (uint32_t)(5 - q) : 0u));
}

__host__ __device__ constexpr PackedTables make_packed_tables() {
  PackedTables t{};
  const PatternTables pt = make_pattern_tables();
  for (int s = 0; s < kNumStates; ++s) { t.ntop[s] = 0; t.nbot[s] = 0; }
  for (int c = 0; c < 36; ++c) {
    const int s = pt.top_state[c];
    t.top[s][t.ntop[s]++] = (uint8_t)c;
  }
  for (int b = 0; b < 36; ++b) {
    const int s = pt.bot_state[b];
    t.bot[s][t.nbot[s]++] = (uint8_t)b;
  }
  for (int i = 0; i < 256; ++i) t.decode[i] = kPadIndex;
  for (int s = 0; s < kNumStates; ++s)
    for (int i = 0; i < t.ntop[s]; ++i)
      for (int k = 0; k < t.nbot[s]; ++k) {
        const int c = t.top[s][i], b = t.bot[s][k];
        const uint32_t tie = pair_tie(0, c / 6) + pair_tie(1, c % 6) + pair_tie(2, b / 6) + pair_tie(3, b % 6);
        t.decode[tie] = pt.index[c * 36 + b];
      }
  return t;
}

// Byte selectors of the compression (prmt): for pattern p and row i, the
// selector that picks the row's two kept 16-bit values, in column order, from
// the row's four values held as two words (columns 0-1, 2-3); for column j, the
// selector that picks the column's two kept values, in row order, from the
// column's four values held as two words (rows 0-1, 2-3).  Four 16-bit
// selectors per pattern and orientation, row (column) i at bits 16 i.
struct SelectTables {
  uint64_t row[256];
  uint64_t col[256];
};

__host__ __device__ constexpr uint64_t pair_selector(int lo, int hi) {
  return (uint64_t)((2 * lo) | ((2 * lo + 1) << 4) | ((2 * hi) << 8) | ((2 * hi + 1) << 12));
}

__host__ __device__ constexpr SelectTables make_select_tables() {
  SelectTables t{};
  const PatternTables pt = make_pattern_tables();
  for (int p = 0; p < 256; ++p) {
    t.row[p] = 0;
    t.col[p] = 0;
    for (int i = 0; i < 4; ++i) {
      const int rc = (pt.rowcode[p] >> (4 * i)) & 0xF, cc = (pt.colcode[p] >> (4 * i)) & 0xF;
      t.row[p] |= pair_selector(rc & 3, rc >> 2) << (16 * i);
      t.col[p] |= pair_selector(cc & 3, cc >> 2) << (16 * i);
    }
  }
  return t;
}

}  // namespace sp24
