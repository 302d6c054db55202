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
//   tie = (35 - top rank) * 6 + (5 - bottom class rank),
// where a bottom combo's class rank is its position, in rank order, among the
// bottom combos that need the same state (at most six).  Among patterns with equal
// sums the larger tie field is the smaller (top rank, bottom rank), i.e. the lower
// pattern index, and the field splits into a top part and a bottom part that ride
// on the combo sums.  decode maps a tie field back to the pattern index.
struct PackedTables {
  uint8_t ntop[kNumStates];      // top combos producing each state
  uint8_t top[kNumStates][6];    // their ranks, ascending
  uint8_t nbot[kNumStates];      // bottom combos needing each state
  uint8_t bot[kNumStates][6];    // their ranks, ascending
  uint8_t tie_top[36];           // (35 - rank) * 6
  uint8_t tie_bot[36];           // 5 - class rank
  uint8_t decode[256];           // tie field -> pattern index (kPadIndex where unused)
};

__host__ __device__ constexpr PackedTables make_packed_tables() {
  PackedTables t{};
  const PatternTables pt = make_pattern_tables();
  for (int s = 0; s < kNumStates; ++s) { t.ntop[s] = 0; t.nbot[s] = 0; }
  for (int c = 0; c < 36; ++c) {
    const int s = pt.top_state[c];
    t.top[s][t.ntop[s]++] = (uint8_t)c;
    t.tie_top[c] = (uint8_t)((35 - c) * 6);
  }
  for (int b = 0; b < 36; ++b) {
    const int s = pt.bot_state[b];
    t.tie_bot[b] = (uint8_t)(5 - t.nbot[s]);
    t.bot[s][t.nbot[s]++] = (uint8_t)b;
  }
  for (int i = 0; i < 256; ++i) t.decode[i] = kPadIndex;
  for (int s = 0; s < kNumStates; ++s)
    for (int i = 0; i < t.ntop[s]; ++i)
      for (int k = 0; k < t.nbot[s]; ++k) {
        const int c = t.top[s][i], b = t.bot[s][k];
        t.decode[t.tie_top[c] + t.tie_bot[b]] = pt.index[c * 36 + b];
      }
  return t;
}

}  // namespace sp24
