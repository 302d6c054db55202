// Bandwidth-bound kernels of the mask path: transposable 2:4 mask search,
// prune + compress into the tensor-core layout, flip count, masked decay.
//
// "Accelerating Transformer Pre-training with 2:4 Sparsity":
//   - reproducibility table, Pseudocode row, Algorithm 1 (mask search: |W|
//     convolved at stride 4 with the candidate patterns, argmax per block);
//   - reproducibility table, Software Dependencies row (transposable mask
//     search, pruning and masked decay kernels);
//   - abstract (flip rate; masked decay term on gradients).
//
// Mask search is exact.  The fast path sums magnitudes in fp64, which holds
// every pattern sum of a fp16 block exactly, and of a bf16 block whose nonzero
// magnitudes span at most 42 binades (search_block_fast).  The remaining bf16
// blocks take an integer search: each |w| becomes an integer multiple of the
// smallest subnormal relative to the block's largest exponent (32 binades
// deep), pre-shifted left by 12 bits; the 12 low bits of a pattern's key hold
// (35 - top rank) << 6 | (35 - bottom rank), so one unsigned 64-bit max picks
// the largest exact sum and, among equal sums, the lowest pattern index.
// Both take the max over the 90 patterns by a dynamic program over
// column-count states (top rows 0-1 and bottom rows 2-3, see sp24_tables.cuh)
// instead of enumerating all 90.  bf16 blocks whose nonzero magnitudes span
// more than 32 binades take an exact multi-word brute force.
#pragma once
#include "sp24_common.cuh"
#include "sp24_tables.cuh"

namespace sp24 {

using u64 = unsigned long long;

__device__ __forceinline__ u64 umax64(u64 a, u64 b) { return a > b ? a : b; }

// Exact-key dynamic program.  v[4*i+j] = |w(i,j)| in fixed point << 12.
// Returns (35 - top rank) << 6 | (35 - bottom rank) of the winning pattern.
__device__ __forceinline__ uint32_t dp_argmax_ranks(const u64 (&v)[16]) {
  constexpr PatternTables T = make_pattern_tables();
  u64 P[4][6];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < 6; ++q) P[i][q] = v[4 * i + pair_lo(q)] + v[4 * i + pair_hi(q)];
  u64 top[kNumStates], bot[kNumStates];
#pragma unroll
  for (int s = 0; s < kNumStates; ++s) { top[s] = 0; bot[s] = 0; }
#pragma unroll
  for (int c = 0; c < 36; ++c) {
    const u64 kt = P[0][c / 6] + P[1][c % 6] + ((u64)(35 - c) << 6);
    top[T.top_state[c]] = umax64(top[T.top_state[c]], kt);
    const u64 kb = P[2][c / 6] + P[3][c % 6] + (u64)(35 - c);
    bot[T.bot_state[c]] = umax64(bot[T.bot_state[c]], kb);
  }
  u64 best = 0;
#pragma unroll
  for (int s = 0; s < kNumStates; ++s) best = umax64(best, top[s] + bot[s]);
  return (uint32_t)(best & 0xFFFu);
}

// Exact brute force over the 90 patterns with 5-limb integer sums (each
// |w| = sig * 2^ep units of 2^-133).  Only reached by bf16 blocks whose
// magnitudes span more than 32 binades.  Takes the block's raw words by value
// so the fast path keeps everything in registers.
__device__ __noinline__ uint32_t exact_search_wide_bf16(uint32_t w00, uint32_t w01, uint32_t w10, uint32_t w11,
                                                        uint32_t w20, uint32_t w21, uint32_t w30, uint32_t w31,
                                                        const uint16_t *bits_tab) {
  const uint32_t words[8] = {w00, w01, w10, w11, w20, w21, w30, w31};
  u64 best[5] = {0, 0, 0, 0, 0};
  uint32_t best_p = 0;
  for (int p = 0; p < kNumPatterns; ++p) {
    u64 acc[5] = {0, 0, 0, 0, 0};
    const uint32_t bits = bits_tab[p];
    for (int c = 0; c < 16; ++c) {
      if (!((bits >> c) & 1u)) continue;
      const uint32_t a = (words[c >> 1] >> ((c & 1) << 4)) & 0x7FFFu;
      const uint32_t e = a >> 7;
      const uint32_t sig = e ? ((a & 0x7Fu) | 0x80u) : a;
      const uint32_t ep = e ? e - 1 : 0;
      if (sig == 0) continue;
      const int limb = (int)(ep >> 6), off = (int)(ep & 63);
      const u64 lo = (u64)sig << off;
      const u64 hi = off ? ((u64)sig >> (64 - off)) : 0ull;
      u64 carry = 0;
      for (int k = limb; k < 5; ++k) {
        const u64 add = (k == limb) ? lo : ((k == limb + 1) ? hi : 0ull);
        const u64 s1 = acc[k] + add;
        const u64 c1 = s1 < add;
        const u64 s2 = s1 + carry;
        const u64 c2 = s2 < carry;
        acc[k] = s2;
        carry = c1 + c2;
      }
    }
    bool greater = false;
    for (int k = 4; k >= 0; --k) {
      if (acc[k] != best[k]) { greater = acc[k] > best[k]; break; }
    }
    if (p == 0 || greater) {
      for (int k = 0; k < 5; ++k) best[k] = acc[k];
      best_p = (uint32_t)p;
    }
  }
  return best_p;
}

// Dynamic program over column-count states on magnitudes v[4*i+j] = |w(i,j)|
// in a type whose sums here are exact.  One state at a time, so only the pair
// sums and the running best stay live: the state's best top and bottom combos
// (the lowest rank among equal sums), then the pattern total against the best
// so far (a larger total wins; an equal total keeps the smaller
// (top rank, bottom rank) key).  Returns top rank << 6 | bottom rank.
template <typename Real>
__device__ __forceinline__ uint32_t dp_state_key(const Real (&v)[16]) {
  constexpr PatternTables T = make_pattern_tables();
  Real P[4][6];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < 6; ++q) P[i][q] = v[4 * i + pair_lo(q)] + v[4 * i + pair_hi(q)];
  Real best = (Real)-1;  // every total is >= 0, so the first state is taken
  uint32_t bkey = 0;
#pragma unroll
  for (int st = 0; st < kNumStates; ++st) {
    Real tv = 0, bv = 0;
    uint32_t tr = 0, br = 0;
    bool tseen = false, bseen = false;
#pragma unroll
    for (int c = 0; c < 36; ++c) {
      if (T.top_state[c] == st) {
        const Real k = P[0][c / 6] + P[1][c % 6];
        if (!tseen) { tv = k; tr = (uint32_t)c; tseen = true; }
        else { const bool gt = k > tv; tv = gt ? k : tv; tr = gt ? (uint32_t)c : tr; }
      }
      if (T.bot_state[c] == st) {
        const Real k = P[2][c / 6] + P[3][c % 6];
        if (!bseen) { bv = k; br = (uint32_t)c; bseen = true; }
        else { const bool gt = k > bv; bv = gt ? k : bv; br = gt ? (uint32_t)c : br; }
      }
    }
    const Real tot = tv + bv;
    const uint32_t key = (tr << 6) | br;
    const bool take = tot > best || (tot == best && key < bkey);
    best = take ? tot : best;
    bkey = take ? key : bkey;
  }
  return bkey;
}

// Pattern index of one 4x4 block given as 4 rows x 2 words (two 16-bit values each).
template <bool BF16>
__device__ __noinline__ uint32_t search_block(const uint32_t (&w)[4][2], const uint8_t *index_tab,
                                                 const uint16_t *bits_tab) {
  u64 v[16];
  if (!BF16) {
    // fp16: |w| = sig * 2^ep units of 2^-24 is below 2^41; a sum of eight is
    // below 2^44 and exact in fp64.
    double d[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint32_t a = (w[c >> 2][(c >> 1) & 1] >> ((c & 1) << 4)) & 0x7FFFu;
      const uint32_t e = a >> 10;
      const uint32_t sig = e ? ((a & 0x3FFu) | 0x400u) : a;
      const uint32_t ep = e ? e - 1 : 0;
      d[c] = __ull2double_rn((u64)sig << ep);
    }
    const uint32_t key = dp_state_key<double>(d);
    return index_tab[(key >> 6) * 36 + (key & 63)];
  } else {
    uint32_t sig[16], ep[16];
    uint32_t emax = 0;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint32_t a = (w[c >> 2][(c >> 1) & 1] >> ((c & 1) << 4)) & 0x7FFFu;
      const uint32_t e = a >> 7;
      sig[c] = e ? ((a & 0x7Fu) | 0x80u) : a;
      ep[c] = e ? e - 1 : 0;
      emax = max(emax, ep[c]);
    }
    const uint32_t base = emax > 32 ? emax - 32 : 0;
    bool exact = true;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const bool lost = sig[c] != 0 && ep[c] < base;
      exact = exact && !lost;
      v[c] = lost ? 0ull : ((u64)sig[c] << (ep[c] - base + 12));
    }
    if (!exact)
      return exact_search_wide_bf16(w[0][0], w[0][1], w[1][0], w[1][1], w[2][0], w[2][1], w[3][0], w[3][1],
                                    bits_tab);
  }
  const uint32_t r = dp_argmax_ranks(v);
  return index_tab[(35 - (r >> 6)) * 36 + (35 - (r & 63))];
}

constexpr uint32_t kNeedsExact = 0xFFu;  // fast path could not certify its sums

__device__ const PackedTables g_packed = make_packed_tables();
__device__ const SelectTables g_select = make_select_tables();

// Packed-key search of one block, exact when the block's nonzero magnitudes span
// at most 10 binades (fp16) or 13 (bf16); otherwise returns kNeedsExact.
//   * |w| becomes the integer v = |w| / U on a per-block unit U: the largest
//     magnitude below 2^21 U (U = 2^-24 2^sh for fp16, 2^-133 2^sh for bf16),
//     which is exact when every nonzero |w| is a multiple of U, i.e. when its
//     exponent field is at least sh + 1 (checked on the raw bits with 16-bit
//     lane max/min; zeros pass).
//   * Pair sums on the FMA pipe: f = |w_a| / U + 2^23 and f + |w_b| / U are exact
//     fp32 integers (below 2^24), whose low 23 bits hold v_a and v_a + v_b; one
//     integer multiply-add turns the word into (v_a + v_b) << 8 plus the row's
//     tie share (the 2^23 offset leaves the word).
//   * A pattern's key is sum(v) << 8 plus the tie field of PackedTables, all
//     below 2^32 (a sum of eight is below 2^24), so one unsigned max picks the
//     largest exact sum and, among equal sums, the lowest pattern index.
//   * The max over the 90 patterns is the same dynamic program over column-count
//     states: per state, the best top and bottom combo, then the best total, each
//     step one add-then-max.
template <bool BF16>
__device__ __forceinline__ uint32_t search_block_packed(const uint32_t (&w)[4][2], const uint8_t *__restrict__ decode,
                                                        uint32_t one) {
  constexpr PackedTables PT = make_packed_tables();
  constexpr int kMant = BF16 ? 7 : 10;               // explicit significand bits
  uint32_t a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = w[k >> 1][k & 1] & 0x7FFF7FFFu;
  uint32_t mx = __vmaxu2(__vmaxu2(__vmaxu2(a[0], a[1]), __vmaxu2(a[2], a[3])),
                         __vmaxu2(__vmaxu2(a[4], a[5]), __vmaxu2(a[6], a[7])));
  uint32_t m1[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m1[k] = __vsub2(a[k], 0x00010001u);   // zeros wrap to 0xFFFF
  uint32_t mn = __vminu2(__vminu2(__vminu2(m1[0], m1[1]), __vminu2(m1[2], m1[3])),
                         __vminu2(__vminu2(m1[4], m1[5]), __vminu2(m1[6], m1[7])));
  mx = max(mx & 0xFFFFu, mx >> 16);
  mn = min(mn & 0xFFFFu, mn >> 16);
  const int emax = max((int)(mx >> kMant), 1);
  const int sh = max(emax - (BF16 ? 14 : 11), 0);
  const int E = (BF16 ? 133 : 24) - sh;              // U = 2^-E
  const bool exact = (sh == 0 || mn + 1u >= ((uint32_t)(sh + 1) << kMant)) && E <= 127;
  if (!exact) return kNeedsExact;
  const float scale = __uint_as_float((uint32_t)(E + 127) << 23);
  const uint32_t k256 = one << 8;
  uint32_t P[4][6];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float x[4];
#pragma unroll
    for (int hw = 0; hw < 2; ++hw) {
      const uint32_t m2 = a[2 * i + hw];
      if (BF16) {
        x[2 * hw] = __uint_as_float(imad(m2, one << 16, 0u));
        x[2 * hw + 1] = __uint_as_float(m2 & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&m2));
        x[2 * hw] = f.x;
        x[2 * hw + 1] = f.y;
      }
    }
    const float f0 = fmaf(x[0], scale, 8388608.0f), f1 = fmaf(x[1], scale, 8388608.0f);
    const float f2 = fmaf(x[2], scale, 8388608.0f);
    const float ps[6] = {fmaf(x[1], scale, f0), fmaf(x[2], scale, f0), fmaf(x[3], scale, f0),
                         fmaf(x[2], scale, f1), fmaf(x[3], scale, f1), fmaf(x[3], scale, f2)};
#pragma unroll
    for (int q = 0; q < 6; ++q) P[i][q] = imad(__float_as_uint(ps[q]), k256, pair_tie(i, q));
  }
  uint32_t best = 0;
#pragma unroll
  for (int st = 0; st < kNumStates; ++st) {
    uint32_t tb = 0, bb = 0;
#pragma unroll
    for (int i = 0; i < 6; ++i) {
      if (i < PT.ntop[st]) {
        const int c = PT.top[st][i];
        tb = __viaddmax_u32(P[0][c / 6], P[1][c % 6], tb);
      }
      if (i < PT.nbot[st]) {
        const int b = PT.bot[st][i];
        bb = __viaddmax_u32(P[2][b / 6], P[3][b % 6], bb);
      }
    }
    best = __viaddmax_u32(tb, bb, best);
  }
  return decode[best & 0xFFu];
}

// Physical word of (W column c_local, block row br_local) in the transposed
// values tile (64 columns x 16 words): the 16-byte chunk of four block rows
// is XOR-swizzled by c_local/8, the word inside it by c_local/32, so the
// staging stores of a warp spread over the banks.
__device__ __forceinline__ int vcol_word(int c_local, int br_local) {
  return c_local * 16 + ((((br_local >> 2) ^ (c_local >> 3)) & 3) << 2) +
         ((br_local & 3) ^ (((c_local >> 5) & 1) << 1));
}

// Loads one unit (4 rows x 8 columns = two blocks) of W; columns past C read as 0.
__device__ __forceinline__ void load_unit(const uint16_t *__restrict__ W, int64_t ldw, int64_t r0, int64_t c0,
                                          int64_t R, int64_t C, bool vec16, uint32_t (&w)[4][4]) {
  const bool row_ok = r0 < R;
  const bool ok0 = row_ok && c0 + 4 <= C;
  const bool ok1 = row_ok && c0 + 8 <= C;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i][0] = w[i][1] = w[i][2] = w[i][3] = 0;
    const uint16_t *src = W + (r0 + i) * ldw + c0;
    if (ok1 && vec16) {
      const uint4 q = __ldg(reinterpret_cast<const uint4 *>(src));
      w[i][0] = q.x; w[i][1] = q.y; w[i][2] = q.z; w[i][3] = q.w;
    } else if (ok1) {
      const uint2 q0 = __ldg(reinterpret_cast<const uint2 *>(src));
      const uint2 q1 = __ldg(reinterpret_cast<const uint2 *>(src + 4));
      w[i][0] = q0.x; w[i][1] = q0.y; w[i][2] = q1.x; w[i][3] = q1.y;
    } else if (ok0) {
      const uint2 q = __ldg(reinterpret_cast<const uint2 *>(src));
      w[i][0] = q.x; w[i][1] = q.y;
    }
  }
}

constexpr int kTile = 64;           // quadrant of a metadata chunk: 64 rows x 64 columns
constexpr int kTileBlocks = kTile / 4;
constexpr int kQuadThreads = 128;   // one unit (4 rows x 8 columns = two blocks) per thread
constexpr int kChunk = 2 * kTile;   // one tensor-core metadata chunk: 128 x 128
// A CTA tile is the two quadrants of one column half of a chunk: 128 rows x 64
// columns of W, 256 threads (two CTA tiles side by side make a chunk).
constexpr int kMaskThreads = 2 * kQuadThreads;
constexpr int kMaskCtaCols = kTile;
constexpr int kMaskTileBytes = kChunk * kTile * 2;   // 16 KB of W per CTA tile
#ifndef SP24_MASK_CTAS_PER_SM
#define SP24_MASK_CTAS_PER_SM 3
#endif
constexpr int kMaskCtasPerSm = SP24_MASK_CTAS_PER_SM;   // search and flip only
// With compression a thread keeps more state live: two CTAs of 128 registers per thread.
template <bool COMPRESS>
constexpr int mask_ctas_per_sm() { return COMPRESS ? 2 : kMaskCtasPerSm; }
constexpr uint64_t kMaskDrainBudget = 1ull << 26;

// Nibble (4 * shift) of each of the four 16-bit codes in v, packed 4 bits apart.
__device__ __forceinline__ uint32_t gather_nibbles(uint2 v, int shift) {
  const uint32_t lo = (v.x >> (4 * shift)) & 0x000F000Fu;   // codes 0, 1
  const uint32_t hi = (v.y >> (4 * shift)) & 0x000F000Fu;   // codes 2, 3
  return (lo & 0xFu) | ((lo >> 12) & 0xF0u) | ((hi & 0xFu) << 8) | ((hi >> 4) & 0xF000u);
}

// Shared memory of one CTA tile, and the pattern tables the CTA reads per block
// (copied from global memory once per CTA): pattern index p takes entry p & 127,
// so the padding index 255 lands on entry 127, which holds its padding codes.
constexpr int kTabEntries = 128;
template <bool SEARCH, bool COMPRESS>
struct MaskSmem {
  uint2 rowsel[COMPRESS ? kTabEntries : 1];   // byte selectors of the kept pairs, rows
  uint2 colsel[COMPRESS ? kTabEntries : 1];   // and columns
  uint32_t codes[COMPRESS ? kTabEntries : 1]; // row codes | column codes << 16
  uint16_t bits[kTabEntries];                 // kept-entry bit sets
  uint8_t decode[SEARCH ? 256 : 4];           // tie field -> pattern index
  uint8_t idx[2][kTileBlocks][kTileBlocks];
  __align__(8) uint16_t rc[COMPRESS ? 2 : 1][kTileBlocks][kTileBlocks];   // row codes, [br][bc]
  __align__(8) uint16_t cc[COMPRESS ? 2 : 1][kTileBlocks][kTileBlocks];   // column codes, [bc][br]
  __align__(16) uint32_t vcol[COMPRESS ? 2 : 1][COMPRESS ? kTile * 16 : 4];
  // Blocks of each warp that need the exact search (two per lane at most).
  uint16_t wq[SEARCH ? kMaskThreads / 32 : 1][SEARCH ? 64 : 2];
};

template <bool SEARCH, bool COMPRESS>
__device__ __forceinline__ void load_mask_tables(MaskSmem<SEARCH, COMPRESS> &sm) {
  for (int e = threadIdx.x; e < kTabEntries; e += blockDim.x) {
    const int pat = e == kTabEntries - 1 ? (int)kPadIndex : e;
    if (COMPRESS) {
      const uint64_t r = g_select.row[pat], c = g_select.col[pat];
      sm.rowsel[e] = make_uint2((uint32_t)r, (uint32_t)(r >> 32));
      sm.colsel[e] = make_uint2((uint32_t)c, (uint32_t)(c >> 32));
      sm.codes[e] = (uint32_t)g_tables.rowcode[pat] | ((uint32_t)g_tables.colcode[pat] << 16);
    }
    sm.bits[e] = g_tables.bits[pat];
  }
  if (SEARCH)
    for (int e = threadIdx.x; e < 256; e += blockDim.x) sm.decode[e] = g_packed.decode[e];
}

// Where a CTA tile's weights come from: straight from global memory (row pitch
// ldw), or from a 128 x 64 tile that the tensor memory accelerator placed in
// shared memory (zeros outside the matrix).  Coordinates are relative to the
// CTA tile's first row and column.
struct GlobalTileSrc {
  const uint16_t *__restrict__ w;   // W at the CTA tile's origin
  int64_t ldw;
  bool vec16;                       // rows 16-byte aligned: one 128-bit load per unit row
  __device__ __forceinline__ void unit(int r, int c, bool ok0, bool ok1, uint32_t (&v)[4][4]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0;
      const uint16_t *src = w + (r + i) * ldw + c;
      if (ok1 && vec16) {
        const uint4 q = __ldg(reinterpret_cast<const uint4 *>(src));
        v[i][0] = q.x; v[i][1] = q.y; v[i][2] = q.z; v[i][3] = q.w;
      } else if (ok1) {
        const uint2 q0 = __ldg(reinterpret_cast<const uint2 *>(src));
        const uint2 q1 = __ldg(reinterpret_cast<const uint2 *>(src + 4));
        v[i][0] = q0.x; v[i][1] = q0.y; v[i][2] = q1.x; v[i][3] = q1.y;
      } else if (ok0) {
        const uint2 q = __ldg(reinterpret_cast<const uint2 *>(src));
        v[i][0] = q.x; v[i][1] = q.y;
      }
    }
  }
  __device__ __forceinline__ void block(int r, int c, uint32_t (&v)[4][2]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint2 q = __ldg(reinterpret_cast<const uint2 *>(w + (r + i) * ldw + c));
      v[i][0] = q.x; v[i][1] = q.y;
    }
  }
};

struct SharedTileSrc {
  const uint16_t *s;   // [128 rows][64 columns]
  __device__ __forceinline__ void unit(int r, int c, bool, bool, uint32_t (&v)[4][4]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = *reinterpret_cast<const uint4 *>(s + (r + i) * kTile + c);
      v[i][0] = q.x; v[i][1] = q.y; v[i][2] = q.z; v[i][3] = q.w;
    }
  }
  __device__ __forceinline__ void block(int r, int c, uint32_t (&v)[4][2]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint2 q = *reinterpret_cast<const uint2 *>(s + (r + i) * kTile + c);
      v[i][0] = q.x; v[i][1] = q.y;
    }
  }
};

// One CTA tile: rows 128 cy .. +127, columns 128 cx + 64 kh .. +63 of W, the
// quadrants rh = 0, 1 of column half kh of metadata chunk (cy, cx).  Thread t
// of quadrant rh = t / 128 owns the unit at unit column t%8 and block row
// (t%128)/8.  Rows and columns past the matrix get the padding code in the
// metadata.
//   SEARCH:   compute the mask (else read it from idx)
//   COMPRESS: write the compressed orientations whose pointers are non-null
//             (values + tensor-core metadata)
//   FLIP:     add the number of mask bits that differ from idx_prev to `flips`
// Search: every block takes the packed-key search; blocks it cannot certify
// (magnitudes spread over more than 10 binades for fp16, 13 for bf16) are queued
// per warp and searched exactly by the lanes of their own warp, with no barrier
// across the CTA.  The body has one CTA barrier with COMPRESS (the compressed
// operands are staged across the CTA's threads) and none without; the caller
// separates consecutive tiles with one more.
template <bool BF16, bool SEARCH, bool COMPRESS, bool FLIP, typename Src>
__device__ __forceinline__ void mask_tile_body(const Src &src, int64_t R, int64_t C, uint32_t cy, uint32_t cx,
                                               int kh, uint32_t chunks_x, uint32_t chunks_y,
                                               uint8_t *__restrict__ idx, const uint8_t *__restrict__ idx_prev,
                                               unsigned &flips, uint16_t *__restrict__ vals_row,
                                               uint8_t *__restrict__ meta_row, uint16_t *__restrict__ vals_col,
                                               uint8_t *__restrict__ meta_col, MaskSmem<SEARCH, COMPRESS> &sm,
                                               uint32_t one, const uint8_t *s_prev = nullptr) {
  const int tid = threadIdx.x;
  const int rh = tid >> 7, lt = tid & (kQuadThreads - 1);

  const int64_t tile_r0 = (int64_t)cy * kChunk, tile_c0 = (int64_t)cx * kChunk + kTile * kh;
  const int64_t tile_r = tile_r0 + kTile * rh;
  const int64_t bcols = C >> 2;
  const int uc = lt & 7;
  const int br = lt >> 3;
  const int lr = kTile * rh + 4 * br, lc = 8 * uc;   // the unit, relative to the CTA tile
  const int64_t r0 = tile_r0 + lr;
  const int64_t c0 = tile_c0 + lc;
  const bool row_ok = r0 < R;
  const bool ok0 = row_ok && c0 + 4 <= C;
  const bool ok1 = row_ok && c0 + 8 <= C;
  const int64_t bidx0 = (r0 >> 2) * bcols + (c0 >> 2);

  uint32_t w[4][4];
  src.unit(lr, lc, ok0, ok1, w);
  uint32_t prev[2] = {0, 0}, given[2] = {kPadIndex, kPadIndex};
  if (FLIP) {
    if (s_prev) {   // the previous mask's tile, staged with W: [32 block rows][16 block columns]
      const int pr = (kTile / 4) * rh + br;
      if (ok0) prev[0] = s_prev[pr * (kTile / 4) + 2 * uc];
      if (ok1) prev[1] = s_prev[pr * (kTile / 4) + 2 * uc + 1];
    } else {
      if (ok0) prev[0] = idx_prev[bidx0];
      if (ok1) prev[1] = idx_prev[bidx0 + 1];
    }
  }
  if (!SEARCH) {
    if (ok0) given[0] = idx[bidx0];
    if (ok1) given[1] = idx[bidx0 + 1];
  }

  // Phase 1: search (SEARCH), or take the given mask (!SEARCH).
  uint32_t p[2];
  bool need[2] = {false, false};
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const bool ok = b ? ok1 : ok0;
    p[b] = given[b];
    if (SEARCH && ok) {
      uint32_t blk[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) { blk[i][0] = w[i][2 * b]; blk[i][1] = w[i][2 * b + 1]; }
      p[b] = search_block_packed<BF16>(blk, sm.decode, one);
      need[b] = p[b] == kNeedsExact;
    }
  }

  // Phase 1b: the blocks that need the exact search, searched by the lanes of
  // their own warp (entry k of the warp's queue by lane k mod 32), with no
  // barrier across the CTA.  The queue lists them by lane, block 0 before 1.
  if (SEARCH) {
    const unsigned n0 = __ballot_sync(0xFFFFFFFFu, need[0]), n1 = __ballot_sync(0xFFFFFFFFu, need[1]);
    if (n0 | n1) {
      const int lane = tid & 31, wid = tid >> 5;
      const unsigned below = (1u << lane) - 1u;
      int pos = __popc(n0 & below) + __popc(n1 & below);
#pragma unroll
      for (int b = 0; b < 2; ++b)
        if (need[b]) sm.wq[wid][pos++] = (uint16_t)((rh << 8) | (br << 4) | (2 * uc + b));
      const int wn = __popc(n0) + __popc(n1);
      __syncwarp();
      for (int k = lane; k < wn; k += 32) {
        const int id = sm.wq[wid][k];
        const int q = id >> 8, qbr = (id >> 4) & 15, qbc = id & 15;
        uint32_t blk[4][2];
        src.block(kTile * q + 4 * qbr, 4 * qbc, blk);
        sm.idx[q][qbr][qbc] = (uint8_t)search_block<BF16>(blk, g_tables.index, g_tables.bits);
      }
      __syncwarp();
#pragma unroll
      for (int b = 0; b < 2; ++b)
        if (need[b]) p[b] = sm.idx[rh][br][2 * uc + b];
    }
  }

  // Phase 2: outputs of this thread's two blocks.  The unit is read again
  // rather than kept live across the exact search's call.
  if (SEARCH && COMPRESS) src.unit(lr, lc, ok0, ok1, w);
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const bool ok = b ? ok1 : ok0;
    if (SEARCH && ok) idx[bidx0 + b] = (uint8_t)p[b];
    if (FLIP && ok) flips += __popc((uint32_t)(sm.bits[prev[b] & 127] ^ sm.bits[p[b] & 127]));
  }
  if (COMPRESS) {
    uint32_t rc[2], cc[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const uint32_t codes = sm.codes[p[b] & 127];
      rc[b] = codes & 0xFFFFu;
      cc[b] = codes >> 16;
      sm.rc[rh][br][2 * uc + b] = (uint16_t)rc[b];
      sm.cc[rh][2 * uc + b][br] = (uint16_t)cc[b];
    }
    if (ok0) {
      // Forward operand: kept values of each row, in column order (one byte
      // permutation of the row's four values per row and block).
      if (vals_row) {
        uint2 rsel[2];
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          rsel[b] = sm.rowsel[p[b] & 127];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t packed[2];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint32_t sel = (i < 2 ? rsel[b].x : rsel[b].y) >> (16 * (i & 1));
            packed[b] = __byte_perm(w[i][2 * b], w[i][2 * b + 1], sel);
          }
          uint16_t *dst = vals_row + (r0 + i) * (C >> 1) + (c0 >> 1);
          if (ok1) *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[1]);
          else *reinterpret_cast<uint32_t *>(dst) = packed[0];
        }
      }
      // Input-gradient operand: kept values of each column, staged transposed.
      // Column j's four values as two words (rows 0-1, rows 2-3), then one byte
      // permutation picks its kept pair.
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint2 csel = sm.colsel[p[b] & 127];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int wi = 2 * b + (j >> 1);
          const uint32_t half = (j & 1) ? 0x7632u : 0x5410u;
          const uint32_t c01 = __byte_perm(w[0][wi], w[1][wi], half);
          const uint32_t c23 = __byte_perm(w[2][wi], w[3][wi], half);
          const uint32_t sel = (j < 2 ? csel.x : csel.y) >> (16 * (j & 1));
          sm.vcol[rh][vcol_word(8 * uc + 4 * b + j, br)] = __byte_perm(c01, c23, sel);
        }
      }
    }
  }
  if (COMPRESS) __syncthreads();

  if (COMPRESS) {
    // Transposed values: W column c (a row of W^T) holds 32 kept values per quadrant.
    const int64_t half_rows = R >> 1;
#pragma unroll
    for (int k = 0; k < (kTile * 4) / kQuadThreads; ++k) {
      const int id = lt + kQuadThreads * k;
      const int c_local = id >> 2, q = id & 3;
      if (vals_col && tile_c0 + c_local < C && tile_r + 16 * q + 16 <= R) {
        const uint4 v =
            *reinterpret_cast<const uint4 *>(&sm.vcol[rh][c_local * 16 + (((q ^ (c_local >> 3)) & 3) << 2)]);
        const bool swap = (c_local >> 5) & 1;
        const uint4 o = swap ? make_uint4(v.z, v.w, v.x, v.y) : v;
        *reinterpret_cast<uint4 *>(vals_col + (tile_c0 + c_local) * half_rows + (tile_r >> 1) + 8 * q) = o;
      }
    }
    // Metadata: one 2048-byte chunk per 128x128 region and orientation.  Lane L,
    // word kk (one 32-column K step of the MMA) holds rows m and m+8,
    // m = (L%8) + 16*(L/16), groups 4*((L/8)%2) .. +3 of that K step; the
    // low 16 bits are row m, the high 16 bits row m+8, one nibble per group.
    // Quadrant (rh, kh) fills lanes 64*rh.., words 2*kh.. of the chunk of the
    // rows of W, and lanes 64*kh.., words 2*rh.. of the chunk of its columns.
    // Thread t builds word t%2 of lane t/2 of the quadrant on each side.
    const int lq = lt >> 1, kx = lt & 1;
    const int m_lo = (lq & 7) + ((lq >> 4) << 4);   // row of the quadrant (0..55)
    const int gq = kx * 8 + ((lq >> 3) & 1) * 4;     // first of four groups, in blocks of the quadrant
    const int shift = m_lo & 3;
    if (meta_row) {
      const uint2 a = *reinterpret_cast<const uint2 *>(&sm.rc[rh][m_lo >> 2][gq]);
      const uint2 c = *reinterpret_cast<const uint2 *>(&sm.rc[rh][(m_lo >> 2) + 2][gq]);
      const uint32_t word = gather_nibbles(a, shift) | (gather_nibbles(c, shift) << 16);
      const size_t chunk = (size_t)cy * chunks_x + cx;
      *reinterpret_cast<uint32_t *>(meta_row + chunk * 2048 + (64 * rh + lq) * 16 + 4 * (2 * kh + kx)) = word;
    }
    if (meta_col) {
      const uint2 a = *reinterpret_cast<const uint2 *>(&sm.cc[rh][m_lo >> 2][gq]);
      const uint2 c = *reinterpret_cast<const uint2 *>(&sm.cc[rh][(m_lo >> 2) + 2][gq]);
      const uint32_t word = gather_nibbles(a, shift) | (gather_nibbles(c, shift) << 16);
      const size_t chunk = (size_t)cx * chunks_y + cy;
      *reinterpret_cast<uint32_t *>(meta_col + chunk * 2048 + (64 * kh + lq) * 16 + 4 * (2 * rh + kx)) = word;
    }
  }
}

// Adds the CTA's flip count to *flip_count (one global atomic per CTA).
__device__ __forceinline__ void mask_flip_flush(unsigned flips, unsigned long long *s_flip,
                                                unsigned long long *__restrict__ flip_count) {
  const unsigned warp_sum = __reduce_add_sync(0xFFFFFFFFu, flips);
  if ((threadIdx.x & 31) == 0 && warp_sum) atomicAdd(s_flip, (unsigned long long)warp_sum);
  __syncthreads();
  if (threadIdx.x == 0 && *s_flip) atomicAdd(flip_count, *s_flip);
}

// One CTA per CTA tile, W read from global memory: the kernel for row pitches
// that the tensor memory accelerator cannot take (ldw not a multiple of 8).
template <bool BF16, bool SEARCH, bool COMPRESS, bool FLIP>
__global__ void __launch_bounds__(kMaskThreads, mask_ctas_per_sm<COMPRESS>()) mask_tile_kernel(
    const uint16_t *__restrict__ W, int64_t R, int64_t C, int64_t ldw, uint8_t *__restrict__ idx,
    const uint8_t *__restrict__ idx_prev, unsigned long long *__restrict__ flip_count,
    uint16_t *__restrict__ vals_row, uint8_t *__restrict__ meta_row, uint16_t *__restrict__ vals_col,
    uint8_t *__restrict__ meta_col) {
  __shared__ MaskSmem<SEARCH, COMPRESS> sm;
  __shared__ unsigned long long s_flip;
  if (threadIdx.x == 0) s_flip = 0;
  load_mask_tables(sm);
  const uint32_t one = *reinterpret_cast<volatile const uint32_t *>(&g_one);
  pdl_launch_dependents();
  pdl_wait();
  const uint32_t cy = blockIdx.y, cx = blockIdx.x >> 1, chunks_x = gridDim.x >> 1;
  const int kh = (int)(blockIdx.x & 1);
  const GlobalTileSrc src{W + (int64_t)cy * kChunk * ldw + (int64_t)cx * kChunk + kTile * kh, ldw, (ldw & 7) == 0};
  __syncthreads();
  unsigned flips = 0;
  mask_tile_body<BF16, SEARCH, COMPRESS, FLIP>(src, R, C, cy, cx, kh, chunks_x, gridDim.y, idx, idx_prev, flips,
                                               vals_row, meta_row, vals_col, meta_col, sm, one);
  if (FLIP) mask_flip_flush(flips, &s_flip, flip_count);
}

// Persistent form: CTA b takes CTA tiles b, b + gridDim.x, ... (column halves
// fastest, then chunks along a row of chunks, then down the rows), with two
// 16 KB shared buffers of W: the tensor memory accelerator loads tile i + 2
// into a buffer as soon as the CTA has finished reading tile i from it, so the
// loads of the next two tiles overlap the work on this one.  Every wait is
// bounded; on a timeout the CTA records the error, lets its copies land and exits.
// One CTA barrier per tile (two with compression): each thread waits for its
// tile's copy itself, and the decision to stop is taken after the end-of-tile
// barrier on a flag of that tile's parity, so a thread already waiting on the
// next tile cannot change the flag the others are about to read.  A tile whose
// wait ran out is computed on whatever the buffer holds; its outputs are void
// (the device status reports the timeout), and every index stays in bounds.
template <bool BF16, bool SEARCH, bool COMPRESS, bool FLIP>
__global__ void __launch_bounds__(kMaskThreads, mask_ctas_per_sm<COMPRESS>()) mask_stream_kernel(
    const __grid_constant__ CUtensorMap tm_w, int64_t R, int64_t C, uint8_t *__restrict__ idx,
    const uint8_t *__restrict__ idx_prev, unsigned long long *__restrict__ flip_count,
    uint16_t *__restrict__ vals_row, uint8_t *__restrict__ meta_row, uint16_t *__restrict__ vals_col,
    uint8_t *__restrict__ meta_col, uint64_t wait_budget, const __grid_constant__ CUtensorMap tm_prev,
    int prev_tma) {
  __shared__ __align__(128) uint16_t s_w[2][kChunk * kTile];
  // FLIP with prev_tma: the previous mask's bytes of each tile arrive with it.
  __shared__ __align__(128) uint8_t s_prev[2][(kChunk / 4) * (kTile / 4)];
  __shared__ MaskSmem<SEARCH, COMPRESS> sm;
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ unsigned long long s_flip;
  __shared__ volatile int s_abort[2];   // per tile parity
  const int tid = threadIdx.x;
  const uint32_t chunks_x = (uint32_t)((C + kChunk - 1) / kChunk);
  const uint32_t chunks_y = (uint32_t)((R + kChunk - 1) / kChunk);
  const int64_t ntiles = 2ll * chunks_x * chunks_y;
  auto tile_xy = [&](int64_t t, uint32_t &cy, uint32_t &cx, int &kh) {
    kh = (int)(t & 1);
    cx = (uint32_t)((t >> 1) % chunks_x);
    cy = (uint32_t)((t >> 1) / chunks_x);
  };
  auto issue = [&](int64_t t, int buf) {
    uint32_t cy, cx;
    int kh;
    tile_xy(t, cy, cx, kh);
    const bool with_prev = FLIP && prev_tma;
    mbar_arrive_expect_tx(&s_full[buf], kMaskTileBytes + (with_prev ? (uint32_t)sizeof(s_prev[0]) : 0u));
    tma_load_2d(s_w[buf], &tm_w, &s_full[buf], (int)(cx * kChunk + kTile * kh), (int)(cy * kChunk));
    if (with_prev)
      tma_load_2d(s_prev[buf], &tm_prev, &s_full[buf], (int)((cx * kChunk + kTile * kh) / 4), (int)(cy * (kChunk / 4)));
  };
  if (tid == 0) {
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    fence_mbarrier_init();
    prefetch_tensormap(&tm_w);
    if (FLIP && prev_tma) prefetch_tensormap(&tm_prev);
    s_flip = 0;
    s_abort[0] = 0;
    s_abort[1] = 0;
  }
  load_mask_tables(sm);
  const uint32_t one = *reinterpret_cast<volatile const uint32_t *>(&g_one);
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();
  int64_t issued = 0, it = 0;   // copies issued (by thread 0) and tiles consumed
  if (tid == 0) {
    for (int k = 0; k < 2; ++k)
      if ((int64_t)blockIdx.x + (int64_t)k * gridDim.x < ntiles) {
        issue((int64_t)blockIdx.x + (int64_t)k * gridDim.x, k);
        ++issued;
      }
  }
  unsigned flips = 0;
  bool aborted = false;
  for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
    const int buf = (int)(it & 1);
    mbar_wait_bounded(&s_full[buf], (uint32_t)((it >> 1) & 1), wait_budget, &s_abort[buf]);
    uint32_t cy, cx;
    int kh;
    tile_xy(t, cy, cx, kh);
    const SharedTileSrc src{s_w[buf]};
    mask_tile_body<BF16, SEARCH, COMPRESS, FLIP>(src, R, C, cy, cx, kh, chunks_x, chunks_y, idx, idx_prev, flips,
                                                 vals_row, meta_row, vals_col, meta_col, sm, one,
                                                 (FLIP && prev_tma) ? s_prev[buf] : nullptr);
    __syncthreads();   // every read of this buffer and of the tile's shared state is done
    if (s_abort[buf]) {
      aborted = true;
      break;
    }
    if (tid == 0) {
      const int64_t nt = t + 2ll * gridDim.x;
      if (nt < ntiles) {
        issue(nt, buf);
        ++issued;
      }
    }
  }
  if (FLIP) mask_flip_flush(flips, &s_flip, flip_count);
  // After an abort, let the copies still in flight land before the CTA exits.
  if (tid == 0 && aborted) {
    for (int64_t k = it; k < issued; ++k) {
      volatile int no_abort = 0;
      mbar_wait_bounded(&s_full[k & 1], (uint32_t)((k >> 1) & 1), kMaskDrainBudget, &no_abort);
    }
  }
}

// Flip count between two masks: popcount of the XOR of their pattern bits.
__global__ void __launch_bounds__(256) flip_count_kernel(const uint8_t *__restrict__ a,
                                                         const uint8_t *__restrict__ b, int64_t n,
                                                         unsigned long long *__restrict__ count) {
  const uint16_t *bits_tab = g_tables.bits;
  pdl_launch_dependents();
  pdl_wait();
  unsigned long long local = 0;
  const int64_t nvec = ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15) ? 0 : n / 16;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    const uint4 qa = __ldg(reinterpret_cast<const uint4 *>(a) + v);
    const uint4 qb = __ldg(reinterpret_cast<const uint4 *>(b) + v);
    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
    const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t pa = (wa[k >> 2] >> (8 * (k & 3))) & 0xFFu;
      const uint32_t pb = (wb[k >> 2] >> (8 * (k & 3))) & 0xFFu;
      local += __popc((uint32_t)(bits_tab[pa] ^ bits_tab[pb]));
    }
  }
  for (int64_t i = nvec * 16 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    local += __popc((uint32_t)(bits_tab[a[i]] ^ bits_tab[b[i]]));
  const unsigned warp_sum = __reduce_add_sync(0xFFFFFFFFu, (unsigned)local);
  if ((threadIdx.x & 31) == 0 && warp_sum) atomicAdd(count, (unsigned long long)warp_sum);
}

// Masked decay: g <- fmaf(lambda, w, g) on pruned entries.  Thread t of
// CTA (x, y) owns the 4x4 block at block column 256x + t of block rows
// y, y + gridDim.y, ...; no thread divides.  The block's four 16-byte rows of
// g and 8-byte rows of W travel by cp.async into the thread's own shared
// slots, so the bytes in flight do not occupy registers and every block of a
// 355M-size weight is in flight in one wave.  A thread reads back only its
// own slots, so no barrier is needed.
__device__ __forceinline__ void cp_async(void *smem_dst, const void *gmem_src, int bytes16or8) {
  if (bytes16or8 == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}

template <bool BF16>
__global__ void __launch_bounds__(256) masked_decay_kernel(float *__restrict__ g,
                                                           const uint16_t *__restrict__ W,
                                                           const uint8_t *__restrict__ idx, int64_t R,
                                                           int64_t C, float lambda) {
  __shared__ __align__(16) float4 s_g[4][256];
  __shared__ __align__(16) uint2 s_w[4][256];
  const uint16_t *bits_tab = g_tables.bits;
  pdl_launch_dependents();
  pdl_wait();
  const int t = threadIdx.x;
  const int64_t bcols = C >> 2;
  const int64_t brows = R >> 2;
  const int64_t bc = (int64_t)blockIdx.x * blockDim.x + t;
  if (bc >= bcols) return;
  for (int64_t br = blockIdx.y; br < brows; br += gridDim.y) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t off = (4 * br + i) * C + 4 * bc;
      cp_async(&s_g[i][t], g + off, 16);
      cp_async(&s_w[i][t], W + off, 8);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const uint32_t p = __ldg(idx + br * bcols + bc);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    const uint32_t keep = bits_tab[p];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 gv = s_g[i][t];
      const uint2 wv = s_w[i][t];
      const uint32_t hw[4] = {wv.x & 0xFFFFu, wv.x >> 16, wv.y & 0xFFFFu, wv.y >> 16};
      float *gs = reinterpret_cast<float *>(&gv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float wf = BF16 ? __uint_as_float(hw[j] << 16) : __half2float(__ushort_as_half((unsigned short)hw[j]));
        if (!((keep >> (4 * i + j)) & 1u)) gs[j] = fmaf(lambda, wf, gs[j]);
      }
      *reinterpret_cast<float4 *>(g + (4 * br + i) * C + 4 * bc) = gv;
    }
  }
}

// Transpose of a row-major [rows x cols] 16-bit matrix into [cols x rows]:
// the input-gradient operand W^T of the dense fine-tuning GEMM.  64x64 tiles,
// 256 threads (16 x 16): every global access is 8 bytes (four elements), a
// half-warp covers 128 contiguous bytes of a row.  The shared tile has a row
// stride of 33 words, so the column reads of the store phase spread over the
// banks.  Edges (rows or cols not multiples of 4 or 64) take element accesses.
constexpr int kTransTile = 64;
constexpr int kTransStride = 66;   // 16-bit elements per shared row (33 words)

__global__ void __launch_bounds__(256) transpose16_kernel(const uint16_t *__restrict__ in,
                                                          uint16_t *__restrict__ out, int64_t rows, int64_t cols) {
  __shared__ __align__(8) uint16_t tile[kTransTile * kTransStride];
  pdl_launch_dependents();
  pdl_wait();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t c0 = (int64_t)blockIdx.x * kTransTile;
  const bool vec_in = (cols & 3) == 0, vec_out = (rows & 3) == 0;
  for (int64_t r0 = (int64_t)blockIdx.y * kTransTile; r0 < rows; r0 += (int64_t)gridDim.y * kTransTile) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int lr = ty + 16 * k;
      const int64_t r = r0 + lr, c = c0 + 4 * tx;
      uint32_t lo = 0, hi = 0;
      if (r < rows) {
        if (vec_in && c + 4 <= cols) {
          const uint2 v = *reinterpret_cast<const uint2 *>(in + r * cols + c);
          lo = v.x;
          hi = v.y;
        } else {
          const uint16_t *src = in + r * cols;
          const uint32_t e0 = c < cols ? src[c] : 0u, e1 = c + 1 < cols ? src[c + 1] : 0u;
          const uint32_t e2 = c + 2 < cols ? src[c + 2] : 0u, e3 = c + 3 < cols ? src[c + 3] : 0u;
          lo = e0 | (e1 << 16);
          hi = e2 | (e3 << 16);
        }
      }
      uint32_t *dst = reinterpret_cast<uint32_t *>(&tile[lr * kTransStride + 4 * tx]);
      dst[0] = lo;
      dst[1] = hi;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int lc = ty + 16 * k;              // output row = input column c0 + lc
      const int64_t c = c0 + lc, r = r0 + 4 * tx;
      if (c < cols) {
        const uint32_t e0 = tile[(4 * tx) * kTransStride + lc], e1 = tile[(4 * tx + 1) * kTransStride + lc];
        const uint32_t e2 = tile[(4 * tx + 2) * kTransStride + lc], e3 = tile[(4 * tx + 3) * kTransStride + lc];
        uint16_t *dst = out + c * rows;
        if (vec_out && r + 4 <= rows) {
          *reinterpret_cast<uint2 *>(dst + r) = make_uint2(e0 | (e1 << 16), e2 | (e3 << 16));
        } else {
          if (r < rows) dst[r] = (uint16_t)e0;
          if (r + 1 < rows) dst[r + 1] = (uint16_t)e1;
          if (r + 2 < rows) dst[r + 2] = (uint16_t)e2;
          if (r + 3 < rows) dst[r + 3] = (uint16_t)e3;
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace sp24
