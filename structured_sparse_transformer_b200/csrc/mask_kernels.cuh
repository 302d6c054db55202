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
// Mask search is exact.  The fast path sums magnitudes in fp32 where the
// block's magnitude range proves those sums exact (search_block_fast); the
// remaining blocks take an integer search.  There each |w| becomes an integer multiple of its dtype's
// smallest subnormal (fp16: always; bf16: relative to the block's largest
// exponent, 32 binades deep), pre-shifted left by 12 bits.  The 12 low bits of
// a pattern's key hold (35 - top rank) << 6 | (35 - bottom rank), so one
// unsigned 64-bit max picks the largest exact sum and, among equal sums, the
// lowest pattern index.  The max over the 90 patterns is taken by a dynamic
// program over column-count states (top rows 0-1 and bottom rows 2-3, see
// sp24_tables.cuh) instead of enumerating all 90.  bf16 blocks whose nonzero
// magnitudes span more than 32 binades take an exact multi-word brute force.
#pragma once
#include "sp24_common.cuh"
#include "sp24_tables.cuh"

namespace sp24 {

using u64 = unsigned long long;

__constant__ PatternTables c_tables = make_pattern_tables();

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
                                                        const uint16_t *s_bits) {
  const uint32_t words[8] = {w00, w01, w10, w11, w20, w21, w30, w31};
  u64 best[5] = {0, 0, 0, 0, 0};
  uint32_t best_p = 0;
  for (int p = 0; p < kNumPatterns; ++p) {
    u64 acc[5] = {0, 0, 0, 0, 0};
    const uint32_t bits = s_bits[p];
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

// Pattern index of one 4x4 block given as 4 rows x 2 words (two 16-bit values each).
template <bool BF16>
__device__ __forceinline__ uint32_t search_block(const uint32_t (&w)[4][2], const uint8_t *s_index,
                                                 const uint16_t *s_bits) {
  u64 v[16];
  if (!BF16) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint32_t a = (w[c >> 2][(c >> 1) & 1] >> ((c & 1) << 4)) & 0x7FFFu;
      const uint32_t e = a >> 10;
      const uint32_t sig = e ? ((a & 0x3FFu) | 0x400u) : a;
      const uint32_t ep = e ? e - 1 : 0;
      v[c] = (u64)sig << (ep + 12);
    }
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
                                    s_bits);
  }
  const uint32_t r = dp_argmax_ranks(v);
  return s_index[(35 - (r >> 6)) * 36 + (35 - (r & 63))];
}

constexpr uint32_t kNeedsExact = 0xFFu;  // fast path could not certify its sums

// Fast path of the search on fp32 arithmetic.  Every |w| converts to fp32
// exactly.  A sum of eight of them is exact in fp32 when the block's smallest
// nonzero magnitude is at least its largest times 2^-10 (fp16: 11-bit
// significands, 3 carry bits, 24-bit fp32 significand) or 2^-13 (bf16); then
// every partial sum below is exact, comparisons are exact, and the result
// equals the exact search.  Blocks that fail the test return kNeedsExact.
// Ranks: within a column-count state the first combo (lowest rank) reaching
// the state's maximum wins (strict >); across states the smallest
// (top rank, bottom rank) among the states reaching the global maximum wins.
template <bool BF16>
__device__ __forceinline__ uint32_t search_block_fast(const uint32_t (&w)[4][2], const uint8_t *s_index) {
  constexpr PatternTables T = make_pattern_tables();
  float v[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t h = (w[c >> 2][(c >> 1) & 1] >> ((c & 1) << 4)) & 0x7FFFu;
    v[c] = BF16 ? __uint_as_float(h << 16) : __half2float(__ushort_as_half((unsigned short)h));
  }
  float vmax = v[0], vmin = v[0] > 0.0f ? v[0] : __int_as_float(0x7F800000);
#pragma unroll
  for (int c = 1; c < 16; ++c) {
    vmax = fmaxf(vmax, v[c]);
    vmin = fminf(vmin, v[c] > 0.0f ? v[c] : __int_as_float(0x7F800000));
  }
  if (!(vmin >= vmax * (BF16 ? 0x1p-13f : 0x1p-10f))) return kNeedsExact;

  float P[4][6];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < 6; ++q) P[i][q] = v[4 * i + pair_lo(q)] + v[4 * i + pair_hi(q)];
  float top[kNumStates], bot[kNumStates];
  uint32_t tr[kNumStates], br[kNumStates];
  bool seen_t[kNumStates] = {}, seen_b[kNumStates] = {};
#pragma unroll
  for (int c = 0; c < 36; ++c) {
    const int st = T.top_state[c];
    const float kt = P[0][c / 6] + P[1][c % 6];
    if (!seen_t[st]) { top[st] = kt; tr[st] = (uint32_t)c; seen_t[st] = true; }
    else { const bool gt = kt > top[st]; top[st] = gt ? kt : top[st]; tr[st] = gt ? (uint32_t)c : tr[st]; }
    const int sb = T.bot_state[c];
    const float kb = P[2][c / 6] + P[3][c % 6];
    if (!seen_b[sb]) { bot[sb] = kb; br[sb] = (uint32_t)c; seen_b[sb] = true; }
    else { const bool gt = kb > bot[sb]; bot[sb] = gt ? kb : bot[sb]; br[sb] = gt ? (uint32_t)c : br[sb]; }
  }
  float tot[kNumStates];
  float best = 0.0f;
#pragma unroll
  for (int st = 0; st < kNumStates; ++st) { tot[st] = top[st] + bot[st]; best = fmaxf(best, tot[st]); }
  uint32_t key = 0xFFFFu;
#pragma unroll
  for (int st = 0; st < kNumStates; ++st)
    if (tot[st] == best) key = min(key, (tr[st] << 6) | br[st]);
  return s_index[(key >> 6) * 36 + (key & 63)];
}

__device__ __forceinline__ uint32_t half_of(const uint32_t (&row)[4], int blk, uint32_t k) {
  const uint32_t wd = (k & 2) ? row[2 * blk + 1] : row[2 * blk];
  return (wd >> ((k & 1) << 4)) & 0xFFFFu;
}

__device__ __forceinline__ uint32_t pick_row(const uint32_t (&w)[4][4], uint32_t i, int word) {
  const uint32_t a = (i & 1) ? w[1][word] : w[0][word];
  const uint32_t b = (i & 1) ? w[3][word] : w[2][word];
  return (i & 2) ? b : a;
}

// Physical word of (W column c_local, block row br_local) in the transposed
// values tile: 16-byte chunks XOR-swizzled by c_local/8, words inside a chunk
// by c_local/64, so the writes of a warp hit 32 distinct banks.
__device__ __forceinline__ int vcol_word(int c_local, int br_local) {
  return c_local * 32 + ((((br_local >> 2) ^ (c_local >> 3)) & 7) << 2) +
         ((br_local & 3) ^ (((c_local >> 6) & 1) << 1));
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

constexpr int kTile = 128;       // W tile: 128 rows x 128 columns per CTA
constexpr int kMaskThreads = 256;

// One CTA per 128x128 tile of W.  Thread t owns units (4 rows x 8 columns =
// two blocks) at unit column t%16 and block rows t/16 and t/16 + 16.
//   SEARCH:   compute the mask (else read it from idx)
//   COMPRESS: write the compressed orientations whose pointers are non-null
//             (values + tensor-core metadata)
//   FLIP:     add the number of mask bits that differ from idx_prev to *flip_count
template <bool BF16, bool SEARCH, bool COMPRESS, bool FLIP>
__global__ void __launch_bounds__(kMaskThreads, 2) mask_tile_kernel(
    const uint16_t *__restrict__ W, int64_t R, int64_t C, int64_t ldw, uint8_t *__restrict__ idx,
    const uint8_t *__restrict__ idx_prev, unsigned long long *__restrict__ flip_count,
    uint16_t *__restrict__ vals_row, uint8_t *__restrict__ meta_row, uint16_t *__restrict__ vals_col,
    uint8_t *__restrict__ meta_col) {
  __shared__ uint16_t s_bits[256];
  __shared__ uint16_t s_rowcode[256];
  __shared__ uint16_t s_colcode[256];
  __shared__ uint8_t s_index[36 * 36];
  __shared__ uint8_t s_idx[32][36];
  __shared__ __align__(16) uint32_t s_vcol[COMPRESS ? kTile * 32 : 4];
  __shared__ uint16_t s_queue[SEARCH ? 1024 : 2];
  __shared__ int s_qn;
  __shared__ unsigned long long s_flip;

  const int tid = threadIdx.x;
  for (int i = tid; i < 256; i += kMaskThreads) {
    s_bits[i] = c_tables.bits[i];
    s_rowcode[i] = c_tables.rowcode[i];
    s_colcode[i] = c_tables.colcode[i];
  }
  for (int i = tid; i < 36 * 36; i += kMaskThreads) s_index[i] = c_tables.index[i];
  if (tid == 0) { s_flip = 0; s_qn = 0; }
  __syncthreads();

  const int64_t tile_r = (int64_t)blockIdx.y * kTile;
  const int64_t tile_c = (int64_t)blockIdx.x * kTile;
  const int64_t bcols = C >> 2;
  const int uc = tid & 15;
  const bool vec16 = (ldw & 7) == 0;  // rows 16-byte aligned: one 128-bit load per row of a unit

  // Phase 1: load both units, search the blocks the fast path can certify,
  // queue the others (SEARCH) or read the given mask (!SEARCH).
  uint32_t w[2][4][4];
#pragma unroll
  for (int half = 0; half < 2; ++half)
    load_unit(W, ldw, tile_r + 4 * ((tid >> 4) + 16 * half), tile_c + 8 * uc, R, C, vec16, w[half]);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int br = (tid >> 4) + 16 * half;
    const int64_t r0 = tile_r + 4 * br;
    const int64_t c0 = tile_c + 8 * uc;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const bool ok = r0 < R && c0 + 4 * (b + 1) <= C;
      uint32_t p = kPadIndex;
      if (ok) {
        if (SEARCH) {
          uint32_t blk[4][2];
#pragma unroll
          for (int i = 0; i < 4; ++i) { blk[i][0] = w[half][i][2 * b]; blk[i][1] = w[half][i][2 * b + 1]; }
          p = search_block_fast<BF16>(blk, s_index);
          if (p == kNeedsExact) {
            const int slot = atomicAdd(&s_qn, 1);
            s_queue[slot] = (uint16_t)(br * 32 + 2 * uc + b);
          }
        } else {
          p = idx[(r0 >> 2) * bcols + (c0 >> 2) + b];
        }
      }
      s_idx[br][2 * uc + b] = (uint8_t)p;
    }
  }

  // Phase 1b: blocks the fast path could not certify take the exact integer search.
  if (SEARCH) {
    __syncthreads();
    const int qn = s_qn;
    for (int k = tid; k < qn; k += kMaskThreads) {
      const int id = s_queue[k];
      const int br = id >> 5, bc = id & 31;
      const uint16_t *src = W + (tile_r + 4 * br) * ldw + tile_c + 4 * bc;
      uint32_t blk[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint2 q = __ldg(reinterpret_cast<const uint2 *>(src + i * ldw));
        blk[i][0] = q.x; blk[i][1] = q.y;
      }
      s_idx[br][bc] = (uint8_t)search_block<BF16>(blk, s_index, s_bits);
    }
  }
  if (SEARCH || COMPRESS || FLIP) __syncthreads();

  // Phase 2: per-thread outputs of its own blocks.
  unsigned long long flips = 0;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int br = (tid >> 4) + 16 * half;
    const int64_t r0 = tile_r + 4 * br;
    const int64_t c0 = tile_c + 8 * uc;
    const bool row_ok = r0 < R;
    const bool ok0 = row_ok && c0 + 4 <= C;
    const bool ok1 = row_ok && c0 + 8 <= C;
    uint32_t p[2];
    uint32_t x[4][4];  // the unit again (an L1 hit): keeps registers free during the search
    if (COMPRESS) load_unit(W, ldw, r0, c0, R, C, vec16, x);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      p[b] = s_idx[br][2 * uc + b];
      const bool ok = b ? ok1 : ok0;
      const int64_t bidx = (r0 >> 2) * bcols + (c0 >> 2) + b;
      if (SEARCH && ok) idx[bidx] = (uint8_t)p[b];
      if (FLIP && ok) flips += __popc((uint32_t)(s_bits[idx_prev[bidx]] ^ s_bits[p[b]]));
    }
    if (COMPRESS && ok0) {
      // Forward operand: kept values of each row, in column order.
      if (vals_row) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t packed[2];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint32_t nib = (s_rowcode[p[b]] >> (4 * i)) & 0xFu;
            packed[b] = half_of(x[i], b, nib & 3u) | (half_of(x[i], b, nib >> 2) << 16);
          }
          uint16_t *dst = vals_row + (r0 + i) * (C >> 1) + (c0 >> 1);
          if (ok1) *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[1]);
          else *reinterpret_cast<uint32_t *>(dst) = packed[0];
        }
      }
      // Input-gradient operand: kept values of each column, staged transposed.
#pragma unroll
      for (int b = 0; b < 2; ++b) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t nib = (s_colcode[p[b]] >> (4 * j)) & 0xFu;
          const int word = 2 * b + (j >> 1);
          const uint32_t lo = (pick_row(x, nib & 3u, word) >> ((j & 1) << 4)) & 0xFFFFu;
          const uint32_t hi = (pick_row(x, nib >> 2, word) >> ((j & 1) << 4)) & 0xFFFFu;
          s_vcol[vcol_word(8 * uc + 4 * b + j, br)] = lo | (hi << 16);
        }
      }
    }
  }

  if (FLIP) {
    const unsigned long long warp_sum = __reduce_add_sync(0xFFFFFFFFu, (unsigned)flips);
    if ((tid & 31) == 0 && warp_sum) atomicAdd(&s_flip, warp_sum);
  }
  if (COMPRESS || FLIP) __syncthreads();
  if (FLIP && tid == 0 && s_flip) atomicAdd(flip_count, s_flip);

  if (COMPRESS) {
    // Transposed values: W column c (a row of W^T) holds 64 kept values per tile.
    const int64_t half_rows = R >> 1;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int id = tid + kMaskThreads * k;
      const int c_local = id >> 3, q = id & 7;
      if (vals_col && tile_c + c_local < C && tile_r + 16 * q + 16 <= R) {
        const uint4 v = *reinterpret_cast<const uint4 *>(
            &s_vcol[c_local * 32 + (((q ^ (c_local >> 3)) & 7) << 2)]);
        const bool swap = (c_local >> 6) & 1;
        const uint4 o = swap ? make_uint4(v.z, v.w, v.x, v.y) : v;
        *reinterpret_cast<uint4 *>(vals_col + (tile_c + c_local) * half_rows + (tile_r >> 1) + 8 * q) = o;
      }
    }
    // Metadata: one 2048-byte chunk per 128x128 tile and orientation.  Lane L,
    // word kk (one 32-column K step of the MMA) holds rows m and m+8,
    // m = (L%8) + 16*(L/16), groups 4*((L/8)%2) .. +3 of that K step; the
    // low 16 bits are row m, the high 16 bits row m+8, one nibble per group.
    const bool col_side = tid >= 128;
    const int L = tid & 127;
    const int m_lo = (L & 7) + ((L >> 4) << 4);
    uint32_t words[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int g = kk * 8 + ((L >> 3) & 1) * 4 + e;
#pragma unroll
        for (int hsel = 0; hsel < 2; ++hsel) {
          const int m = m_lo + 8 * hsel;
          uint32_t nib;
          if (!col_side) nib = (s_rowcode[s_idx[m >> 2][g]] >> (4 * (m & 3))) & 0xFu;
          else nib = (s_colcode[s_idx[g][m >> 2]] >> (4 * (m & 3))) & 0xFu;
          word |= nib << (16 * hsel + 4 * e);
        }
      }
      words[kk] = word;
    }
    uint8_t *dst = col_side
                       ? (meta_col ? meta_col + ((size_t)blockIdx.x * gridDim.y + blockIdx.y) * 2048 + L * 16 : nullptr)
                       : (meta_row ? meta_row + ((size_t)blockIdx.y * gridDim.x + blockIdx.x) * 2048 + L * 16 : nullptr);
    if (dst) *reinterpret_cast<uint4 *>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
  }
}

// Flip count between two masks: popcount of the XOR of their pattern bits.
__global__ void __launch_bounds__(256) flip_count_kernel(const uint8_t *__restrict__ a,
                                                         const uint8_t *__restrict__ b, int64_t n,
                                                         unsigned long long *__restrict__ count) {
  __shared__ uint16_t s_bits[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bits[i] = c_tables.bits[i];
  __syncthreads();
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
      local += __popc((uint32_t)(s_bits[pa] ^ s_bits[pb]));
    }
  }
  for (int64_t i = nvec * 16 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    local += __popc((uint32_t)(s_bits[a[i]] ^ s_bits[b[i]]));
  const unsigned warp_sum = __reduce_add_sync(0xFFFFFFFFu, (unsigned)local);
  if ((threadIdx.x & 31) == 0 && warp_sum) atomicAdd(count, (unsigned long long)warp_sum);
}

// Masked decay: one thread per 4x4 block; g <- fmaf(lambda, w, g) on pruned entries.
template <bool BF16>
__global__ void __launch_bounds__(256) masked_decay_kernel(float *__restrict__ g,
                                                           const uint16_t *__restrict__ W,
                                                           const uint8_t *__restrict__ idx, int64_t R,
                                                           int64_t C, float lambda) {
  __shared__ uint16_t s_bits[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bits[i] = c_tables.bits[i];
  __syncthreads();
  const int64_t bcols = C >> 2;
  const int64_t nblocks = (R >> 2) * bcols;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
    const int64_t r0 = (b / bcols) * 4, c0 = (b % bcols) * 4;
    const uint32_t keep = s_bits[idx[b]];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 *gp = reinterpret_cast<float4 *>(g + (r0 + i) * C + c0);
      float4 gv = *gp;
      const uint2 wv = __ldg(reinterpret_cast<const uint2 *>(W + (r0 + i) * C + c0));
      const uint32_t hw[4] = {wv.x & 0xFFFFu, wv.x >> 16, wv.y & 0xFFFFu, wv.y >> 16};
      float wf[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        wf[j] = BF16 ? __uint_as_float(hw[j] << 16) : __half2float(__ushort_as_half((unsigned short)hw[j]));
      float *gs = reinterpret_cast<float *>(&gv);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (!((keep >> (4 * i + j)) & 1u)) gs[j] = fmaf(lambda, wf[j], gs[j]);
      *gp = gv;
    }
  }
}

}  // namespace sp24
