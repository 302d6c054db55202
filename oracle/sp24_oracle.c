/*
 * CPU oracle for the 2:4 transposable-mask path -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares no code with the CUDA path.  It is written to
 * be slow and obviously correct: brute force over every candidate pattern,
 * exact integer arithmetic, no blocking, no fusion.
 *
 * Source: "Accelerating Transformer Pre-training with 2:4 Sparsity".
 *   - Reproducibility table, Pseudocode row, Algorithm 1 (transposable mask
 *     search): take |W|, convolve it at stride 4 with the candidate 4x4 mask
 *     patterns m, and return the argmax over the patterns for every block.
 *   - Abstract: masked decay is applied on gradients; the flip rate monitors
 *     mask stability (its formula lives in the Python half of the oracle).
 *
 * Readings of the pages (the pages leave these open):
 *   - The candidate set m is every 4x4 0/1 matrix with exactly two ones in each
 *     row and each column (transposable 2:4).  Order: each row picks a column
 *     pair from (0,1),(0,2),(0,3),(1,2),(1,3),(2,3); row 0's choice varies
 *     slowest; a tuple is kept iff every column ends with two ones.  This is
 *     lexicographic order on the (row0, row1, row2, row3) pair tuple.
 *   - The convolution output of a pattern is the EXACT real sum of the eight
 *     |W| values it covers; the argmax takes the lowest pattern index on ties
 *     (first maximal index, as argmax conventionally returns).
 *   - The masked decay is g <- g + lambda * W on pruned entries (mask 0), kept
 *     entries unchanged, computed as one fp32 fused multiply-add.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_NONFINITE (-1)
#define ORACLE_BAD_SHAPE (-2)
#define ORACLE_BAD_DTYPE (-3)

enum { DT_F16 = 0, DT_BF16 = 1 };

/* ---------------------------------------------------------------- patterns */

static uint16_t g_pattern[128]; /* bit 4*i+j set <=> row i, column j kept */
static int g_npattern = -1;

static void build_patterns(void) {
  static const int pair[6][2] = {{0, 1}, {0, 2}, {0, 3}, {1, 2}, {1, 3}, {2, 3}};
  int n = 0;
  for (int r0 = 0; r0 < 6; ++r0)
    for (int r1 = 0; r1 < 6; ++r1)
      for (int r2 = 0; r2 < 6; ++r2)
        for (int r3 = 0; r3 < 6; ++r3) {
          int choice[4] = {r0, r1, r2, r3};
          int colcount[4] = {0, 0, 0, 0};
          uint16_t bits = 0;
          for (int i = 0; i < 4; ++i) {
            int a = pair[choice[i]][0], b = pair[choice[i]][1];
            colcount[a] += 1;
            colcount[b] += 1;
            bits |= (uint16_t)(1u << (4 * i + a));
            bits |= (uint16_t)(1u << (4 * i + b));
          }
          if (colcount[0] == 2 && colcount[1] == 2 && colcount[2] == 2 && colcount[3] == 2)
            g_pattern[n++] = bits;
        }
  g_npattern = n;
}

int oracle_pattern_count(void) {
  if (g_npattern < 0) build_patterns();
  return g_npattern;
}

/* Copies the pattern table (bit 4*i+j = row i, column j kept) into out[0..n). */
int oracle_patterns(uint16_t *out) {
  int n = oracle_pattern_count();
  for (int p = 0; p < n; ++p) out[p] = g_pattern[p];
  return n;
}

/* ------------------------------------------------ exact magnitudes (bigint) */

/* |w| as an exact integer multiple of the dtype's smallest subnormal:
 * fp16: units of 2^-24 (value = sig * 2^shift units), bf16: units of 2^-133.
 * A sum of eight such integers stays below 2^264, so five 64-bit limbs hold it. */
#define LIMBS 5
typedef struct { uint64_t w[LIMBS]; } big_t;

static int decode_magnitude(uint16_t bits, int dtype, uint64_t *sig, int *shift) {
  uint32_t a = bits & 0x7FFFu;
  uint32_t e, f, emax, implicit;
  if (dtype == DT_F16) { e = a >> 10; f = a & 0x3FFu; emax = 31; implicit = 0x400u; }
  else                 { e = a >> 7;  f = a & 0x7Fu;  emax = 255; implicit = 0x80u; }
  if (e == emax) return ORACLE_NONFINITE;
  if (e == 0) { *sig = f; *shift = 0; }
  else        { *sig = f | implicit; *shift = (int)e - 1; }
  return ORACLE_OK;
}

static void big_add_shifted(big_t *acc, uint64_t sig, int shift) {
  int limb = shift / 64, off = shift % 64;
  unsigned __int128 v = (unsigned __int128)sig << off;
  uint64_t part[2] = {(uint64_t)v, (uint64_t)(v >> 64)};
  unsigned __int128 carry = 0;
  for (int i = limb; i < LIMBS; ++i) {
    unsigned __int128 s = (unsigned __int128)acc->w[i] + carry;
    if (i - limb < 2) s += part[i - limb];
    acc->w[i] = (uint64_t)s;
    carry = s >> 64;
  }
}

static int big_cmp(const big_t *a, const big_t *b) {
  for (int i = LIMBS - 1; i >= 0; --i) {
    if (a->w[i] > b->w[i]) return 1;
    if (a->w[i] < b->w[i]) return -1;
  }
  return 0;
}

/* --------------------------------------------------------- Algorithm 1 */

/* idx[(r/4)*(cols/4) + c/4] = argmax over patterns of the exact kept |W| sum of
 * the 4x4 block at (r, c); ties go to the lowest pattern index.
 * w is row-major with leading dimension ldw (elements). */
int oracle_mask_search(const uint16_t *w, int dtype, int64_t rows, int64_t cols, int64_t ldw,
                       uint8_t *idx) {
  if (dtype != DT_F16 && dtype != DT_BF16) return ORACLE_BAD_DTYPE;
  if (rows % 4 || cols % 4 || rows < 0 || cols < 0 || ldw < cols) return ORACLE_BAD_SHAPE;
  int np = oracle_pattern_count();
  int64_t brows = rows / 4, bcols = cols / 4;
  int status = ORACLE_OK;
#pragma omp parallel for schedule(static)
  for (int64_t br = 0; br < brows; ++br) {
    for (int64_t bc = 0; bc < bcols; ++bc) {
      uint64_t sig[16];
      int shift[16];
      int bad = 0;
      for (int i = 0; i < 4; ++i)
        for (int j = 0; j < 4; ++j)
          if (decode_magnitude(w[(4 * br + i) * ldw + 4 * bc + j], dtype, &sig[4 * i + j],
                               &shift[4 * i + j]) != ORACLE_OK)
            bad = 1;
      if (bad) {
#pragma omp atomic write
        status = ORACLE_NONFINITE;
        idx[br * bcols + bc] = 0;
        continue;
      }
      big_t best;
      int best_p = -1;
      for (int p = 0; p < np; ++p) {
        big_t acc;
        memset(&acc, 0, sizeof acc);
        for (int cell = 0; cell < 16; ++cell)
          if (g_pattern[p] >> cell & 1u) big_add_shifted(&acc, sig[cell], shift[cell]);
        if (best_p < 0 || big_cmp(&acc, &best) > 0) { best = acc; best_p = p; }
      }
      idx[br * bcols + bc] = (uint8_t)best_p;
    }
  }
  return status;
}

/* --------------------------------------------------------- masked decay */

static float to_float(uint16_t bits, int dtype) {
  if (dtype == DT_BF16) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
  }
  uint64_t sig;
  int shift;
  if (decode_magnitude(bits, DT_F16, &sig, &shift) != ORACLE_OK) {
    /* exponent all ones: infinity (zero fraction) or NaN, outside the finite-weight contract */
    float inf = (bits & 0x3FFu) ? NAN : INFINITY;
    return (bits & 0x8000u) ? -inf : inf;
  }
  float mag = ldexpf((float)sig, shift - 24); /* exact: sig < 2^11 */
  return (bits & 0x8000u) ? -mag : mag;
}

/* g[r*ldg + c] <- fmaf(lambda, W[r][c], g) where the mask of (r, c) is 0;
 * unchanged where it is 1.  One rounding (fused multiply-add). */
int oracle_masked_decay(float *g, int64_t ldg, const uint16_t *w, int dtype, int64_t rows,
                        int64_t cols, int64_t ldw, const uint8_t *idx, float lambda) {
  if (dtype != DT_F16 && dtype != DT_BF16) return ORACLE_BAD_DTYPE;
  if (rows % 4 || cols % 4 || ldw < cols || ldg < cols) return ORACLE_BAD_SHAPE;
  int np = oracle_pattern_count();
  int64_t bcols = cols / 4;
  int status = ORACLE_OK;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      int p = idx[(r / 4) * bcols + c / 4];
      if (p >= np) {
#pragma omp atomic write
        status = ORACLE_BAD_SHAPE;
        continue;
      }
      int kept = g_pattern[p] >> (4 * (r % 4) + (c % 4)) & 1u;
      if (!kept) g[r * ldg + c] = fmaf(lambda, to_float(w[r * ldw + c], dtype), g[r * ldg + c]);
    }
  }
  return status;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
