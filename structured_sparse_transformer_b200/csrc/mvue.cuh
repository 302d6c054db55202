// MVUE 2:4 sparsification of dY^T along tokens: the sparse operand of the
// weight-gradient GEMM dW = MVUE(dY^T) X.
//
// "Accelerating Transformer Pre-training with 2:4 Sparsity", reproducibility
// table, Software Dependencies row (the MVUE kernel).  The pages do not define
// the estimator; this kernel computes the minimum-variance unbiased estimate that
// keeps exactly two of every four consecutive tokens of each column of dY:
// keep probabilities p_i = min(1, c |v_i|) summing to 2, kept values v_i / p_i,
// two entries drawn by systematic sampling with one uniform per group:
//   * no |v_i| reaches half the group's sum S: points u S/2 and u S/2 + S/2 on
//     the cumulative sums of |v| in index order pick two entries, each kept as
//     sign(v_i) S/2;
//   * else the largest |v_m| (lowest index among equal) is kept as is, and the
//     point u R on the cumulative sums of the other three (R their sum) picks
//     the second, kept as sign(v_k) R (R = 0: the lowest other position, +0).
// An entry is picked by counting the cumulative sums at or below the point.
// Every decision is an fp64 operation in that order, without contraction (each
// sum is exact for an fp16 group), and a kept value is stored as
// RNE_dtype(RNE_fp32(estimate)).
//
// Uniforms: group g (tokens 4g..4g+3) of column n takes the 32-bit half
// (g % 2) of word (g % 8) / 2 of Philox4x64-10 (Salmon, Moraes, Dror and Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011) at counter
// (g / 8, n, 0, 0) with key (seed, offset); u = (bits >> 8) * 2^-24.
//
// Layout: dY [T x N] row-major (leading dimension ldy) in; out the compressed
// rows of dY^T, values [N x T/2] and the tensor-core metadata chunks of an
// [N x T] operand (2048 bytes per 128 rows x 128 tokens, chunk index
// (n / 128) * ceil(T / 128) + t / 128), exactly as the forward operand of W.
// One CTA per 128 tokens x 64 columns (half a chunk's rows): the tile is staged
// in shared memory (16-byte loads along the columns), then each of 256 threads
// takes one column and 32 tokens (eight groups: one Philox block), writes 32
// bytes of its output row and its metadata nibbles into the CTA's 1 KB half of
// the chunk, which the CTA then stores with 16-byte writes.  Groups past T and rows past N get the
// padding code (positions 0, 1), so whole chunks are always written.
#pragma once
#include "sp24_common.cuh"

namespace sp24 {

constexpr int kMvueTokens = 128;
constexpr int kMvueCols = 64;
constexpr int kMvueThreads = 256;

// Both 64-bit halves of the 128-bit product a * b from three 32 x 32 -> 64
// partial products and one more for the top (schoolbook, carries folded into
// the wide multiply-adds: each partial sum stays below 2^64).
__device__ __forceinline__ void mulhilo64(uint64_t a, uint64_t b, uint64_t &hi, uint64_t &lo) {
  const uint32_t al = (uint32_t)a, ah = (uint32_t)(a >> 32), bl = (uint32_t)b, bh = (uint32_t)(b >> 32);
  const uint64_t t0 = (uint64_t)al * bl;
  const uint64_t t1 = (uint64_t)al * bh + (t0 >> 32);
  const uint64_t t2 = (uint64_t)ah * bl + (uint32_t)t1;
  hi = (uint64_t)ah * bh + (t1 >> 32) + (t2 >> 32);
  lo = (t2 << 32) | (uint32_t)t0;
}

// The ten round keys of Philox4x64-10 for key (k0, k1): round r uses
// (k0 + r W0, k1 + r W1) mod 2^64 with the Weyl increments W0, W1.  The same
// for every thread, so the host computes them once per launch.
struct PhiloxKeys {
  uint64_t k0[10], k1[10];
};

__host__ __device__ inline PhiloxKeys philox4x64_keys(uint64_t k0, uint64_t k1) {
  PhiloxKeys ks;
  for (int r = 0; r < 10; ++r) {
    ks.k0[r] = k0 + (uint64_t)r * 0x9E3779B97F4A7C15ull;
    ks.k1[r] = k1 + (uint64_t)r * 0xBB67AE8584CAA73Bull;
  }
  return ks;
}

__device__ __forceinline__ void philox4x64_10(uint64_t (&c)[4], const PhiloxKeys &ks) {
  constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ull, kM1 = 0xCA5A826395121157ull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    uint64_t hi0, lo0, hi1, lo1;
    mulhilo64(c[0], kM0, hi0, lo0);
    mulhilo64(c[2], kM1, hi1, lo1);
    const uint64_t n0 = hi1 ^ c[1] ^ ks.k0[r], n2 = hi0 ^ c[3] ^ ks.k1[r];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
  }
}

// Number of the cumulative sums c1, c2, c3 at or below the point: the entry it falls in.
__device__ __forceinline__ int count_le(double c1, double c2, double c3, double p) {
  return (int)(c1 <= p) + (int)(c2 <= p) + (int)(c3 <= p);
}

template <bool BF16>
__device__ __forceinline__ uint32_t mvue_bits(double x) {
  const float f = __double2float_rn(x);
  if (BF16) return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
  return (uint32_t)__half_as_ushort(__float2half_rn(f));
}

// |v| of two 16-bit values packed in one word (sign bits cleared), exact in fp64.
template <bool BF16>
__device__ __forceinline__ void mag2_f64(uint32_t m2, double &lo, double &hi) {
  if (BF16) {
    lo = (double)__uint_as_float(m2 << 16);
    hi = (double)__uint_as_float(m2 & 0xFFFF0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&m2));
    lo = (double)f.x;
    hi = (double)f.y;
  }
}

template <bool BF16>
__device__ __forceinline__ double mag_f64(uint32_t m) {
  if (BF16) return (double)__uint_as_float(m << 16);
  return (double)__half2float(__ushort_as_half((unsigned short)m));
}

// Integer constants formed from the run-time 1 (multiply-adds by them stay on
// the FMA pipe; the ALU pipe is this kernel's busy one).
struct MvueConsts {
  uint32_t k4, k16, k22, k10, k64k;   // 4, 16, 0x22, 0x10, 65536
  __device__ __forceinline__ explicit MvueConsts(uint32_t one)
      : k4(one << 2), k16(one << 4), k22(one * 0x22u), k10(one << 4), k64k(one << 16) {}
};

// Entry i (0..3) of a group held as lo = v0 | v1 << 16, hi = v2 | v3 << 16, in
// the low 16 bits of one byte permutation (selector 0x22 i + 0x10 picks bytes
// 2i and 2i + 1 of the pair; the upper 16 bits are left unspecified).
__device__ __forceinline__ uint32_t entry_bits(uint32_t lo, uint32_t hi, int i, const MvueConsts &K) {
  return __byte_perm(lo, hi, imad((uint32_t)i, K.k22, K.k10));
}

// One group of four (16-bit storage bits in lo/hi), without branches on the
// group's case: the cumulative sums run over w = |v| with the largest entry
// zeroed when it is kept outright, which are the sums of |v| (first case) or of
// the other three (second case) in the same operation order.  Both kept
// estimates have the magnitude `step` (S/2, or R) except the entry kept as is,
// so one rounding RNE_dtype(RNE_fp32(step)) serves both and the signs come from
// the stored bits.  The largest |v| is found on the magnitude bits (for finite
// values their order is that of the magnitudes; equal magnitudes, equal bits):
// keys (bits << 2) | (3 - i) make one unsigned max pick the largest, lowest
// index first.  Returns the metadata code pa | pb << 2 of the kept positions
// pa < pb and their output bits packed as bits(pa) | bits(pb) << 16.
template <bool BF16>
__device__ __forceinline__ void mvue_group(uint32_t lo, uint32_t hi, double u, const MvueConsts &K,
                                           uint32_t &code, uint32_t &packed) {
  const uint32_t lm = lo & 0x7FFF7FFFu, hm = hi & 0x7FFF7FFFu;
  double a[4];
  mag2_f64<BF16>(lm, a[0], a[1]);
  mag2_f64<BF16>(hm, a[2], a[3]);
  const double s = __dadd_rn(__dadd_rn(__dadd_rn(a[0], a[1]), a[2]), a[3]);
  const uint32_t km = max(max(imad(lm & 0xFFFFu, K.k4, 3u), imad(lm >> 16, K.k4, 2u)),
                          max(imad(hm & 0xFFFFu, K.k4, 1u), imad(hm >> 16, K.k4, 0u)));
  const int m = (int)((km & 3u) ^ 3u);
  const double am = mag_f64<BF16>(km >> 2);
  const bool capped = __dadd_rn(am, am) >= s;
  // A 16-bit magnitude widened to fp64 has a zero low word, so zeroing the
  // entry kept outright only selects the high word.
  double w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = __hiloint2double((capped && i == m) ? 0 : __double2hiint(a[i]), 0);
  const double e1 = w[0];
  const double e2 = __dadd_rn(e1, w[1]);
  const double e3 = __dadd_rn(e2, w[2]);
  const double tot = __dadd_rn(e3, w[3]);
  const double step = capped ? tot : __dmul_rn(tot, 0.5);
  const double q1 = __dmul_rn(u, step);
  int i1 = count_le(e1, e2, e3, q1);
  const int i2 = capped ? m : count_le(e1, e2, e3, __dadd_rn(q1, step));
  const bool empty = capped && !(tot > 0.0);        // at most one nonzero entry
  if (empty) i1 = m == 0 ? 1 : 0;
  // In the first case the two points always select two different nonzero
  // entries, although the cumulative sums are rounded: round-to-nearest-even is
  // monotone, so the second point (half the total past the first) passes the
  // first point's entry; the one way to stay would need the total to round up
  // by half an ulp of the last entry's complement, and ties-to-even then makes
  // that entry reach half the total, i.e. the group capped.
  const uint32_t mag = empty ? 0u : mvue_bits<BF16>(step);
  // Entry i1 takes the estimate's magnitude and its own sign (nothing when empty);
  // entry i2 keeps its stored bits when it is the capped entry m (i2 == m then).
  const uint32_t b1 = (entry_bits(lo, hi, i1, K) & (empty ? 0u : 0x8000u)) | mag;
  const uint32_t b2 = (entry_bits(lo, hi, i2, K) & (capped ? 0xFFFFu : 0x8000u)) | (capped ? 0u : mag);
  const bool fwd = i1 < i2;
  code = fwd ? imad((uint32_t)i2, K.k4, (uint32_t)i1) : imad((uint32_t)i1, K.k4, (uint32_t)i2);
  packed = fwd ? imad(b2, K.k64k, b1) : imad(b1, K.k64k, b2);
}

template <bool BF16>
__global__ void __launch_bounds__(kMvueThreads) mvue_sparsify_kernel(
    const uint16_t *__restrict__ dy, int64_t T, int64_t N, int64_t ldy, const __grid_constant__ PhiloxKeys keys,
    uint16_t *__restrict__ vals, uint8_t *__restrict__ meta) {
  __shared__ __align__(16) uint32_t s_tile[kMvueTokens][kMvueCols / 2];   // [token][column pair]
  __shared__ __align__(16) uint16_t s_meta[512];                           // this CTA's half chunk
  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * kMvueTokens;
  const int64_t n0 = (int64_t)blockIdx.y * kMvueCols;
  pdl_launch_dependents();
  pdl_wait();

  // Stage dY[t0 .. t0+127][n0 .. n0+63] (zeros outside the matrix).
#pragma unroll
  for (int k = 0; k < (kMvueTokens * kMvueCols * 2 / 16) / kMvueThreads; ++k) {
    const int id = tid + kMvueThreads * k;
    const int row = id >> 3, ch = id & 7;
    uint4 q = make_uint4(0u, 0u, 0u, 0u);
    if (t0 + row < T && n0 + 8 * ch < N)
      q = __ldg(reinterpret_cast<const uint4 *>(dy + (t0 + row) * ldy + n0 + 8 * ch));
    *reinterpret_cast<uint4 *>(&s_tile[row][4 * ch]) = q;
  }
  __syncthreads();

  // Thread (segment w, column p): column n0 + p, tokens 32w .. 32w + 31 (eight groups,
  // one Philox block).  A warp takes 32 consecutive columns of one segment.
  const int p = tid & 63, w = tid >> 6;
  const int64_t tseg = t0 + 32 * w;                         // first token of this thread's segment
  const int ngroups = (int)max((int64_t)0, min((int64_t)8, (T - tseg) / 4));
  const int rh = (int)(blockIdx.y & 1);
  const int64_t n = n0 + p;
  uint64_t rnd[4] = {(uint64_t)(tseg >> 5), (uint64_t)n, 0ull, 0ull};
  philox4x64_10(rnd, keys);
  const MvueConsts K(load_one());
  uint32_t nib = 0;                                         // built from group 7 down (Horner, base 16)
  uint32_t packed[8];
  const uint32_t sel = (p & 1) ? 0x7632u : 0x5410u;         // this column's halves of the staged words
#pragma unroll
  for (int j = 7; j >= 0; --j) {
    packed[j] = 0u;
    uint32_t code = 4u;                                     // padding: positions 0, 1
    if (j < ngroups) {
      const uint32_t *col = &s_tile[32 * w + 4 * j][p >> 1];
      const uint32_t lo = __byte_perm(col[0], col[kMvueCols / 2], sel);
      const uint32_t hi = __byte_perm(col[kMvueCols], col[3 * kMvueCols / 2], sel);
      const uint32_t u32 = (uint32_t)(rnd[j >> 1] >> (32 * (j & 1)));
      const double u = (double)(u32 >> 8) * 0x1p-24;
      mvue_group<BF16>(lo, hi, u, K, code, packed[j]);
    }
    nib = imad(nib, K.k16, code);
  }
  if (n < N && ngroups > 0) {
    uint16_t *dst = vals + n * (T >> 1) + (tseg >> 1);
    *reinterpret_cast<uint4 *>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    if (ngroups > 4) *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  }
  if (n >= N) nib = 0x44444444u;
  {
    // Metadata: row r of the chunk, K step w; groups 0-3 go to lane
    // (r % 8) + 16 (r / 16), groups 4-7 to that lane + 8; the 16-bit half is (r / 8) % 2.
    const int r = 64 * rh + p;
    const int lane0 = (r & 7) + 16 * (r >> 4) - 64 * rh;
    const int half = (r >> 3) & 1;
    s_meta[(lane0 * 16 + 4 * w + 2 * half) >> 1] = (uint16_t)(nib & 0xFFFFu);
    s_meta[((lane0 + 8) * 16 + 4 * w + 2 * half) >> 1] = (uint16_t)(nib >> 16);
  }
  __syncthreads();
  if (tid < 64) {
    const size_t chunk = (size_t)(blockIdx.y >> 1) * gridDim.x + blockIdx.x;
    *reinterpret_cast<uint4 *>(meta + chunk * 2048 + 1024 * rh + 16 * tid) =
        *reinterpret_cast<const uint4 *>(&s_meta[8 * tid]);
  }
}

}  // namespace sp24
