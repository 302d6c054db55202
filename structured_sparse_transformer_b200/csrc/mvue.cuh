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
// in shared memory (16-byte loads along the columns), then thread (warp w,
// lane p) takes columns 2p, 2p+1 and tokens 32w..32w+31 (one Philox block per
// column: eight groups), writes 32 bytes of each of its two output rows and
// its metadata nibbles into the CTA's 1 KB half of the chunk, which the CTA
// then stores with 16-byte writes.  Groups past T and rows past N get the
// padding code (positions 0, 1), so whole chunks are always written.
#pragma once
#include "sp24_common.cuh"

namespace sp24 {

constexpr int kMvueTokens = 128;
constexpr int kMvueCols = 64;
constexpr int kMvueThreads = 128;

__device__ __forceinline__ void philox4x64_10(uint64_t (&c)[4], uint64_t k0, uint64_t k1) {
  constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ull, kM1 = 0xCA5A826395121157ull;
  constexpr uint64_t kW0 = 0x9E3779B97F4A7C15ull, kW1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint64_t hi0 = __umul64hi(kM0, c[0]), lo0 = kM0 * c[0];
    const uint64_t hi1 = __umul64hi(kM1, c[2]), lo1 = kM1 * c[2];
    const uint64_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
  }
}

__device__ __forceinline__ double pick4(const double (&x)[4], int i) {
  return i == 0 ? x[0] : (i == 1 ? x[1] : (i == 2 ? x[2] : x[3]));
}

// Number of the cumulative sums c1, c2, c3 at or below the point: the entry it falls in.
__device__ __forceinline__ int count_le(double c1, double c2, double c3, double p) {
  return (int)(c1 <= p) + (int)(c2 <= p) + (int)(c3 <= p);
}

// One group: kept positions pa < pb and their fp64 estimates.
__device__ __forceinline__ void mvue_group(const double (&v)[4], double u, int &pa, int &pb, double &xa,
                                           double &xb) {
  double a[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = fabs(v[i]);
  const double c1 = a[0];
  const double c2 = __dadd_rn(c1, a[1]);
  const double c3 = __dadd_rn(c2, a[2]);
  const double s = __dadd_rn(c3, a[3]);
  int m = 0;
  double am = a[0];
#pragma unroll
  for (int i = 1; i < 4; ++i)
    if (a[i] > am) {
      am = a[i];
      m = i;
    }
  int p0, p1;
  double x0, x1;
  if (__dadd_rn(am, am) >= s) {
    const double b0 = m == 0 ? 0.0 : a[0], b1 = m == 1 ? 0.0 : a[1];
    const double b2 = m == 2 ? 0.0 : a[2], b3 = m == 3 ? 0.0 : a[3];
    const double e1 = b0;
    const double e2 = __dadd_rn(e1, b1);
    const double e3 = __dadd_rn(e2, b2);
    const double r = __dadd_rn(e3, b3);
    p0 = m;
    x0 = pick4(v, m);
    if (r > 0.0) {
      p1 = count_le(e1, e2, e3, __dmul_rn(u, r));
      x1 = copysign(r, pick4(v, p1));
    } else {
      p1 = m == 0 ? 1 : 0;
      x1 = 0.0;
    }
  } else {
    const double h = __dmul_rn(s, 0.5);
    const double q1 = __dmul_rn(u, h);
    const double q2 = __dadd_rn(q1, h);
    p0 = count_le(c1, c2, c3, q1);
    p1 = count_le(c1, c2, c3, q2);
    if (p1 == p0) {
      // Only a rounded cumulative sum puts both points in one entry: the second
      // goes to the next nonzero entry after it, else the last nonzero one before.
      int nxt = -1, prv = -1;
#pragma unroll
      for (int j = 3; j >= 0; --j)
        if (j > p0 && a[j] > 0.0) nxt = j;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j < p0 && a[j] > 0.0) prv = j;
      p1 = nxt >= 0 ? nxt : prv;
    }
    x0 = copysign(h, pick4(v, p0));
    x1 = copysign(h, pick4(v, p1));
  }
  if (p0 > p1) {
    pa = p1; pb = p0; xa = x1; xb = x0;
  } else {
    pa = p0; pb = p1; xa = x0; xb = x1;
  }
}

template <bool BF16>
__device__ __forceinline__ uint32_t mvue_bits(double x) {
  const float f = __double2float_rn(x);
  if (BF16) return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
  return (uint32_t)__half_as_ushort(__float2half_rn(f));
}

template <bool BF16>
__device__ __forceinline__ double half_bits_to_f64(uint32_t b) {
  if (BF16) return (double)__uint_as_float(b << 16);
  return (double)__half2float(__ushort_as_half((unsigned short)b));
}

template <bool BF16>
__global__ void __launch_bounds__(kMvueThreads) mvue_sparsify_kernel(
    const uint16_t *__restrict__ dy, int64_t T, int64_t N, int64_t ldy, uint64_t seed, uint64_t offset,
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

  const int w = tid >> 5, p = tid & 31;
  const int64_t tseg = t0 + 32 * w;                         // first token of this thread's segment
  const int ngroups = (int)max((int64_t)0, min((int64_t)8, (T - tseg) / 4));
  const int rh = (int)(blockIdx.y & 1);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int64_t n = n0 + 2 * p + c;
    uint32_t nib = 0x44444444u;                             // padding: positions 0, 1
    if (n < N && ngroups > 0) {
      uint64_t ctr[4] = {(uint64_t)(tseg >> 5), (uint64_t)n, 0ull, 0ull};
      philox4x64_10(ctr, seed, offset);
      uint32_t packed[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < ngroups) {
          const uint64_t word = ctr[j >> 1];
          const uint32_t u32 = (uint32_t)(word >> (32 * (j & 1)));
          const double u = (double)(u32 >> 8) * 0x1p-24;
          double v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = half_bits_to_f64<BF16>((s_tile[32 * w + 4 * j + i][p] >> (16 * c)) & 0xFFFFu);
          int pa, pb;
          double xa, xb;
          mvue_group(v, u, pa, pb, xa, xb);
          nib = (nib & ~(0xFu << (4 * j))) | ((uint32_t)(pa | (pb << 2)) << (4 * j));
          packed[j] = mvue_bits<BF16>(xa) | (mvue_bits<BF16>(xb) << 16);
        } else {
          packed[j] = 0u;
        }
      }
      uint16_t *dst = vals + n * (T >> 1) + (tseg >> 1);
      *reinterpret_cast<uint4 *>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      if (ngroups > 4) *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    }
    // Metadata: row r of the chunk, K step w; groups 0-3 go to lane
    // (r % 8) + 16 (r / 16), groups 4-7 to that lane + 8; the 16-bit half is (r / 8) % 2.
    const int r = 64 * rh + 2 * p + c;
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
