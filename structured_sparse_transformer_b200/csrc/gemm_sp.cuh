// 2:4 sparse FFN GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Accelerating Transformer Pre-training with 2:4 Sparsity", reproducibility
// table, Software Dependencies row (2:4 sparse matrix multiplications) and the
// abstract (transposable masks make the input-gradient product 2:4 as well).
//
// One kernel serves both products.  With A the 2:4-compressed operand
// [M x Kd] (2 of every 4 values along Kd kept) and B = activations [T x Kd]:
//     out[T x M] = B * A^T
//   forward:        A = W   [N x K] compressed along K,  B = X  -> Y  [T x N]
//   input gradient: A = W^T [K x N] compressed along N,  B = dY -> dX [T x K]
// The sparse operand must be the MMA's A operand, so each CTA computes a
// transposed tile out^T[128 x BN] in tensor memory (lane = output feature,
// column = token) and the epilogue transposes it through shared memory into a
// TMA store of row-major out.
//
// CTA = 6 warps: warp 0 issues TMA loads, warp 1 allocates TMEM and issues the
// MMAs (one elected thread), warps 2-5 run the epilogue.  A 4-stage ring holds,
// per 128-wide logical K step: A (128 x 64 kept values, 128B swizzle),
// B (BN x 128, two 128B-swizzled boxes) and the 2 KB metadata chunk, which
// tcgen05.cp moves into 4 TMEM columns before the four K=32 sparse MMAs of the
// step read it.  Every wait is bounded; a wait that runs out records a timeout
// in the device error word and the CTA drains its copies and exits.
#pragma once
#include "sp24_common.cuh"

namespace sp24 {

constexpr int kGemmBM = 128;             // output features per CTA (MMA M)
constexpr int kGemmBN = 128;             // tokens per CTA (MMA N)
constexpr int kGemmBK = 128;             // logical K per pipeline stage
constexpr int kGemmBKc = kGemmBK / 2;    // kept values per stage and row
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kSmemA = kGemmBM * kGemmBKc * 2;          // 16 KB
constexpr int kSmemBBox = kGemmBN * 64 * 2;             // one 128-byte-wide box
constexpr int kSmemB = 2 * kSmemBBox;                   // 32 KB
constexpr int kSmemE = 2048;                            // metadata chunk
constexpr int kStageBytes = kSmemA + kSmemB + kSmemE;
constexpr int kEpiTokens = 32;                          // tokens per epilogue store
constexpr int kSmemOut = kEpiTokens * kGemmBM * 2;      // 8 KB staging
constexpr int kTmemCols = 256;                          // accumulator 128 + metadata 16
constexpr int kTmemMetaCol = kGemmBN;
constexpr int kGemmSmemBytes = kGemmStages * kStageBytes + 2 * kSmemOut + 256 + 1024;
constexpr uint64_t kDrainBudget = 1ull << 26;

enum : int { kEpiNone = 0, kEpiGelu = 1, kEpiDgelu = 2 };

__device__ __forceinline__ float gelu_f(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

__device__ __forceinline__ float gelu_grad_f(float x) {
  return 0.5f * (1.0f + erff(x * 0.70710678118654752f)) + x * expf(-0.5f * x * x) * 0.39894228040143268f;
}

template <bool BF16>
__device__ __forceinline__ uint32_t f32_to_bits(float x) {
  if (BF16) return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
  return (uint32_t)__half_as_ushort(__float2half_rn(x));
}

template <bool BF16>
__device__ __forceinline__ float bits_to_f32(uint32_t b) {
  if (BF16) return __uint_as_float(b << 16);
  return __half2float(__ushort_as_half((unsigned short)b));
}

template <bool BF16, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    sp24_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_aux,
                     const uint8_t *__restrict__ meta, const uint16_t *__restrict__ aux_in, int M, int T,
                     int num_kt, uint64_t wait_budget) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stage_base = smem;
  uint16_t *s_out = reinterpret_cast<uint16_t *>(smem + kGemmStages * kStageBytes);
  uint16_t *s_aux = s_out + kSmemOut / 2;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kGemmStages * kStageBytes + 2 * kSmemOut);
  uint64_t *full = bars;                       // [kGemmStages]
  uint64_t *empty = bars + kGemmStages;        // [kGemmStages]
  uint64_t *acc_full = bars + 2 * kGemmStages;
  uint64_t *drain = acc_full + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = blockIdx.x;
  const int m0 = mt * kGemmBM;
  const int n0 = blockIdx.y * kGemmBN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbarrier_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    int issued = 0;
    for (int kt = 0; kt < num_kt; ++kt) {
      const int s = kt % kGemmStages;
      const uint32_t it = (uint32_t)(kt / kGemmStages);
      if (!mbar_wait_bounded(&empty[s], (it & 1u) ^ 1u, wait_budget, s_abort)) break;
      uint8_t *st = stage_base + s * kStageBytes;
      mbar_arrive_expect_tx(&full[s], kStageBytes);
      tma_load_2d(st, &tm_a, &full[s], kt * kGemmBKc, m0);
      tma_load_2d(st + kSmemA, &tm_b, &full[s], kt * kGemmBK, n0);
      tma_load_2d(st + kSmemA + kSmemBBox, &tm_b, &full[s], kt * kGemmBK + 64, n0);
      bulk_load(st + kSmemA + kSmemB, meta + ((size_t)mt * num_kt + kt) * kSmemE, kSmemE, &full[s]);
      ++issued;
    }
    // Let every copy this thread started land before the CTA can exit.
    for (int kt = issued > kGemmStages ? issued - kGemmStages : 0; kt < issued; ++kt) {
      volatile int no_abort = 0;
      mbar_wait_bounded(&full[kt % kGemmStages], (uint32_t)(kt / kGemmStages) & 1u, kDrainBudget, &no_abort);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc_sparse(BF16, kGemmBM, kGemmBN);
    bool ok = true;
    for (int kt = 0; kt < num_kt && ok; ++kt) {
      const int s = kt % kGemmStages;
      const uint32_t it = (uint32_t)(kt / kGemmStages);
      ok = mbar_wait_bounded(&full[s], it & 1u, wait_budget, s_abort);
      if (!ok) break;
      tc_fence_after();
      const uint8_t *st = stage_base + s * kStageBytes;
      const uint32_t a_addr = smem_u32(st);
      const uint32_t b_addr = smem_u32(st + kSmemA);
      const uint32_t e_addr = smem_u32(st + kSmemA + kSmemB);
      const uint32_t t_meta = tmem_base + kTmemMetaCol + 4 * s;
      tc_cp_128x128b(t_meta, smem_desc(e_addr, 128, 128, kSwizzleNone));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t adesc = smem_desc(a_addr + kk * 32, 16, 1024, kSwizzle128B);
        const uint64_t bdesc = smem_desc(b_addr + (kk >> 1) * kSmemBBox + (kk & 1) * 64, 16, 1024, kSwizzle128B);
        tc_mma_sp_f16(tmem_base, adesc, bdesc, t_meta + kk, idesc, (kt | kk) != 0 ? 1u : 0u);
      }
      tc_commit(&empty[s]);
    }
    if (ok) {
      tc_commit(acc_full);
    } else {
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, kDrainBudget, &no_abort);
    }
  } else if (warp >= 2) {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quadrant this warp may access
    const int m_local = 32 * q + lane;
    const int m = m0 + m_local;
    const bool leader = threadIdx.x == 64;
    if (mbar_wait_bounded(acc_full, 0, wait_budget, s_abort)) {
      tc_fence_after();
      for (int c = 0; c < kGemmBN / kEpiTokens; ++c) {
        const int t0 = n0 + c * kEpiTokens;
        if (t0 >= T) break;
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(c * kEpiTokens), r);
        tmem_wait_ld();
        if (leader) bulk_wait_group_read<0>();
        named_barrier_sync(1, 128);
#pragma unroll
        for (int j = 0; j < kEpiTokens; ++j) {
          const float acc = __uint_as_float(r[j]);
          float out = acc;
          if (EPI == kEpiGelu) {
            s_aux[j * kGemmBM + m_local] = (uint16_t)f32_to_bits<BF16>(acc);
            out = gelu_f(acc);
          } else if (EPI == kEpiDgelu) {
            const int t = t0 + j;
            const float pre = (t < T && m < M) ? bits_to_f32<BF16>(aux_in[(size_t)t * M + m]) : 0.0f;
            out = acc * gelu_grad_f(pre);
          }
          s_out[j * kGemmBM + m_local] = (uint16_t)f32_to_bits<BF16>(out);
        }
        fence_proxy_async_smem();
        named_barrier_sync(1, 128);
        if (leader) {
          tma_store_2d(&tm_out, s_out, m0, t0);
          if (EPI == kEpiGelu) tma_store_2d(&tm_aux, s_aux, m0, t0);
          bulk_commit_group();
        }
      }
      if (leader) bulk_wait_group<0>();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace sp24
