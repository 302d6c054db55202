// 2:4 sparse FFN GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Accelerating Transformer Pre-training with 2:4 Sparsity", reproducibility
// table, Software Dependencies row (2:4 sparse matrix multiplications) and the
// abstract (transposable masks make the input-gradient product 2:4 as well).
//
// One kernel serves the FFN products.  With A the 2:4-compressed operand
// [M x Kd] (2 of every 4 values along Kd kept) and B = activations [T x Kd]:
//     out[T x M] = B * A^T
//   forward:        A = W   [N x K] compressed along K,  B = X  -> Y  [T x N]
//   input gradient: A = W^T [K x N] compressed along N,  B = dY -> dX [T x K]
// The sparse operand must be the MMA's A operand, so the tensor-memory tile is
// out^T (lane = output feature, column = token); each epilogue thread owns one
// feature and writes it for consecutive tokens of row-major out.
// The weight-gradient variant (EPI = kEpiWgrad) contracts over tokens instead:
// A = MVUE(dY^T) [N x T] compressed along T (or, dense, dY^T), B = the layer
// input [T x K] read as stored (MN-major), out = dW [N x K] fp32 in the natural
// orientation (see PairGeom and the weight-gradient epilogue).  The same kernel
// with SPARSE = false runs the dense fine-tuning products.
//
// CTA pairs (clusters of 2, tcgen05 cta_group::2).  A pair computes a tile of
// 256 output features x N tokens (N = 240 or 224; 224 only where the epilogue's
// staging leaves no room for 240, or, for variants built both ways, where the
// host finds the waves fuller at 224; see PairGeom): each CTA holds 128 rows of the compressed
// operand and N/2 token rows of the activations in its own shared memory, and
// the pair's even (leader) CTA issues MMAs of M = 256, N, K = 32 that read
// both.  At N = 240, per CTA and 128-wide K step this moves 48 KB (A 16 KB,
// B 30 KB, metadata 2 KB) for 7.9 MFLOP dense-equivalent; a single-CTA
// 128 x 128 tile moves 50 KB for 4.2 MFLOP and is bound by the latency of its
// L2 -> SM stream.
// Persistent: each pair walks tiles pair, pair + npairs, ... (feature tiles
// fastest, so the pairs running at once share token tiles through L2).
//
// Warps: 0 = TMA producer (both CTAs), 1 = TMEM allocation and, in the leader,
// the MMA issuer, 2-13 = epilogue: three groups of four warps take alternate
// 16-token chunks (warp w may read TMEM lanes 32*(w%4)..+31 only, so each group
// covers the four lane quadrants).  Each epilogue warp works alone, with no
// cross-warp barrier: TMEM -> registers (two adjacent tokens of one feature
// per thread) -> packed 16-bit pairs -> stmatrix.trans into its own staging
// tile [16 tokens x 32 features] -> one TMA store per chunk and output.
// Shared memory: a 4-stage ring of {A 128x64 kept values, B (N/2)x128 as two
// boxes (both 128B-swizzled), the 2 KB metadata chunk}, then 1 KB staging
// tiles per epilogue warp (out; + aux for GELU; two pre-activation tiles for
// dGELU).
// Tensor memory per CTA: two N-column fp32 accumulators (tile i+1 runs its
// MMAs while tile i drains) and 4 metadata columns per stage.
// Protocol:
//   - both producers TMA-load their halves, counting bytes on the leader's
//     `full` barrier (the leader alone arms it with the pair's byte count);
//   - the leader's MMA thread moves both metadata chunks into tensor memory
//     (tcgen05.cp over the pair), issues the MMAs, and commits to `empty` and
//     `acc_full` of both CTAs;
//   - every epilogue warp of both CTAs arrives once on the leader's
//     `acc_empty` when it has read its last chunk of a tile.
// The dGELU epilogue TMA-loads its pre-activation tiles two chunks ahead (the
// first two before waiting for the accumulator, so the main loop hides them).
// No load uses cluster multicast; each CTA reads its own tiles.
// Every wait is bounded; a wait that runs out records a timeout in the device
// error word, raises the CTA's abort flag, and the CTA drains and exits.
#pragma once
#include "sp24_common.cuh"
#include "sp24_tables.cuh"

namespace sp24 {

#ifndef SP24_EPI_WARPS
#define SP24_EPI_WARPS 12
#endif
constexpr int kEpiWarps = SP24_EPI_WARPS;              // epilogue warps: kEpiWarps / 4 per TMEM lane quadrant
static_assert(kEpiWarps == 8 || kEpiWarps == 12, "two or three epilogue warps per lane quadrant");
constexpr int kEpiGroups = kEpiWarps / 4;              // warp groups taking alternate chunks
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kSmemE = 2048;                           // metadata chunk (128 rows x 128 columns)
constexpr int kEpiTokens = 16;                         // tokens per epilogue chunk
constexpr int kTmemCols = 512;
constexpr uint64_t kDrainBudget = 1ull << 26;

constexpr int kPairRows = 128;                         // compressed-operand rows per CTA
constexpr int kPairSmemA = kPairRows * 64 * 2;        // 16 KB: 128 rows x 64 values (128B swizzle)
constexpr int kPairBNWide = 240;                       // tokens per pair tile where shared memory allows
constexpr int kPairBNNarrow = 224;                     // else

// Epilogues: none; GELU (aux <- pre-activation); GELU' (aux = pre-activation,
// read); gated GELU on a gate/up-interleaved output (out = gelu(gate) * up at
// half width, aux <- both pre-activations); and its input gradient (aux =
// both pre-activations, read; out = (d gate, d up) interleaved at twice the
// accumulator width).
// The weight gradient (wgrad) is its own variant: A = the MVUE-sparsified dY^T
// [N x T], B = the layer input [T x K] read MN-major, out = dW [N x K] fp32 in
// the natural orientation (see PairGeom and the wgrad epilogue below).
// Derivative-saving pair: the forward writes gelu'(acc) as aux, so the input
// gradient only multiplies by it (out = acc * aux); the same product as
// GELU / GELU', with the derivative rounded to the dtype instead of the
// pre-activation.
enum : int {
  kEpiNone = 0, kEpiGelu = 1, kEpiDgelu = 2, kEpiGeglu = 3, kEpiDgeglu = 4, kEpiWgrad = 5, kEpiGeluDeriv = 6,
  kEpiMulAux = 7,
  // The derivative-saving pair with the derivative in the packed chunk layout
  // (below): written and read straight from registers, no staging tile.
  kEpiGeluDerivPacked = 8,
  kEpiMulAuxPacked = 9
};
// Packed chunk layout of a 16-bit [T x M] matrix: blocks of 16 tokens x 32
// features (1 KB), block (t / 16, m / 32) at element offset
// ((t / 16) * ceil(M / 32) + m / 32) * 512.  Inside a block, half h (features
// 16h .. 16h + 15) is 512 bytes; lane l's 16 bytes at 16 l hold the four 32-bit
// registers i = 0..3 of the epilogue fragment: tokens 8 (i / 2) + 2 (l % 4) + {0, 1}
// (low, high half) of feature 16 h + 8 (i % 2) + l / 4.  A warp's fragment of one
// chunk is then two 512-byte runs, stored and loaded with 16-byte accesses.
constexpr int kGegluGroup = 16;   // rows of W_gate, then of W_up, alternate in the stacked gated weight

// Pipeline stage of the 2:4 GEMM (SPARSE) and of the dense GEMM of the dense
// fine-tuning phase.  Sparse: 128 logical K per stage = 64 kept values of A,
// two 64-K boxes of B and the 2 KB metadata chunk (46 KB), 4 stages (3 when
// the gated-GELU gradient epilogue takes 6 KB of staging per warp).  Dense:
// 64 K per stage, one box of A and one of B (30 KB), 6 stages.
//
// Weight gradient (EPI == kEpiWgrad, sparse): pair tiles of 256 rows of dW x
// 256 columns.  B comes from the row-major layer input [T x K] (K contiguous),
// i.e. MN-major for the MMA: per stage each CTA loads two 128B-swizzled atoms
// of 64 columns x 128 tokens (16 KB each; atom a of CTA r holds columns
// 128r + 64a .. +63 of the tile), so a stage is 50 KB and 4 stages fit.  Each
// 32-token K step issues one MMA of N = 256 (each CTA's 128 columns, its two
// atoms one descriptor stride apart).  One 256-column accumulator (no double
// buffering: the weight-gradient tiles run one per pair at the FFN sizes).
// The dense variant (dense fine-tuning) takes A = dY [T x N] as stored, read
// MN-major like B (two 8 KB atoms of 64 rows of dW x 64 tokens), 64 tokens per
// stage: A 16 KB + two 8 KB atoms of B, 6 stages; each 16-token K step issues
// one dense MMA of N = 256.  (Tiles of 128 dW columns with double-buffered
// accumulators were measured 10-15% slower at the 1.5B shapes, although they
// leave fewer column-waves idle: each stage then carries half the MMA work for
// the same A tile and per-stage overhead.)
constexpr int kEpiBufBytes = kEpiTokens * 32 * 2;      // staging tile: 16 tokens x 32 features, 64B-swizzled
constexpr int kPairBarBytes = 512;                     // mbarriers, TMEM address, abort flag

// Staging per epilogue warp, in 1 KB tiles: out; out + pre-activation; out +
// two pre-activation inputs; gated: half-width out (in a 1 KB tile) +
// pre-activations; gated gradient: a 2 KB out tile + two 2 KB pre-activation
// inputs.
__host__ __device__ constexpr int epi_bufs(int epi) {
  return epi == kEpiWgrad ? 0
                          : (epi == kEpiNone || epi == kEpiGeluDerivPacked || epi == kEpiMulAuxPacked) ? 1
                          : (epi == kEpiGelu || epi == kEpiGeglu || epi == kEpiGeluDeriv) ? 2
                          : ((epi == kEpiDgelu || epi == kEpiMulAux) ? 3 : 6);
}

// Tokens per pair tile (kBN): with WIDE, 240 where the shared memory still
// holds the same number of stages, else 224 (the host picks WIDE per call: the
// wider tile is cheaper per token but can leave a wave less full).  TMEM holds two accumulators of kBN columns and 4
// metadata columns per stage (2 x 240 + 16 = 496 of 512).  240 = 15 chunks of
// 16 tokens, five per epilogue warp group; 240 tokens per pair are 120 B rows
// per CTA, a 15 KB box (a whole number of 1 KB swizzle atoms).
template <bool SPARSE, int EPI, bool WIDE = true>
struct PairGeom {
  static constexpr bool kWg = EPI == kEpiWgrad;
  static constexpr int kBK = SPARSE ? 128 : 64;          // logical K per stage
  static constexpr int kAcols = 64;                      // A values per row and stage
  static constexpr int kBBoxes = (SPARSE || kWg) ? 2 : 1;  // wgrad: two 64-column atoms
  static constexpr int kMeta = SPARSE ? kSmemE : 0;
  static constexpr int kStages = SPARSE ? (EPI == kEpiDgeglu ? 3 : 4) : (EPI == kEpiDgeglu ? 4 : 6);
  static constexpr int kAccBufs = kWg ? 1 : 2;
  __host__ __device__ static constexpr int box_bytes(int bn) { return kWg ? 64 * kBK * 2 : (bn / 2) * 64 * 2; }
  __host__ __device__ static constexpr int smem_for(int bn) {
    return kStages * (kPairSmemA + kBBoxes * box_bytes(bn) + kMeta) + kEpiWarps * epi_bufs(EPI) * kEpiBufBytes +
           kPairBarBytes + 1024 + (kWg ? 8192 : 0);
  }
  static constexpr int kBN = kWg ? 256 : ((WIDE && smem_for(kPairBNWide) <= 232448) ? kPairBNWide : kPairBNNarrow);
  static constexpr int kBBoxBytes = box_bytes(kBN);      // one B box (or wgrad atom)
  static constexpr int kStageBytes = kPairSmemA + kBBoxes * kBBoxBytes + kMeta;
  static constexpr int kChunks = kBN / kEpiTokens;       // 16-token epilogue chunks per tile
  static constexpr int kMetaCol = kAccBufs * kBN;        // metadata columns after the accumulators
};
// The wgrad variant keeps 8 KB unused after its barriers, so that its MN-major
// B reads stay inside the allocation under any reading of the descriptor strides.
template <bool SPARSE, int EPI, bool WIDE = true>
__host__ __device__ constexpr int pair_smem_bytes() {
  return PairGeom<SPARSE, EPI, WIDE>::smem_for(PairGeom<SPARSE, EPI, WIDE>::kBN);
}
static_assert(pair_smem_bytes<true, kEpiMulAux>() == pair_smem_bytes<true, kEpiDgelu>() &&
                  pair_smem_bytes<false, kEpiMulAux>() == pair_smem_bytes<false, kEpiDgelu>() &&
                  pair_smem_bytes<true, kEpiGeluDeriv>() == pair_smem_bytes<true, kEpiGelu>(),
              "the derivative-saving pair stages like GELU / GELU'");
static_assert(PairGeom<true, kEpiNone>::kBN == 240 && PairGeom<true, kEpiGeluDeriv>::kBN == 240 &&
                  PairGeom<true, kEpiMulAux>::kBN == 224 && PairGeom<false, kEpiMulAux>::kBN == 240,
              "tile widths of the headline variants");
static_assert(pair_smem_bytes<true, kEpiDgelu>() <= 232448 && pair_smem_bytes<false, kEpiDgelu>() <= 232448 &&
                  pair_smem_bytes<true, kEpiDgeglu>() <= 232448 && pair_smem_bytes<false, kEpiDgeglu>() <= 232448 &&
                  pair_smem_bytes<true, kEpiWgrad>() <= 232448,
              "shared memory per CTA");
static_assert(pair_smem_bytes<false, kEpiWgrad>() <= 232448, "shared memory per CTA (dense wgrad)");

// The producer loads A and two B atoms (and, sparse, the metadata chunk) per stage of a
// weight-gradient pipeline: the stage, and the byte count armed on its barrier, hold all of them.
static_assert(PairGeom<true, kEpiWgrad>::kStageBytes == kPairSmemA + 2 * (64 * 128 * 2) + kSmemE &&
                  PairGeom<false, kEpiWgrad>::kStageBytes == kPairSmemA + 2 * (64 * 64 * 2),
              "wgrad stage = A + two B atoms (+ metadata)");
static_assert(PairGeom<true, kEpiWgrad>::kStageBytes % 1024 == 0 && PairGeom<true, kEpiWgrad>::kBBoxBytes % 1024 == 0 &&
                  PairGeom<false, kEpiWgrad>::kStageBytes % 1024 == 0 &&
                  PairGeom<false, kEpiWgrad>::kBBoxBytes % 1024 == 0,
              "128B-swizzled tiles need 1 KB aligned starts");
static_assert(PairGeom<true, kEpiWgrad>::kMetaCol + 4 * PairGeom<true, kEpiWgrad>::kStages <= kTmemCols,
              "tensor memory budget (wgrad)");
static_assert(PairGeom<true, kEpiNone>::kStageBytes % 1024 == 0 && PairGeom<false, kEpiNone>::kStageBytes % 1024 == 0 &&
                  PairGeom<true, kEpiMulAux>::kStageBytes % 1024 == 0 && kPairSmemA % 1024 == 0 &&
                  PairGeom<true, kEpiNone>::kBBoxBytes % 1024 == 0 && PairGeom<true, kEpiMulAux>::kBBoxBytes % 1024 == 0,
              "128B-swizzled tiles need 1 KB aligned starts");
static_assert(PairGeom<true, kEpiNone>::kMetaCol + 4 * PairGeom<true, kEpiNone>::kStages <= kTmemCols &&
                  PairGeom<true, kEpiDgeglu>::kMetaCol + 4 * PairGeom<true, kEpiDgeglu>::kStages <= kTmemCols,
              "tensor memory budget");
static_assert(2 * PairGeom<false, kEpiNone>::kStages + 16 + 2 * kEpiWarps <= kPairBarBytes / 8, "barrier space");

// Work schedule of a CTA pair: a sequence of segments (tile, K steps kb..ke-1).
// Data-parallel (every GEMM): pair p takes tiles p, p + P, p + 2P, ... over all
// num_kt K steps, so the P pairs of a wave walk K in step and share each K
// window of both operands in L2.  Split tail (the weight gradient, when
// `split` > 1): the full waves stay data-parallel, and the r = tiles mod P
// tiles of the last wave are cut along K into `split` (<= P / r) parts of
// num_kt / split steps; part j of tail tile i goes to pair i * split + j.  The
// pair holding part 0 (K steps from 0) adds the other parts' partial
// accumulators, written by pairs i * split + 1 .. i * split + split - 1 while it
// runs its own part, and stores the tile.
struct PairSchedule {
  int tile, pair, npairs, num_tiles, num_kt, split, full_tiles;
  bool tail_taken;
  __device__ PairSchedule(int sp, int p, int np, int tiles, int kt)
      : tile(p), pair(p), npairs(np), num_tiles(tiles), num_kt(kt), split(sp),
        full_tiles(sp > 1 ? (tiles / np) * np : tiles), tail_taken(false) {}
  __device__ bool next(int &t, int &kb, int &ke) {
    if (tile < full_tiles) {
      t = tile;
      kb = 0;
      ke = num_kt;
      tile += npairs;
      return true;
    }
    if (split > 1 && !tail_taken) {
      tail_taken = true;
      if (pair < (num_tiles - full_tiles) * split) {
        const int part = pair % split;
        t = full_tiles + pair / split;
        kb = part * num_kt / split;
        ke = (part + 1) * num_kt / split;
        return true;
      }
    }
    return false;
  }
};

// Partial accumulator of one CTA of a split tail tile (128 rows x 256 columns of dW, fp32):
// per epilogue warp, its 16-column chunks as [chunk][row half][8-column block]
// [lane] float4s, the registers of tmem_ld_16x256b_x2 as loaded, so the CTA
// that adds it reads back exactly what the same warp and lane of its own
// accumulator hold.  Ready counters: one per epilogue warp, raised by 1 per
// lane with release semantics once the lane's stores are issued.
constexpr int kWgChunksPerWarp = (256 / 16 + kEpiGroups - 1) / kEpiGroups;
constexpr int kMaxSplit = 8;   // parts of a split tail tile (part 0 adds the others one after another)
constexpr int64_t kSkPartFloatsPerCta = (int64_t)kEpiWarps * kWgChunksPerWarp * 4 * 32 * 4;

// GELU (exact erf form) and its derivative for the epilogues:
//   gelu(x) = x Phi(x),  gelu'(x) = Phi(x) + x phi(x),
//   Phi(x) = 1 - erfc(x/sqrt2)/2 (x >= 0),  erfc(|x|/sqrt2)/2 (x < 0),
//   phi(x) = exp(-x^2/2) / sqrt(2 pi).
// erfc(z) = exp(-z^2) R(z) with R(z) = erfc(z) exp(z^2); R is evaluated with a
// degree-12 polynomial in u = z/2 - 1 from a Chebyshev least-squares fit on
// z in [0, 4] (csrc/fit_gelu_poly.py derives the coefficients; the fp32 Horner
// evaluation stays within 9.1e-6 relative of R there).  The tail is thus
// accurate to ~1e-5 relative on both sides of 0, far inside the fp16/bf16
// output rounding; beyond z = 4 (|x| > 5.66) z is clamped for R only, where
// exp(-z^2) < 1.2e-7 makes the tail vanish against 1 or round to 0.  One
// exponential serves both Phi and phi; the sign cases fold into a max and a
// fused multiply-add, so the epilogue spends ~20 instructions per element.
// 2^y with the hardware's approximate base-2 exponential (relative error ~2^-22).
__device__ __forceinline__ float ex2_approx(float y) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
  return r;
}

// The epilogue evaluates elements in pairs (two adjacent tokens of one
// feature) with the packed f32x2 FMA path: every add, multiply and fused
// multiply-add below is the IEEE fp32 operation on each lane, two results per
// instruction.
__device__ __forceinline__ float2 splat(float v) { return make_float2(v, v); }

// R(z)/2 at z = min(|x|, 4 sqrt 2) / sqrt 2, in u = z/2 - 1 (the fitted
// coefficients scaled by 1/2, exact).
__device__ __forceinline__ float2 half_r2(float2 ax) {
  const float2 zc = make_float2(fminf(ax.x, 5.65685424949238f), fminf(ax.y, 5.65685424949238f));
  const float2 u = __ffma2_rn(zc, splat(0.353553390593274f), splat(-1.0f));
  float2 r = splat(1.858228817e-03f);
  r = __ffma2_rn(r, u, splat(-3.360528732e-03f));
  r = __ffma2_rn(r, u, splat(5.786734400e-04f));
  r = __ffma2_rn(r, u, splat(-1.290832530e-03f));
  r = __ffma2_rn(r, u, splat(8.399816230e-03f));
  r = __ffma2_rn(r, u, splat(-1.360862422e-02f));
  r = __ffma2_rn(r, u, splat(1.851560920e-02f));
  r = __ffma2_rn(r, u, splat(-2.878958545e-02f));
  r = __ffma2_rn(r, u, splat(4.359827935e-02f));
  r = __ffma2_rn(r, u, splat(-6.190539895e-02f));
  r = __ffma2_rn(r, u, splat(8.360114695e-02f));
  r = __ffma2_rn(r, u, splat(-1.067943201e-01f));
  r = __ffma2_rn(r, u, splat(1.276978850e-01f));
  return r;
}

// exp(-x^2/2) = 2^(-x^2 log2(e) / 2)
__device__ __forceinline__ float2 gauss_e2(float2 x) {
  const float2 a = __fmul2_rn(x, __fmul2_rn(x, splat(-0.721347520444482f)));
  return make_float2(ex2_approx(a.x), ex2_approx(a.y));
}

// gelu(x) = x Phi(x) = max(x, 0) - |x| t with t = erfc(|x|/sqrt2)/2 = e R/2.
__device__ __forceinline__ float2 gelu2(float2 x) {
  const float2 ax = make_float2(fabsf(x.x), fabsf(x.y));
  const float2 t = __fmul2_rn(half_r2(ax), gauss_e2(x));
  return __ffma2_rn(make_float2(-ax.x, -ax.y), t, make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f)));
}

// gelu'(x) = Phi(x) + x phi(x) with phi = e / sqrt(2 pi):
//   x <  0:  t - |x| phi      = e (R/2 - |x|/sqrt(2 pi))
//   x >= 0:  1 - t + |x| phi  = 1 - e (R/2 - |x|/sqrt(2 pi))
// (both give 1/2 at x = 0, so -0 may take either side).
__device__ __forceinline__ float2 gelu_grad2(float2 x) {
  const float2 ax = make_float2(fabsf(x.x), fabsf(x.y));
  const float2 e = gauss_e2(x);
  const float2 q = __ffma2_rn(make_float2(-ax.x, -ax.y), splat(0.39894228040143268f), half_r2(ax));
  const bool p0 = x.x >= 0.0f, p1 = x.y >= 0.0f;
  return __ffma2_rn(make_float2(p0 ? -e.x : e.x, p1 ? -e.y : e.y), q, make_float2(p0 ? 1.0f : 0.0f, p1 ? 1.0f : 0.0f));
}

// gelu and gelu' of the same pair, sharing the exponential and the polynomial
// (each result is computed exactly as gelu2 and gelu_grad2 compute it).
__device__ __forceinline__ void gelu_and_grad2(float2 x, float2 &g, float2 &gp) {
  const float2 ax = make_float2(fabsf(x.x), fabsf(x.y));
  const float2 nax = make_float2(-ax.x, -ax.y);
  const float2 e = gauss_e2(x);
  const float2 hr = half_r2(ax);
  g = __ffma2_rn(nax, __fmul2_rn(hr, e), make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f)));
  const float2 q = __ffma2_rn(nax, splat(0.39894228040143268f), hr);
  const bool p0 = x.x >= 0.0f, p1 = x.y >= 0.0f;
  gp = __ffma2_rn(make_float2(p0 ? -e.x : e.x, p1 ? -e.y : e.y), q, make_float2(p0 ? 1.0f : 0.0f, p1 ? 1.0f : 0.0f));
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

// 32 lanes x 16 consecutive 32-bit columns.
// 16 TMEM lanes x 16 columns (two 16x256b blocks).  Thread t receives, for
// column block i (registers 4i..4i+3): lane t/4 at columns 8i + 2(t%4) + {0, 1},
// then lane t/4 + 8 at the same two columns.
__device__ __forceinline__ void tmem_ld_16x256b_x2(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

// After tmem_wait_ld, reg_fence on the loaded registers keeps every use of
// them below the wait.  Makes the compiler treat the registers as redefined
// here (emits nothing).
__device__ __forceinline__ void reg_fence(uint32_t (&r)[8]) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]));
}

// Four 8x8 16-bit matrices, transposed on the way: register j of thread t
// holds row t/4, columns 2(t%4) and 2(t%4)+1 of matrix j; lane 8j + r gives
// the shared address of (stored) row r of matrix j.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t saddr, const uint32_t (&r)[4]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t saddr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr)
               : "memory");
}

// Byte offset of 16-byte column c of row `row` in a 64B-swizzled tile of
// 64-byte rows (the TMA's 64B pattern: the column index is XORed with row/2 mod 4).
__host__ __device__ constexpr uint32_t swz64(int row, int c) {
  return (uint32_t)(row * 64 + ((c ^ ((row >> 1) & 3)) << 4));
}

// The same for 128-byte rows and the TMA's 128B pattern (column index XOR row mod 8).
__host__ __device__ constexpr uint32_t swz128(int row, int c) {
  return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4));
}

// Two floats -> one register of 16-bit values, lo in the low half (round to nearest even).
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t d;
  if (BF16) asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  else asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

template <bool BF16>
__device__ __forceinline__ void unpack2(uint32_t v, float &lo, float &hi) {
  if (BF16) {
    lo = __uint_as_float(v << 16);
    hi = __uint_as_float(v & 0xFFFF0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&v));
    lo = f.x;
    hi = f.y;
  }
}

template <bool BF16, int EPI, bool SPARSE, bool WIDE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    sp24_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_meta, const __grid_constant__ CUtensorMap tm_out,
                          const __grid_constant__ CUtensorMap tm_aux, int M, int T, int num_kt,
                          uint64_t wait_budget, float *__restrict__ out_f32, int64_t ld_out,
                          const uint16_t *__restrict__ dec_w, const uint8_t *__restrict__ dec_idx,
                          float dec_lambda, float *__restrict__ sk_part, unsigned *__restrict__ sk_flags,
                          int sk_split, int cols_fastest, int a_mn, uint16_t *__restrict__ aux_packed,
                          int aux_nbf) {
  // T counts the B operand's rows of the output: tokens, or for the weight
  // gradient the columns of dW (out_f32 [M x T], leading dimension ld_out).
  // Weight gradient with dec_w set: the masked decay of dW in the epilogue, W and
  // its pattern indices dec_idx [M/4][T/4] in the layout of dW (see below).
  // Weight gradient with cols_fastest set: tiles are numbered along dW's
  // columns first, so a wave of pairs shares the row tiles' A operand (chosen
  // when A is the larger operand, which each wave would otherwise read again).
  // Weight gradient with sk_part set: the split-tail schedule with sk_split
  // parts per tail tile, partial accumulators in sk_part (kSkPartFloatsPerCta
  // per CTA) and ready counters in sk_flags (kEpiWarps per CTA, zero at launch
  // and left zero).
  // Packed-derivative epilogues: aux_packed in the packed chunk layout with
  // aux_nbf = ceil(M / 32) feature blocks per token block.
  // Dense with a_mn set: A is read as stored [K x M] (M contiguous), MN-major
  // like the dense weight gradient's A: the input gradient takes W itself.
  using G = PairGeom<SPARSE, EPI, WIDE>;
  constexpr bool WG = G::kWg;
  constexpr int kPairStages = G::kStages;
  constexpr int kPairStageBytes = G::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stage_base = smem;
  uint8_t *epi_smem = smem + kPairStages * kPairStageBytes;   // staging tiles, 1 KB aligned
  uint64_t *bars = reinterpret_cast<uint64_t *>(epi_smem + kEpiWarps * epi_bufs(EPI) * kEpiBufBytes);
  uint64_t *full = bars;                          // [stages] leader: TMA (both CTAs) -> MMA
  uint64_t *empty = bars + kPairStages;           // [stages] MMA -> this CTA's TMA
  uint64_t *acc_full = bars + 2 * kPairStages;    // [2] MMA -> this CTA's epilogue
  uint64_t *acc_empty = acc_full + 2;             // [2] leader: both epilogues -> MMA
  uint64_t *drain = acc_empty + 2;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
  uint64_t *aux_bars = bars + 2 * kPairStages + 8;  // [kEpiWarps][2] dGELU pre-activation tiles

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool is_leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_mt = (M + 2 * kPairRows - 1) / (2 * kPairRows);
  const int num_row_tiles = (M + kPairRows - 1) / kPairRows;
  const int num_nt = (T + G::kBN - 1) / G::kBN;
  const int num_tiles = num_mt * num_nt;
  const bool by_cols = WG && cols_fastest != 0;
  auto tile_mt = [&](int t) { return by_cols ? t / num_nt : t % num_mt; };
  auto tile_nt = [&](int t) { return by_cols ? t % num_nt : t / num_mt; };
  const int split = (WG && sk_part != nullptr) ? sk_split : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    if (EPI == kEpiDgelu || EPI == kEpiDgeglu || EPI == kEpiMulAux)
      for (int i = 0; i < 2 * kEpiWarps; ++i) mbar_init(&aux_bars[i], 1);
    *s_abort = 0;
    fence_mbarrier_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    if (SPARSE) prefetch_tensormap(&tm_meta);
    prefetch_tensormap(&tm_out);
    if (EPI != kEpiNone) prefetch_tensormap(&tm_aux);
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or byte count
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  pdl_launch_dependents();
  pdl_wait();  // the previous kernel's outputs (operands, pre-activations) are complete

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ producer (both CTAs)
    uint32_t g = 0;
    bool ok = true;
    PairSchedule sched(split, pair, npairs, num_tiles, num_kt);
    int tile, kb, ke;
    while (ok && sched.next(tile, kb, ke)) {
      const int mt = tile_mt(tile);
      const int a_row = mt * 2 * kPairRows + (int)rank * kPairRows;
      const int b_row = tile_nt(tile) * G::kBN + (int)rank * (WG ? 128 : G::kBN / 2);
      // A pair tile past the last 128-row tile reads zero rows (TMA fill); give
      // it the last real metadata chunk so every code the MMA sees is valid.
      const int chunk_row = min(2 * mt + (int)rank, num_row_tiles - 1) * num_kt;
      for (int kt = kb; kt < ke; ++kt, ++g) {
        const int s = (int)(g % kPairStages);
        if (!mbar_wait_bounded(&empty[s], ((g / kPairStages) & 1u) ^ 1u, wait_budget, s_abort)) {
          ok = false;
          break;
        }
        uint8_t *st = stage_base + s * kPairStageBytes;
        if (is_leader) mbar_arrive_expect_tx(&full[s], 2 * kPairStageBytes);
        if (!SPARSE && (WG || a_mn)) {
          // Dense A read as stored, MN-major, in two 64-row atoms 8 KB apart
          // (x = output row, y = K): dY for the weight gradient, W for the input
          // gradient.
          tma_load_2d_pair(st, &tm_a, &full[s], a_row, kt * G::kBK);
          tma_load_2d_pair(st + kPairSmemA / 2, &tm_a, &full[s], a_row + 64, kt * G::kBK);
        } else {
          tma_load_2d_pair(st, &tm_a, &full[s], kt * G::kAcols, a_row);
        }
        if (WG) {
          // MN-major atoms: x = dW column (b_row, b_row + 64), y = token.
          tma_load_2d_pair(st + kPairSmemA, &tm_b, &full[s], b_row, kt * G::kBK);
          if (G::kBBoxes == 2)
            tma_load_2d_pair(st + kPairSmemA + G::kBBoxBytes, &tm_b, &full[s], b_row + 64, kt * G::kBK);
        } else {
          tma_load_2d_pair(st + kPairSmemA, &tm_b, &full[s], kt * G::kBK, b_row);
          if (SPARSE) tma_load_2d_pair(st + kPairSmemA + G::kBBoxBytes, &tm_b, &full[s], kt * G::kBK + 64, b_row);
        }
        if (SPARSE)
          tma_load_2d_pair(st + kPairSmemA + G::kBBoxes * G::kBBoxBytes, &tm_meta, &full[s], 0, chunk_row + kt);
      }
    }
    // The leader's `full` barriers count both CTAs' bytes: let every copy land.
    if (is_leader) {
      for (uint32_t i = g > kPairStages ? g - kPairStages : 0; i < g; ++i) {
        volatile int no_abort = 0;
        mbar_wait_bounded(&full[i % kPairStages], (i / kPairStages) & 1u, kDrainBudget, &no_abort);
      }
    }
  } else if (warp == 1 && lane == 0 && is_leader) {
    // ----------------------------------------------------- MMA issuer (leader)
    // Descriptors of stage 0; stage s and K step kk only move the 14-bit start
    // address field (all of shared memory is below 2^18 bytes, so it never carries).
    // wgrad: one MMA of N = 256 per K step, B MN-major (instruction descriptor
    // bit 16): each CTA holds 128 of the tile's columns as two 64-column atoms,
    // and the B descriptor's leading field is the atom stride (kBBoxBytes), its
    // stride field the 1024 bytes between 8-token groups.
    // Dense wgrad: A MN-major too (bit 15); its descriptor's leading field is the
    // 8 KB between its two 64-row atoms, its stride field the 1024 bytes between
    // 8-token groups.
    constexpr uint32_t idesc = WG ? ((SPARSE ? make_idesc_sparse(BF16, 2 * kPairRows, 256)
                                             : (make_idesc_dense(BF16, 2 * kPairRows, 256) | (1u << 15))) |
                                    (1u << 16))
                               : SPARSE ? make_idesc_sparse(BF16, 2 * kPairRows, G::kBN)
                                        : make_idesc_dense(BF16, 2 * kPairRows, G::kBN);
    // Dense input gradient with a_mn: the same MN-major A as the dense wgrad (bit 15).
    const uint32_t idesc_amn = idesc | (1u << 15);
    const uint64_t a_desc0 =
        smem_desc(smem_u32(stage_base), (!SPARSE && (WG || a_mn)) ? kPairSmemA / 2 : 16, 1024, kSwizzle128B);
    const uint64_t b_desc0 =
        smem_desc(smem_u32(stage_base + kPairSmemA), WG ? G::kBBoxBytes : 16, 1024, kSwizzle128B);
    const uint64_t e_desc0 =
        smem_desc(smem_u32(stage_base + kPairSmemA + G::kBBoxes * G::kBBoxBytes), 128, 128, kSwizzleNone);
    uint32_t g = 0;
    bool ok = true;
    int j = 0;
    PairSchedule sched(split, pair, npairs, num_tiles, num_kt);
    int tile, kb, ke;
    for (; ok && sched.next(tile, kb, ke); ++j) {
      const int b = j % G::kAccBufs;
      const uint32_t use = (uint32_t)(j / G::kAccBufs);
      if (!(ok = mbar_wait_bounded(&acc_empty[b], (use & 1u) ^ 1u, wait_budget, s_abort))) break;
      tc_fence_after();
      const uint32_t acc = tmem_base + (uint32_t)(b * G::kBN);
      for (int kt = kb; kt < ke; ++kt, ++g) {
        const int s = (int)(g % kPairStages);
        if (!(ok = mbar_wait_bounded(&full[s], (g / kPairStages) & 1u, wait_budget, s_abort))) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((s * kPairStageBytes) >> 4);
        const uint64_t ad = a_desc0 + so, bd = b_desc0 + so;
        if (WG && !SPARSE) {
          // Dense weight gradient: K step kk of 16 tokens moves A and B 16 tokens
          // (2048 bytes) each; atom 1 of B sits 8 KB after atom 0.
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kt != kb || kk != 0) ? 1u : 0u;
            tc_mma_f16_pair(acc, ad + (uint64_t)(kk * (2048 >> 4)), bd + (uint64_t)(kk * (2048 >> 4)), idesc, accum);
          }
        } else if (WG) {
          const uint32_t t_meta = tmem_base + G::kMetaCol + 4 * s;
          tc_cp_128x128b_pair(t_meta, e_desc0 + so);
          // K step kk: A advances 32 bytes along its swizzled rows, B 32 tokens
          // (4096 bytes); atom 1 of B sits 16 KB after atom 0.
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t tm = t_meta + 2 * (kk >> 1);
            const uint32_t id = idesc | (uint32_t)(kk & 1);
            const uint32_t accum = (kt != kb || kk != 0) ? 1u : 0u;
            tc_mma_sp_f16_pair(acc, ad + 2 * kk, bd + (uint64_t)(kk * (4096 >> 4)), tm, id, accum);
          }
        } else if (SPARSE) {
          const uint32_t t_meta = tmem_base + G::kMetaCol + 4 * s;
          tc_cp_128x128b_pair(t_meta, e_desc0 + so);
          // The metadata operand address must be 2-column aligned; the low column
          // bit travels in the descriptor's sparsity-selector field instead.
          tc_mma_sp_f16_pair(acc, ad, bd, t_meta, idesc, kt != kb ? 1u : 0u);
          tc_mma_sp_f16_pair(acc, ad + 2, bd + 4, t_meta, idesc | 1u, 1u);
          tc_mma_sp_f16_pair(acc, ad + 4, bd + (G::kBBoxBytes >> 4), t_meta + 2, idesc, 1u);
          tc_mma_sp_f16_pair(acc, ad + 6, bd + (G::kBBoxBytes >> 4) + 4, t_meta + 2, idesc | 1u, 1u);
        } else if (a_mn) {
          // A MN-major: a K = 16 step moves A 16 rows of 128 bytes (2048 bytes) and
          // B 32 bytes along its swizzled rows.
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_f16_pair(acc, ad + (uint64_t)(kk * (2048 >> 4)), bd + 2 * kk, idesc_amn,
                            (kt != kb || kk != 0) ? 1u : 0u);
        } else {
          // Four K = 16 steps through the 128-byte swizzled rows of A and B (32 bytes each).
          tc_mma_f16_pair(acc, ad, bd, idesc, kt != kb ? 1u : 0u);
          tc_mma_f16_pair(acc, ad + 2, bd + 2, idesc, 1u);
          tc_mma_f16_pair(acc, ad + 4, bd + 4, idesc, 1u);
          tc_mma_f16_pair(acc, ad + 6, bd + 6, idesc, 1u);
        }
        tc_commit_pair(&empty[s], 0x3);
      }
      if (ok) tc_commit_pair(&acc_full[b], 0x3);
    }
    if (!ok) {
      tc_commit_pair(drain, 0x1);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, kDrainBudget, &no_abort);
    }
  } else if (warp >= 2 && WG) {
    // ------------------------------------------ weight-gradient epilogue (both CTAs)
    // Warp w drains TMEM lanes 32q..32q+31 (q = w%4; rows of dW) at the 16-column
    // chunks grp, grp + kEpiGroups, ... of the accumulator, three chunks per
    // round trip.  Register layout of tmem_ld_16x256b_x2: thread t holds row
    // t/4 (+8) at columns 2(t%4), +1 of each 8-column block, so each float2
    // store of a warp writes 8 rows x 32 contiguous bytes (whole sectors of dW).
    // Masked decay (dec_w set): the two entries of a store that the mask of W
    // prunes become fmaf(lambda, W, acc), the fp32 operation of the separate
    // decay pass on the stored gradient, so both give the same bits.  The
    // accumulator is not double-buffered here, so W's values and keep bits of
    // all of a warp's stores are loaded before it waits for the tile, while the
    // main loop still runs.
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;
    constexpr int kChunks = G::kBN / 16;
    constexpr int kPerWarp = (kChunks + kEpiGroups - 1) / kEpiGroups;
    constexpr int kBatch = 2;
    static_assert(!WG || kPerWarp == kWgChunksPerWarp, "split-tail partial layout");
    const int64_t idx_cols = ld_out >> 2;
    const int ew = warp - 2;
    // Split tail: this CTA's partial slot and counter; the CTA of the same rank in
    // pair p + d uses slot and counter blockIdx.x + 2d.
    float4 *part_own = split > 1 ? reinterpret_cast<float4 *>(sk_part + (int64_t)blockIdx.x * kSkPartFloatsPerCta) +
                                       (int64_t)ew * kPerWarp * 4 * 32 + lane
                                 : nullptr;
    unsigned *flag_own = split > 1 ? sk_flags + (int64_t)blockIdx.x * kEpiWarps + ew : nullptr;
    int j = 0;
    PairSchedule sched(split, pair, npairs, num_tiles, num_kt);
    int tile, kbeg, kend;
    for (; sched.next(tile, kbeg, kend); ++j) {
      const bool to_part = kbeg > 0;                   // a later part of a split tile: another pair stores it
      const bool merge = kbeg == 0 && kend < num_kt;   // part 0: pairs p + 1 .. p + split - 1 hold the rest
      const bool decay = dec_w != nullptr && !to_part;
      const int m0 = tile_mt(tile) * 2 * kPairRows + (int)rank * kPairRows + 32 * q;
      const int n0 = tile_nt(tile) * G::kBN;
      // Decay operands of the warp's stores in this tile: W's two values (one
      // 32-bit word) and their two keep bits; entries outside dW keep both.
      uint32_t wv[kPerWarp][8], kb[kPerWarp];
      if (decay) {
#pragma unroll
        for (int kc = 0; kc < kPerWarp; ++kc) {
          const int ch = grp + kc * kEpiGroups;
          kb[kc] = 0xFFFFu;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int h = e >> 2, i = (e >> 1) & 1, sub = e & 1;
            const int row = m0 + 16 * h + 8 * sub + (lane >> 2);
            const int col = n0 + 16 * ch + 8 * i + 2 * (lane & 3);
            wv[kc][e] = 0u;
            if (ch < kChunks && row < M && col < T) {
              wv[kc][e] = __ldg(reinterpret_cast<const uint32_t *>(dec_w + (int64_t)row * ld_out + col));
              const uint32_t pat = __ldg(dec_idx + (int64_t)(row >> 2) * idx_cols + (col >> 2));
              const uint32_t two = ((uint32_t)g_tables.bits[pat] >> (4 * (row & 3) + (col & 3))) & 3u;
              kb[kc] = (kb[kc] & ~(3u << (2 * e))) | (two << (2 * e));
            }
          }
        }
      }
      const int ab = j % G::kAccBufs;   // accumulator buffer of this tile
      const bool got = mbar_wait_bounded(&acc_full[ab], (uint32_t)(j / G::kAccBufs) & 1u, wait_budget, s_abort);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      if (merge) {
        // The other parts of this tile: all 32 lanes of the same warp of each
        // have released their stores (the parts run side by side in the last
        // wave).  Each lane then acquires every counter itself.
        bool ready = true;
        if (lane == 0)
          for (int d = 1; d < split && ready; ++d)
            ready = flag_wait_bounded(flag_own + 2 * d * kEpiWarps, 32u, wait_budget, s_abort);
        if (!__shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0)) break;
        for (int d = 1; d < split; ++d) (void)flag_load_acquire(flag_own + 2 * d * kEpiWarps);
      }
      const uint32_t t_base = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * G::kBN);
#pragma unroll
      for (int k0 = 0; k0 < kPerWarp; k0 += kBatch) {
        uint32_t r[kBatch][2][8];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
          const int ch = grp + (k0 + k) * kEpiGroups;
          if (ch < kChunks) {
            tmem_ld_16x256b_x2(t_base + (uint32_t)(16 * ch), r[k][0]);
            tmem_ld_16x256b_x2(t_base + (16u << 16) + (uint32_t)(16 * ch), r[k][1]);
          }
        }
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
          reg_fence(r[k][0]);
          reg_fence(r[k][1]);
        }
        // Part 0 of a split tile: its own sum, then parts 1, 2, ... in order (fp32
        // additions into the loaded accumulator), a chunk's four loads at a time.
        if (merge) {
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            if (grp + (k0 + k) * kEpiGroups >= kChunks) break;
            for (int d = 1; d < split; ++d) {
              const float4 *src = part_own + 2 * d * kSkPartFloatsPerCta / 4 + (k0 + k) * 4 * 32;
              float4 pv[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) pv[e] = __ldcg(src + e * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint32_t *a = &r[k][e >> 1][4 * (e & 1)];
                a[0] = __float_as_uint(__fadd_rn(__uint_as_float(a[0]), pv[e].x));
                a[1] = __float_as_uint(__fadd_rn(__uint_as_float(a[1]), pv[e].y));
                a[2] = __float_as_uint(__fadd_rn(__uint_as_float(a[2]), pv[e].z));
                a[3] = __float_as_uint(__fadd_rn(__uint_as_float(a[3]), pv[e].w));
              }
            }
          }
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
          const int ch = grp + (k0 + k) * kEpiGroups;
          if (ch >= kChunks) break;
          if (to_part) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int i = 0; i < 2; ++i)
                part_own[((k0 + k) * 4 + 2 * h + i) * 32] =
                    make_float4(__uint_as_float(r[k][h][4 * i]), __uint_as_float(r[k][h][4 * i + 1]),
                                __uint_as_float(r[k][h][4 * i + 2]), __uint_as_float(r[k][h][4 * i + 3]));
            continue;
          }
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
              for (int sub = 0; sub < 2; ++sub) {
                const int row = m0 + 16 * h + 8 * sub + (lane >> 2);
                const int col = n0 + 16 * ch + 8 * i + 2 * (lane & 3);
                float2 v = make_float2(__uint_as_float(r[k][h][4 * i + 2 * sub]),
                                       __uint_as_float(r[k][h][4 * i + 2 * sub + 1]));
                if (decay && k0 + k < kPerWarp) {
                  const int e = 4 * h + 2 * i + sub;
                  const uint32_t two = kb[k0 + k] >> (2 * e);
                  if (!(two & 1u)) v.x = fmaf(dec_lambda, bits_to_f32<BF16>(wv[k0 + k][e] & 0xFFFFu), v.x);
                  if (!(two & 2u)) v.y = fmaf(dec_lambda, bits_to_f32<BF16>(wv[k0 + k][e] >> 16), v.y);
                }
                if (row < M && col < T) *reinterpret_cast<float2 *>(out_f32 + (int64_t)row * ld_out + col) = v;
              }
        }
      }
      if (to_part) flag_add_release(flag_own, 1u);   // this lane's partial stores are issued
      if (merge) {
        __syncwarp();   // every lane has read the partials: the counters return to zero for the next launch
        if (lane == 0)
          for (int d = 1; d < split; ++d) flag_store_relaxed(flag_own + 2 * d * kEpiWarps, 0u);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader(&acc_empty[ab]);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------- epilogue (both CTAs)
    // Warp w reads TMEM lane quadrant q = w%4 (features 32q..32q+31 of this
    // CTA's rows) and takes the 16-token chunks grp, grp + kEpiGroups, ...
    // (grp = (w-2)/4) of every tile.  It issues all its TMEM loads of a tile
    // at once and returns the accumulator to the MMA after one round trip; the
    // math, packing and stores then overlap the next tiles' main loop.
    // Decisions after a bounded wait are made per warp (__all_sync), so the
    // .sync.aligned instructions stay convergent.
    const int ew = warp - 2;
    const int grp = ew >> 2;
    const int q = warp & 3;
    constexpr int kMaxChunksPerWarp = (G::kChunks + kEpiGroups - 1) / kEpiGroups;
    constexpr bool kPre = EPI == kEpiDgelu || EPI == kEpiDgeglu || EPI == kEpiMulAux;   // TMA-loaded aux tiles
    constexpr int kPreBytes = EPI == kEpiDgeglu ? 2 * kEpiBufBytes : kEpiBufBytes;
    constexpr int kOutBytes = EPI == kEpiDgeglu ? 2 * kEpiBufBytes : kEpiBufBytes;
    // Staging of warp ew: [out][aux] (GELU, gated), [out][pre 0][pre 1] (gradients).
    uint8_t *stg = epi_smem + ew * epi_bufs(EPI) * kEpiBufBytes;
    const uint32_t stg_u32 = smem_u32(stg);
    uint64_t *pre_bar = aux_bars + 2 * ew;
    // stmatrix/ldmatrix addressing: lane l names row l%8 of matrix l/8; matrix
    // j holds tokens 8(j/2).. and features 8(j%2).. (+16 for the upper 16 TMEM lanes).
    const int mrow = 8 * (lane >> 4) + (lane & 7);
    const int mcol = (lane >> 3) & 1;
    const uint32_t lane_off0 = swz64(mrow, mcol);
    const uint32_t lane_off1 = swz64(mrow, 2 + mcol);
    // Columns (features) of this warp in out and aux: the gated output has half
    // the accumulator's width, the gated gradient twice it.
    auto out_col = [&](int m0) { return EPI == kEpiGeglu ? m0 / 2 : (EPI == kEpiDgeglu ? 2 * m0 : m0); };
    auto pre_col = [&](int m0) { return EPI == kEpiDgeglu ? 2 * m0 : m0; };
    auto release = [&](int buf) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader(&acc_empty[buf]);
    };
    uint32_t pre_issued = 0, pre_used = 0;   // pre-activation tiles (tile s uses buffer s%2)
    auto pre_load = [&](int x, int y) {
      const uint32_t seq = pre_issued++;
      if (lane == 0) {
        uint64_t *bar = &pre_bar[seq & 1];
        mbar_arrive_expect_tx(bar, kPreBytes);
        tma_load_2d(stg + kOutBytes + kPreBytes * (seq & 1), &tm_aux, bar, x, y);
      }
    };
    // This lane's 16 bytes of half 0 of the packed block holding chunk (t0, m0);
    // half 1 is 256 elements further.
    auto packed_at = [&](int t0, int m0) {
      return aux_packed + ((((size_t)(t0 >> 4) * (size_t)aux_nbf + (size_t)(m0 >> 5)) << 9) + 8 * (size_t)lane);
    };
    uint4 pk_cur[2], pk_nxt[2];   // MulAuxPacked: this chunk's and the next chunk's derivative
    auto packed_load = [&](int t0, int m0, uint4 (&v)[2]) {
      if (m0 < M) {
        const uint16_t *src = packed_at(t0, m0);
        v[0] = __ldg(reinterpret_cast<const uint4 *>(src));
        v[1] = __ldg(reinterpret_cast<const uint4 *>(src + 256));
      } else {
        v[0] = v[1] = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    bool alive = true;
    int j = 0;
    for (int tile = pair; tile < num_tiles && alive; tile += npairs, ++j) {
      const int b = j & 1;
      const int m0 = (tile % num_mt) * 2 * kPairRows + (int)rank * kPairRows + 32 * q;
      const int n0 = (tile / num_mt) * G::kBN;
      const int nchunks = min(G::kChunks, (T - n0 + kEpiTokens - 1) / kEpiTokens);
      const int nk = grp < nchunks ? (nchunks - 1 - grp) / kEpiGroups + 1 : 0;   // this warp's chunks
      if (kPre)
        for (int k = 0; k < 2 && k < nk; ++k) pre_load(pre_col(m0), n0 + (grp + k * kEpiGroups) * kEpiTokens);
      if (EPI == kEpiMulAuxPacked && nk > 0) packed_load(n0 + grp * kEpiTokens, m0, pk_nxt);
      const bool got = mbar_wait_bounded(&acc_full[b], (uint32_t)(j >> 1) & 1u, wait_budget, s_abort);
      if (!__all_sync(0xFFFFFFFFu, got)) {
        alive = false;
        break;
      }
      tc_fence_after();
      uint32_t r[kMaxChunksPerWarp][2][8];
      const uint32_t t_base = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * G::kBN);
#pragma unroll
      for (int k = 0; k < kMaxChunksPerWarp; ++k) {
        if (k < nk) {
          const uint32_t col = (uint32_t)((grp + k * kEpiGroups) * kEpiTokens);
          tmem_ld_16x256b_x2(t_base + col, r[k][0]);
          tmem_ld_16x256b_x2(t_base + (16u << 16) + col, r[k][1]);
        }
      }
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < kMaxChunksPerWarp; ++k) {
        reg_fence(r[k][0]);
        reg_fence(r[k][1]);
      }
      release(b);
#pragma unroll
      for (int k = 0; k < kMaxChunksPerWarp; ++k) {
        if (k >= nk) break;
        const int t0 = n0 + (grp + k * kEpiGroups) * kEpiTokens;
        uint32_t pre_src = 0;
        if (kPre) {
          const uint32_t seq = pre_used;
          const bool ready = mbar_wait_bounded(&pre_bar[seq & 1], (seq >> 1) & 1u, wait_budget, s_abort);
          if (!__all_sync(0xFFFFFFFFu, ready)) {
            alive = false;
            break;
          }
          ++pre_used;
          pre_src = stg_u32 + kOutBytes + kPreBytes * (seq & 1);
        }
        // The staging tiles are rewritten only once the previous chunk's TMA
        // stores have read them: the gated epilogues wait here, the others after
        // their arithmetic (which then overlaps those reads).
        auto staging_free = [&]() {
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
        };
        if (EPI == kEpiGeglu || EPI == kEpiDgeglu) staging_free();
        if (EPI == kEpiMulAuxPacked) {
          pk_cur[0] = pk_nxt[0];
          pk_cur[1] = pk_nxt[1];
          if (k + 1 < nk) packed_load(t0 + kEpiGroups * kEpiTokens, m0, pk_nxt);   // one chunk ahead
        }
        // Register i of half h: tokens 8(i/2) + 2(lane%4) + {0, 1} of feature
        // 16h + 8(i%2) + lane/4 (TMEM registers 4(i/2) + 2(i%2) + {0, 1}).
        if (EPI == kEpiGeglu) {
          // Half 0 holds the gate rows, half 1 the up rows of the same 16
          // features: out = gelu(gate) * up [16 tokens x 16 features, 32-byte
          // rows], aux <- both halves as accumulated.
          uint32_t po[4], pa[2][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int ri = 4 * (i >> 1) + 2 * (i & 1);
            const float2 g = make_float2(__uint_as_float(r[k][0][ri]), __uint_as_float(r[k][0][ri + 1]));
            const float2 u = make_float2(__uint_as_float(r[k][1][ri]), __uint_as_float(r[k][1][ri + 1]));
            const float2 y = __fmul2_rn(gelu2(g), u);
            po[i] = pack2<BF16>(y.x, y.y);
            pa[0][i] = pack2<BF16>(g.x, g.y);
            pa[1][i] = pack2<BF16>(u.x, u.y);
          }
          stmatrix_x4_trans(stg_u32 + (uint32_t)(mrow * 32 + mcol * 16), po);
          stmatrix_x4_trans(stg_u32 + kEpiBufBytes + lane_off0, pa[0]);
          stmatrix_x4_trans(stg_u32 + kEpiBufBytes + lane_off1, pa[1]);
        } else if (EPI == kEpiDgeglu) {
          // The pre-activation tile is [16 tokens x 64 columns, 128B-swizzled]:
          // the gate and up values of the warp's 32 features, in 16-column
          // groups gate(h=0), up(h=0), gate(h=1), up(h=1).  The output has the
          // same layout: (d gate, d up) = (acc * up * gelu'(gate), acc * gelu(gate)).
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t hg[4], hu[4], og[4], ou[4];
            ldmatrix_x4_trans(pre_src + swz128(mrow, 4 * h + mcol), hg);
            ldmatrix_x4_trans(pre_src + swz128(mrow, 4 * h + 2 + mcol), hu);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int ri = 4 * (i >> 1) + 2 * (i & 1);
              const float2 a = make_float2(__uint_as_float(r[k][h][ri]), __uint_as_float(r[k][h][ri + 1]));
              float2 g, u, gel, gp;
              unpack2<BF16>(hg[i], g.x, g.y);
              unpack2<BF16>(hu[i], u.x, u.y);
              gelu_and_grad2(g, gel, gp);
              const float2 dg = __fmul2_rn(__fmul2_rn(a, u), gp);
              const float2 du = __fmul2_rn(a, gel);
              og[i] = pack2<BF16>(dg.x, dg.y);
              ou[i] = pack2<BF16>(du.x, du.y);
            }
            stmatrix_x4_trans(stg_u32 + swz128(mrow, 4 * h + mcol), og);
            stmatrix_x4_trans(stg_u32 + swz128(mrow, 4 * h + 2 + mcol), ou);
          }
        } else {
          uint32_t hx[2][4];
          if (EPI == kEpiDgelu || EPI == kEpiMulAux) {
            ldmatrix_x4_trans(pre_src + lane_off0, hx[0]);
            ldmatrix_x4_trans(pre_src + lane_off1, hx[1]);
          }
          if (EPI == kEpiMulAuxPacked) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              hx[h][0] = pk_cur[h].x;
              hx[h][1] = pk_cur[h].y;
              hx[h][2] = pk_cur[h].z;
              hx[h][3] = pk_cur[h].w;
            }
          }
          uint32_t po[2][4], pa[2][4];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int ri = 4 * (i >> 1) + 2 * (i & 1);
              const float2 acc = make_float2(__uint_as_float(r[k][h][ri]), __uint_as_float(r[k][h][ri + 1]));
              float2 y = acc;
              if (EPI == kEpiGelu) {
                y = gelu2(acc);
                pa[h][i] = pack2<BF16>(acc.x, acc.y);
              } else if (EPI == kEpiGeluDeriv || EPI == kEpiGeluDerivPacked) {
                float2 gp;
                gelu_and_grad2(acc, y, gp);
                pa[h][i] = pack2<BF16>(gp.x, gp.y);
              } else if (EPI == kEpiMulAux || EPI == kEpiMulAuxPacked) {
                float2 hv;
                unpack2<BF16>(hx[h][i], hv.x, hv.y);
                y = __fmul2_rn(acc, hv);
              } else if (EPI == kEpiDgelu) {
                float2 hv;
                unpack2<BF16>(hx[h][i], hv.x, hv.y);
                y = __fmul2_rn(acc, gelu_grad2(hv));
              }
              po[h][i] = pack2<BF16>(y.x, y.y);
            }
          }
          if (EPI == kEpiGeluDerivPacked && m0 < M) {   // the derivative, straight from registers
            uint16_t *dst = packed_at(t0, m0);
            *reinterpret_cast<uint4 *>(dst) = make_uint4(pa[0][0], pa[0][1], pa[0][2], pa[0][3]);
            *reinterpret_cast<uint4 *>(dst + 256) = make_uint4(pa[1][0], pa[1][1], pa[1][2], pa[1][3]);
          }
          staging_free();
          stmatrix_x4_trans(stg_u32 + lane_off0, po[0]);
          stmatrix_x4_trans(stg_u32 + lane_off1, po[1]);
          if (EPI == kEpiGelu || EPI == kEpiGeluDeriv) {
            stmatrix_x4_trans(stg_u32 + kEpiBufBytes + lane_off0, pa[0]);
            stmatrix_x4_trans(stg_u32 + kEpiBufBytes + lane_off1, pa[1]);
          }
        }
        // One proxy fence orders this warp's shared-memory accesses of the
        // chunk (the stmatrix writes, and for the gradients the ldmatrix reads
        // of the pre-activation tile) before the TMA store that reads the
        // staging tile and the TMA load that refills the pre-activation tile.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && m0 < M) {   // the TMA unit clips columns past the tensor and tokens >= T
          tma_store_2d(&tm_out, stg, out_col(m0), t0);
          if (EPI == kEpiGelu || EPI == kEpiGeglu || EPI == kEpiGeluDeriv)
            tma_store_2d(&tm_aux, stg + kEpiBufBytes, m0, t0);
          bulk_commit_group();
        }
        if (kPre && k + 2 < nk) pre_load(pre_col(m0), t0 + 2 * kEpiGroups * kEpiTokens);
      }
    }
    if (lane == 0) {
      bulk_wait_group<0>();
      // After an abort, let the pre-activation loads still in flight land.
      for (uint32_t seq = pre_used; seq < pre_issued; ++seq) {
        volatile int no_abort = 0;
        mbar_wait_bounded(&pre_bar[seq & 1], (seq >> 1) & 1u, kDrainBudget, &no_abort);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's MMAs, copies and arrivals into this CTA are over
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace sp24
