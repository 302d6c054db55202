// libsp24: host side of the C ABI declared in include/sp24.h.
//
// Every entry point validates its arguments on the host first (nothing is
// launched when a check fails), then enqueues its kernels on the caller's
// stream.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "sp24.h"
#include "gemm_sp.cuh"
#include "mask_kernels.cuh"
#include "mvue.cuh"

namespace {

using namespace sp24;

std::atomic<uint64_t> g_wait_budget{1ull << 32};

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_dtype(sp24_dtype d) { return d == SP24_F16 || d == SP24_BF16; }

sp24_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SP24_ERR_NO_DEVICE; }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return SP24_ERR_NO_DEVICE;
  }
  return major == 10 ? SP24_OK : SP24_ERR_NO_DEVICE;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while its predecessor in the stream drains; each kernel here calls
// griddepcontrol.wait before its first global-memory access.
template <typename... KArgs, typename... Args>
sp24_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return SP24_ERR_CUDA;
  }
  return SP24_OK;
}

constexpr int kMaxDevices = 64;

// A value computed once per device (under std::call_once, so concurrent host
// threads and several devices in one process each see their own).
struct PerDevice {
  std::once_flag once[kMaxDevices];
  int value[kMaxDevices] = {};
};

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}

int sm_count() {
  static PerDevice cache;
  const int dev = current_device();
  if (dev < 0) return 148;
  std::call_once(cache.once[dev], [dev] {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cache.value[dev] = n;
  });
  return cache.value[dev];
}

// --------------------------------------------------------- tensor maps (TMA)

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major [outer x inner] array of 16-bit (or `type`) elements.
bool make_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t pitch_bytes,
                 uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle,
                 CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_UINT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- GEMM launch

// CTA-pair kernel: clusters of two CTAs, tiles of 256 rows x 240 or 224 tokens (see gemm_sp.cuh).
// SPARSE: A = kept values [M x Kd/2] + metadata chunks; dense: A = [M x Kd].
// Weight gradient (kEpiWgrad): B = the layer input [Kd tokens x T columns]
// read MN-major, out = fp32 [M x T]; tiles of 256 x 256.
// Per device, once: the shared-memory opt-in of an instantiation and the number
// of its CTA pairs that fit at once (0: the set-up failed; -1: no device).
template <bool BF16, int EPI, bool SPARSE, bool WIDE = false>
int gemm_pairs() {
  constexpr int smem_bytes = pair_smem_bytes<SPARSE, EPI, WIDE>();
  auto kernel = sp24_gemm_pair_kernel<BF16, EPI, SPARSE, WIDE>;
  static PerDevice pairs_cache;
  const int dev = current_device();
  if (dev < 0) return -1;
  std::call_once(pairs_cache.once[dev], [&] {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess) {
      cudaGetLastError();
      pairs_cache.value[dev] = 0;
      return;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)(sm_count() / 2));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = sm_count() / 2;
    }
    pairs_cache.value[dev] = n;
  });
  return pairs_cache.value[dev];
}

// Split-tail workspace of the weight gradient, one per (device, stream), so that
// launches on different streams never share one (launches on one stream run
// one after another): the partial accumulators and ready counters of every
// CTA of a full-width launch.  Allocated on first use and kept for the life of
// the process.  The counters start at zero and every launch that completes
// leaves them at zero; after a kernel gives up waiting, sp24_device_status
// clears them.
struct SkWorkspace {
  float *part = nullptr;
  unsigned *flags = nullptr;
  int ctas = 0;
};
std::mutex g_sk_mutex;
std::map<std::pair<int, cudaStream_t>, SkWorkspace> g_sk_workspaces;

sp24_status sk_workspace(cudaStream_t stream, int ctas, SkWorkspace *out) {
  const int dev = current_device();
  if (dev < 0) return SP24_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_sk_mutex);
  SkWorkspace &w = g_sk_workspaces[std::make_pair(dev, stream)];
  if (w.ctas < ctas) {
    // cudaFree waits for the device, so no earlier launch still uses the old buffers.
    if (w.part) cudaFree(w.part);
    if (w.flags) cudaFree(w.flags);
    w = SkWorkspace{};
    float *part = nullptr;
    unsigned *flags = nullptr;
    if (cudaMalloc(&part, (size_t)ctas * kSkPartFloatsPerCta * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&flags, (size_t)ctas * kEpiWarps * sizeof(unsigned)) != cudaSuccess ||
        cudaMemsetAsync(flags, 0, (size_t)ctas * kEpiWarps * sizeof(unsigned), stream) != cudaSuccess) {
      cudaGetLastError();
      if (part) cudaFree(part);
      if (flags) cudaFree(flags);
      return SP24_ERR_CUDA;
    }
    w.part = part;
    w.flags = flags;
    w.ctas = ctas;
  }
  *out = w;
  return SP24_OK;
}

// Zero the ready counters of every split-tail workspace of the current device
// (after a kernel gave up waiting, one may have been left raised).
sp24_status sk_clear_flags() {
  const int dev = current_device();
  if (dev < 0) return SP24_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_sk_mutex);
  if (cudaDeviceSynchronize() != cudaSuccess) return SP24_ERR_CUDA;
  for (auto &kv : g_sk_workspaces)
    if (kv.first.first == dev && cudaMemset(kv.second.flags, 0, (size_t)kv.second.ctas * kEpiWarps * sizeof(unsigned)) !=
                                     cudaSuccess)
      return SP24_ERR_CUDA;
  return SP24_OK;
}

// Fixed scratch of sp24_gemm_wgrad_noalloc, in the module's static device
// memory (zero at load): the split-tail partial sums of kNoAllocCtas CTAs, then
// their ready counters.
constexpr int kNoAllocCtas = 128;
constexpr size_t kNoAllocPartBytes = (size_t)kNoAllocCtas * kSkPartFloatsPerCta * sizeof(float);
constexpr size_t kNoAllocBytes = kNoAllocPartBytes + (size_t)kNoAllocCtas * kEpiWarps * sizeof(unsigned);
static_assert(kNoAllocPartBytes % 256 == 0, "counters start 256-byte aligned");
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Its address on the current device, looked up once per device (with that
// device current) and checked.
sp24_status noalloc_scratch(SkWorkspace *out) {
  static std::once_flag once[kMaxDevices];
  static void *addr[kMaxDevices];
  static cudaError_t err[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return SP24_ERR_NO_DEVICE;
  std::call_once(once[dev], [dev] {
    void *p = nullptr;
    err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err[dev] != cudaSuccess) cudaGetLastError();
    addr[dev] = p;
  });
  if (err[dev] != cudaSuccess || addr[dev] == nullptr) return SP24_ERR_CUDA;
  out->part = static_cast<float *>(addr[dev]);
  out->flags = reinterpret_cast<unsigned *>(static_cast<unsigned char *>(addr[dev]) + kNoAllocPartBytes);
  out->ctas = kNoAllocCtas;
  return SP24_OK;
}

// Weight gradient with decay: dec_w/dec_idx/dec_lambda (the masked decay of dW in
// the epilogue); null dec_w elsewhere.  `fixed`: a caller-given split-tail
// scratch (its counters are zeroed here before the launch) instead of the
// per-stream workspace; null for every entry point but sp24_gemm_wgrad_noalloc.
template <bool BF16, int EPI, bool SPARSE, bool WIDE>
sp24_status launch_gemm_pair_w(const void *B, int64_t T, int64_t Kd, const void *vals, const void *meta, int64_t M,
                               void *out, void *aux, cudaStream_t stream, const void *dec_w, const uint8_t *dec_idx,
                               float dec_lambda, const SkWorkspace *fixed, bool a_mn) {
  using G = PairGeom<SPARSE, EPI, WIDE>;
  const int num_kt = (int)((Kd + G::kBK - 1) / G::kBK);
  const int64_t row_tiles = (M + kPairRows - 1) / kPairRows;
  const uint64_t a_cols = SPARSE ? (uint64_t)(Kd / 2) : (uint64_t)Kd;
  CUtensorMap ta, tb, tm;
  const bool b_ok = G::kWg ? make_map_2d(&tb, B, (uint64_t)T, (uint64_t)Kd, (uint64_t)T * 2, 64, (uint32_t)G::kBK,
                                         CU_TENSOR_MAP_SWIZZLE_128B)
                           : make_map_2d(&tb, B, (uint64_t)Kd, (uint64_t)T, (uint64_t)Kd * 2, 64, (uint32_t)(G::kBN / 2),
                                         CU_TENSOR_MAP_SWIZZLE_128B);
  // Dense weight gradient (A = dY [Kd tokens x M]) and dense input gradient with
  // a_mn (A = W [Kd x M]): A read MN-major in 64 x kBK boxes.
  a_mn = a_mn && !SPARSE && !G::kWg;
  const bool a_ok = (G::kWg && !SPARSE) || a_mn
                        ? make_map_2d(&ta, vals, (uint64_t)M, (uint64_t)Kd, (uint64_t)M * 2, 64, (uint32_t)G::kBK,
                                      CU_TENSOR_MAP_SWIZZLE_128B)
                        : make_map_2d(&ta, vals, a_cols, (uint64_t)M, a_cols * 2, G::kAcols, kPairRows,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (!a_ok || !b_ok) return SP24_ERR_CUDA;
  if (SPARSE) {
    if (!make_map_2d(&tm, meta, kSmemE / 8, (uint64_t)(row_tiles * num_kt), kSmemE, kSmemE / 8, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_UINT64))
      return SP24_ERR_CUDA;
  } else {
    tm = ta;  // unused by the dense kernel
  }
  // Epilogue staging tiles of row-major out / aux, 16 tokens high: 32 features
  // (64B swizzle); gated: out 16 features (no swizzle), aux 32; gated
  // gradient: out and aux 64 columns (128B swizzle) over twice the width.
  CUtensorMap to, tx;
  bool maps_ok;
  if (G::kWg) {   // direct fp32 stores: no staging maps
    to = ta;
    tx = ta;
    maps_ok = true;
  } else if (EPI == kEpiGeglu) {
    maps_ok = make_map_2d(&to, out, (uint64_t)M / 2, (uint64_t)T, (uint64_t)M, 16, kEpiTokens, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map_2d(&tx, aux, (uint64_t)M, (uint64_t)T, (uint64_t)M * 2, 32, kEpiTokens, CU_TENSOR_MAP_SWIZZLE_64B);
  } else if (EPI == kEpiDgeglu) {
    maps_ok = make_map_2d(&to, out, (uint64_t)M * 2, (uint64_t)T, (uint64_t)M * 4, 64, kEpiTokens, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map_2d(&tx, aux, (uint64_t)M * 2, (uint64_t)T, (uint64_t)M * 4, 64, kEpiTokens, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    maps_ok = make_map_2d(&to, out, (uint64_t)M, (uint64_t)T, (uint64_t)M * 2, 32, kEpiTokens, CU_TENSOR_MAP_SWIZZLE_64B) &&
              make_map_2d(&tx, (EPI == kEpiNone || EPI == kEpiGeluDerivPacked || EPI == kEpiMulAuxPacked) ? out : aux,
                          (uint64_t)M, (uint64_t)T, (uint64_t)M * 2, 32, kEpiTokens, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (!maps_ok) return SP24_ERR_CUDA;
  constexpr int smem_bytes = pair_smem_bytes<SPARSE, EPI, WIDE>();
  auto kernel = sp24_gemm_pair_kernel<BF16, EPI, SPARSE, WIDE>;
  const int max_pairs = gemm_pairs<BF16, EPI, SPARSE, WIDE>();
  if (max_pairs <= 0) return max_pairs == 0 ? SP24_ERR_CUDA : SP24_ERR_NO_DEVICE;
  const int64_t tiles = ((M + 2 * kPairRows - 1) / (2 * kPairRows)) * ((T + G::kBN - 1) / G::kBN);
  const int pairs = (int)(tiles < max_pairs ? tiles : max_pairs);
  // Weight gradient: number the tiles along dW's columns first when the A
  // operand is the larger one (each wave of pairs then reads it once).
  const double a_bytes = (double)M * (double)Kd * (SPARSE ? 1.0 + 1.0 / 8 : 2.0);
  const double b_bytes = (double)Kd * (double)T * 2.0;
  const int cols_fastest = (G::kWg && a_bytes > b_bytes) ? 1 : 0;
  // Weight gradient: when the last wave would leave pairs idle, split its r
  // tiles along K into min(P / r, 8, num_kt) parts on all P pairs.
  SkWorkspace ws;
  int split = 1, grid_pairs = pairs;
  const int64_t tail = tiles % max_pairs;
  if (G::kWg && tail != 0) {
    int64_t s = max_pairs / tail < num_kt ? max_pairs / tail : num_kt;
    if (s > kMaxSplit) s = kMaxSplit;
    if (s > 1) {
      if (fixed) {   // CTAs 0 .. 2 tail s - 1 use their partial slots and counters
        const int64_t used = 2 * tail * s;
        if (used > fixed->ctas) return SP24_ERR_SCRATCH_TOO_SMALL;
        ws = *fixed;
        if (cudaMemsetAsync(ws.flags, 0, (size_t)used * kEpiWarps * sizeof(unsigned), stream) != cudaSuccess) {
          cudaGetLastError();
          return SP24_ERR_CUDA;
        }
      } else {
        const sp24_status st = sk_workspace(stream, 2 * max_pairs, &ws);
        if (st != SP24_OK) return st;
      }
      split = (int)s;
      grid_pairs = max_pairs;
    }
  }
  return launch_pdl(kernel, dim3(2 * grid_pairs), dim3(kGemmThreads), smem_bytes, stream, ta, tb, tm, to, tx, (int)M,
                    (int)T, num_kt, (uint64_t)g_wait_budget.load(), G::kWg ? static_cast<float *>(out) : nullptr,
                    (int64_t)(G::kWg ? T : 0), static_cast<const uint16_t *>(dec_w), dec_idx, dec_lambda, ws.part,
                    ws.flags, split, cols_fastest, a_mn ? 1 : 0,
                    (EPI == kEpiGeluDerivPacked || EPI == kEpiMulAuxPacked) ? static_cast<uint16_t *>(aux) : nullptr,
                    (int)((M + 31) / 32));
}

// Tile width per call, for the variants that have both: the busiest pair's token
// columns, ceil(tiles / pairs) x width, with the 240-token tile counted 5% cheaper
// per token (measured on the 1.5B FFN launches, where its waves are as full);
// where waves quantise differently (e.g. 148 tiles of 224 tokens on 74 pairs
// against 140 of 240) the narrower tile is kept.
template <bool BF16, int EPI, bool SPARSE>
sp24_status launch_gemm_pair_t(const void *B, int64_t T, int64_t Kd, const void *vals, const void *meta, int64_t M,
                               void *out, void *aux, cudaStream_t stream, const void *dec_w = nullptr,
                               const uint8_t *dec_idx = nullptr, float dec_lambda = 0.0f,
                               const SkWorkspace *fixed = nullptr, bool a_mn = false) {
  constexpr int kWideBN = PairGeom<SPARSE, EPI, true>::kBN, kNarrowBN = PairGeom<SPARSE, EPI, false>::kBN;
  if constexpr (kWideBN != kNarrowBN) {
    const int P = gemm_pairs<BF16, EPI, SPARSE, false>();
    if (P > 0) {
      const int64_t mt = (M + 2 * kPairRows - 1) / (2 * kPairRows);
      auto busiest = [&](int bn) {
        const int64_t tiles = mt * ((T + bn - 1) / bn);
        return (double)((tiles + P - 1) / P) * (double)bn;
      };
      if (busiest(kWideBN) * 0.95 < busiest(kNarrowBN))
        return launch_gemm_pair_w<BF16, EPI, SPARSE, true>(B, T, Kd, vals, meta, M, out, aux, stream, dec_w, dec_idx,
                                                           dec_lambda, fixed, a_mn);
    }
  }
  return launch_gemm_pair_w<BF16, EPI, SPARSE, false>(B, T, Kd, vals, meta, M, out, aux, stream, dec_w, dec_idx,
                                                      dec_lambda, fixed, a_mn);
}

template <bool SPARSE>
sp24_status launch_gemm(const void *B, int64_t T, int64_t Kd, const void *vals, const void *meta, int64_t M,
                        sp24_dtype dt, void *out, int epi, void *aux, cudaStream_t s, bool a_mn = false) {
  const bool bf = dt == SP24_BF16;
  switch (epi) {
    case kEpiNone: return bf ? launch_gemm_pair_t<true, kEpiNone, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                             : launch_gemm_pair_t<false, kEpiNone, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
    case kEpiGelu: return bf ? launch_gemm_pair_t<true, kEpiGelu, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                             : launch_gemm_pair_t<false, kEpiGelu, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
    case kEpiDgelu: return bf ? launch_gemm_pair_t<true, kEpiDgelu, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                              : launch_gemm_pair_t<false, kEpiDgelu, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
    case kEpiGeluDeriv:
      return bf ? launch_gemm_pair_t<true, kEpiGeluDeriv, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                : launch_gemm_pair_t<false, kEpiGeluDeriv, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
    case kEpiMulAux:
      return bf ? launch_gemm_pair_t<true, kEpiMulAux, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                : launch_gemm_pair_t<false, kEpiMulAux, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
    case kEpiGeluDerivPacked:
      return bf ? launch_gemm_pair_t<true, kEpiGeluDerivPacked, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                : launch_gemm_pair_t<false, kEpiGeluDerivPacked, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
    case kEpiMulAuxPacked:
      return bf ? launch_gemm_pair_t<true, kEpiMulAuxPacked, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                : launch_gemm_pair_t<false, kEpiMulAuxPacked, SPARSE>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
    default: break;
  }
  if (SPARSE) {   // the gated epilogues serve the 2:4 GEMMs
    switch (epi) {
      case kEpiGeglu: return bf ? launch_gemm_pair_t<true, kEpiGeglu, true>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                                : launch_gemm_pair_t<false, kEpiGeglu, true>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
      case kEpiDgeglu: return bf ? launch_gemm_pair_t<true, kEpiDgeglu, true>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn)
                                 : launch_gemm_pair_t<false, kEpiDgeglu, true>(B, T, Kd, vals, meta, M, out, aux, s, nullptr, nullptr, 0.0f, nullptr, a_mn);
      default: break;
    }
  }
  return SP24_ERR_INVALID_ARG;
}

// The epilogues each product takes (bit e of the mask allows epilogue e).
constexpr unsigned kFwdEpis = (1u << SP24_EPI_NONE) | (1u << SP24_EPI_GELU) | (1u << SP24_EPI_GEGLU) |
                              (1u << SP24_EPI_GELU_DERIV) | (1u << SP24_EPI_GELU_DERIV_PACKED);
constexpr unsigned kDgradEpis = (1u << SP24_EPI_NONE) | (1u << SP24_EPI_DGELU) | (1u << SP24_EPI_DGEGLU) |
                                (1u << SP24_EPI_MUL_AUX) | (1u << SP24_EPI_MUL_AUX_PACKED);
constexpr unsigned kDenseEpis = (1u << SP24_EPI_NONE) | (1u << SP24_EPI_GELU) | (1u << SP24_EPI_DGELU) |
                                (1u << SP24_EPI_GELU_DERIV) | (1u << SP24_EPI_MUL_AUX) |
                                (1u << SP24_EPI_GELU_DERIV_PACKED) | (1u << SP24_EPI_MUL_AUX_PACKED);
constexpr unsigned kDenseDgradEpis = (1u << SP24_EPI_NONE) | (1u << SP24_EPI_DGELU) | (1u << SP24_EPI_MUL_AUX) |
                                     (1u << SP24_EPI_MUL_AUX_PACKED);
static_assert((int)SP24_EPI_GELU_DERIV_PACKED == (int)kEpiGeluDerivPacked &&
                  (int)SP24_EPI_MUL_AUX_PACKED == (int)kEpiMulAuxPacked &&
                  (int)SP24_EPI_GELU_DERIV == (int)kEpiGeluDeriv && (int)SP24_EPI_MUL_AUX == (int)kEpiMulAux,
              "public and kernel epilogue numbers");

sp24_status validate_gemm(const void *B, int64_t T, int64_t Kd, const void *vals, const void *meta, int64_t M,
                          sp24_dtype dt, const void *out, int epi, const void *aux, unsigned allowed_epis) {
  if (!B && T > 0) return SP24_ERR_INVALID_ARG;
  if (!vals || !meta || (!out && T > 0)) return SP24_ERR_INVALID_ARG;
  if (T < 0 || Kd <= 0 || M <= 0) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dt)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (epi < 0 || epi > 31 || !((allowed_epis >> epi) & 1u)) return SP24_ERR_INVALID_ARG;
  if (epi == SP24_EPI_GEGLU && M % (2 * kGegluGroup)) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (epi != SP24_EPI_NONE && !aux && T > 0) return SP24_ERR_INVALID_ARG;   // T == 0 touches nothing
  if (Kd % 16 || M % 16) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (T > INT32_MAX || M > INT32_MAX || Kd > INT32_MAX) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(B) || !aligned16(vals) || !aligned16(meta) || !aligned16(out) ||
      (epi != SP24_EPI_NONE && !aligned16(aux)))
    return SP24_ERR_MISALIGNED;
  return SP24_OK;
}

// ------------------------------------------------------------ mask launches

template <bool BF16, bool SEARCH, bool COMPRESS, bool FLIP>
sp24_status launch_mask_t(const void *W, int64_t R, int64_t C, int64_t ldw, uint8_t *idx, const uint8_t *prev,
                          unsigned long long *flip, void *vr, void *mr, void *vc, void *mc, cudaStream_t s) {
  // CTA tiles cover whole 128x128 regions (one metadata chunk of each orientation).
  const int64_t chunks_x = (C + kChunk - 1) / kChunk, chunks_y = (R + kChunk - 1) / kChunk;
  if (chunks_y > 65535 || chunks_x * (kChunk / kMaskCtaCols) > INT32_MAX) return SP24_ERR_UNSUPPORTED_SHAPE;
  const int64_t ntiles = chunks_x * chunks_y * (kChunk / kMaskCtaCols);
  CUtensorMap tm;
  // Persistent form with tensor-memory-accelerator loads of W (row pitch a multiple of 16 bytes).
  if (ldw % 8 == 0 && C <= INT32_MAX && R <= INT32_MAX &&
      make_map_2d(&tm, W, (uint64_t)C, (uint64_t)R, (uint64_t)ldw * 2, kMaskCtaCols, kChunk,
                  CU_TENSOR_MAP_SWIZZLE_NONE)) {
    const int64_t ctas = (int64_t)sm_count() * mask_ctas_per_sm<COMPRESS>();
    const unsigned grid = (unsigned)(ntiles < ctas ? ntiles : ctas);
    // The previous mask travels with each W tile by TMA ([R/4][C/4] bytes, a 16 x 32
    // box per tile) when its row pitch is a multiple of 16 bytes; else plain loads.
    CUtensorMap tp = tm;
    const int prev_tma = (FLIP && prev && (C / 4) % 16 == 0 && aligned16(prev) &&
                          make_map_2d(&tp, prev, (uint64_t)(C / 4), (uint64_t)(R / 4), (uint64_t)(C / 4), kMaskCtaCols / 4,
                                      kChunk / 4, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_UINT8))
                             ? 1
                             : 0;
    return launch_pdl(mask_stream_kernel<BF16, SEARCH, COMPRESS, FLIP>, dim3(grid), dim3(kMaskThreads), 0, s, tm, R,
                      C, idx, prev, flip, static_cast<uint16_t *>(vr), static_cast<uint8_t *>(mr),
                      static_cast<uint16_t *>(vc), static_cast<uint8_t *>(mc), (uint64_t)g_wait_budget.load(), tp,
                      prev_tma);
  }
  dim3 grid((unsigned)(chunks_x * (kChunk / kMaskCtaCols)), (unsigned)chunks_y);
  return launch_pdl(mask_tile_kernel<BF16, SEARCH, COMPRESS, FLIP>, grid, dim3(kMaskThreads), 0, s,
                    static_cast<const uint16_t *>(W), R, C, ldw, idx, prev, flip, static_cast<uint16_t *>(vr),
                    static_cast<uint8_t *>(mr), static_cast<uint16_t *>(vc), static_cast<uint8_t *>(mc));
}

template <bool SEARCH, bool COMPRESS, bool FLIP>
sp24_status launch_mask_d(bool bf, const void *W, int64_t R, int64_t C, int64_t ldw, uint8_t *idx,
                          const uint8_t *prev, unsigned long long *flip, void *vr, void *mr, void *vc, void *mc,
                          cudaStream_t s) {
  return bf ? launch_mask_t<true, SEARCH, COMPRESS, FLIP>(W, R, C, ldw, idx, prev, flip, vr, mr, vc, mc, s)
            : launch_mask_t<false, SEARCH, COMPRESS, FLIP>(W, R, C, ldw, idx, prev, flip, vr, mr, vc, mc, s);
}

sp24_status validate_w(const void *W, sp24_dtype dt, int64_t rows, int64_t cols, int64_t ldw) {
  if (rows < 0 || cols < 0 || ldw < cols) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dt)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (rows % 4 || cols % 4) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (rows > 0 && cols > 0) {
    if (!W) return SP24_ERR_INVALID_ARG;
    if (!aligned16(W) || ldw % 4) return SP24_ERR_MISALIGNED;
  }
  return SP24_OK;
}

size_t meta_bytes_of(int64_t rows, int64_t cols) {
  return (size_t)((rows + 127) / 128) * (size_t)((cols + 127) / 128) * 2048u;
}

// Byte offset, inside the device metadata of a [rows x cols] matrix, of the
// nibble for row r, group g (columns 4g..4g+3), and the nibble's bit shift.
inline size_t meta_nibble_pos(int64_t r, int64_t g, int64_t cols, int *shift) {
  const int64_t kt_count = (cols + 127) / 128;
  const int64_t mt = r / 128, m = r % 128;
  const int64_t kt = g / 32, gk = g % 32;           // 32 groups per 128-column chunk
  const int64_t kk = gk / 8, gg = gk % 8;           // 8 groups per 32-column K step
  const int64_t lane = (m % 8) + 8 * (gg / 4) + 16 * (m / 16);
  const int bit = 4 * (int)(gg % 4) + 16 * (int)((m / 8) % 2);
  *shift = bit % 8;
  return (size_t)(mt * kt_count + kt) * 2048 + (size_t)lane * 16 + (size_t)kk * 4 + (size_t)(bit / 8);
}

// Weight gradient: tiles of 256 rows x 256 columns of dW (see PairGeom).
template <bool BF16, bool SPARSE>
sp24_status launch_wgrad(const void *X, int64_t T, int64_t K, const void *A, const void *meta, int64_t N, float *dW,
                         cudaStream_t s, const void *dec_w = nullptr, const uint8_t *dec_idx = nullptr,
                         float dec_lambda = 0.0f, const SkWorkspace *fixed = nullptr) {
  return launch_gemm_pair_t<BF16, kEpiWgrad, SPARSE>(X, K, T, A, meta, N, dW, nullptr, s, dec_w, dec_idx, dec_lambda,
                                                     fixed);
}

}  // namespace

namespace {
// (packed chunk layout of the derivative-saving epilogues; see gemm_sp.cuh)
// Element offset, in the packed chunk layout of a [T x M] matrix, of (t, m).
size_t aux_packed_offset(int64_t t, int64_t m, int64_t M) {
  const int64_t tin = t & 15, fin = m & 31, h = fin >> 4, ff = fin & 15;
  const int64_t lane = 4 * (ff & 7) + ((tin & 7) >> 1), reg = 2 * (tin >> 3) + (ff >> 3);
  const int64_t block = (t >> 4) * ((M + 31) / 32) + (m >> 5);
  return (size_t)(block * 512 + h * 256 + lane * 8 + reg * 2 + (tin & 1));
}
}  // namespace

extern "C" {

const char *sp24_status_string(sp24_status st) {
  switch (st) {
    case SP24_OK: return "SP24_OK";
    case SP24_ERR_INVALID_ARG: return "SP24_ERR_INVALID_ARG";
    case SP24_ERR_UNSUPPORTED_SHAPE: return "SP24_ERR_UNSUPPORTED_SHAPE";
    case SP24_ERR_UNSUPPORTED_DTYPE: return "SP24_ERR_UNSUPPORTED_DTYPE";
    case SP24_ERR_MISALIGNED: return "SP24_ERR_MISALIGNED";
    case SP24_ERR_CUDA: return "SP24_ERR_CUDA";
    case SP24_ERR_TIMEOUT: return "SP24_ERR_TIMEOUT";
    case SP24_ERR_NO_DEVICE: return "SP24_ERR_NO_DEVICE";
    case SP24_ERR_SCRATCH_TOO_SMALL: return "SP24_ERR_SCRATCH_TOO_SMALL";
  }
  return "SP24_UNKNOWN_STATUS";
}

sp24_status sp24_pattern_table(uint16_t *out) {
  if (!out) return SP24_ERR_INVALID_ARG;
  constexpr PatternTables t = make_pattern_tables();
  for (int p = 0; p < kNumPatterns; ++p) out[p] = t.bits[p];
  return SP24_OK;
}

sp24_status sp24_compressed_size(int64_t rows, int64_t cols, sp24_dtype dtype, size_t *vals_bytes,
                                 size_t *meta_bytes) {
  if (!vals_bytes || !meta_bytes || rows < 0 || cols < 0) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (rows % 4 || cols % 4) return SP24_ERR_UNSUPPORTED_SHAPE;
  *vals_bytes = (size_t)rows * (size_t)(cols / 2) * 2u;
  *meta_bytes = meta_bytes_of(rows, cols);
  return SP24_OK;
}

sp24_status sp24_mask_step(const void *W, sp24_dtype dtype, int64_t rows, int64_t cols, int64_t ldw, uint8_t *idx,
                           const uint8_t *idx_prev, unsigned long long *d_flip_count, void *vals_row,
                           void *meta_row, void *vals_col, void *meta_col, void *stream) {
  sp24_status st = validate_w(W, dtype, rows, cols, ldw);
  if (st != SP24_OK) return st;
  const bool flip = idx_prev != nullptr;
  if ((idx_prev == nullptr) != (d_flip_count == nullptr)) return SP24_ERR_INVALID_ARG;
  const bool any_c = vals_row || meta_row || vals_col || meta_col;
  const bool all_c = vals_row && meta_row && vals_col && meta_col;
  if (any_c && !all_c) return SP24_ERR_INVALID_ARG;
  if (!idx && rows > 0 && cols > 0) return SP24_ERR_INVALID_ARG;
  if (all_c) {
    if (rows % 16 || cols % 16) return SP24_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(vals_row) || !aligned16(meta_row) || !aligned16(vals_col) || !aligned16(meta_col))
      return SP24_ERR_MISALIGNED;
  }
  if ((st = check_device()) != SP24_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (flip && cudaMemsetAsync(d_flip_count, 0, sizeof(unsigned long long), s) != cudaSuccess)
    return SP24_ERR_CUDA;
  if (rows == 0 || cols == 0) return SP24_OK;
  const bool bf = dtype == SP24_BF16;
  if (all_c && flip)
    return launch_mask_d<true, true, true>(bf, W, rows, cols, ldw, idx, idx_prev, d_flip_count, vals_row, meta_row,
                                           vals_col, meta_col, s);
  if (all_c)
    return launch_mask_d<true, true, false>(bf, W, rows, cols, ldw, idx, nullptr, nullptr, vals_row, meta_row,
                                            vals_col, meta_col, s);
  if (flip)
    return launch_mask_d<true, false, true>(bf, W, rows, cols, ldw, idx, idx_prev, d_flip_count, nullptr, nullptr,
                                            nullptr, nullptr, s);
  return launch_mask_d<true, false, false>(bf, W, rows, cols, ldw, idx, nullptr, nullptr, nullptr, nullptr,
                                           nullptr, nullptr, s);
}

sp24_status sp24_mask_search(const void *W, sp24_dtype dtype, int64_t rows, int64_t cols, int64_t ldw, uint8_t *idx,
                             void *stream) {
  return sp24_mask_step(W, dtype, rows, cols, ldw, idx, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        stream);
}

sp24_status sp24_prune_compress(const void *W, sp24_dtype dtype, int64_t rows, int64_t cols, int64_t ldw,
                                const uint8_t *idx, void *vals_row, void *meta_row, void *vals_col, void *meta_col,
                                void *stream) {
  sp24_status st = validate_w(W, dtype, rows, cols, ldw);
  if (st != SP24_OK) return st;
  if ((vals_row == nullptr) != (meta_row == nullptr) || (vals_col == nullptr) != (meta_col == nullptr))
    return SP24_ERR_INVALID_ARG;
  if (rows % 16 || cols % 16) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (rows > 0 && cols > 0 && !idx) return SP24_ERR_INVALID_ARG;
  if ((vals_row && (!aligned16(vals_row) || !aligned16(meta_row))) ||
      (vals_col && (!aligned16(vals_col) || !aligned16(meta_col))))
    return SP24_ERR_MISALIGNED;
  if ((st = check_device()) != SP24_OK) return st;
  if (rows == 0 || cols == 0 || (!vals_row && !vals_col)) return SP24_OK;
  return launch_mask_d<false, true, false>(dtype == SP24_BF16, W, rows, cols, ldw, const_cast<uint8_t *>(idx),
                                           nullptr, nullptr, vals_row, meta_row, vals_col, meta_col,
                                           as_stream(stream));
}

sp24_status sp24_gemm_fwd(const void *X, int64_t T, int64_t K, const void *vals_row, const void *meta_row, int64_t N,
                          sp24_dtype dtype, void *Y, sp24_epilogue epi, void *aux, void *stream) {
  sp24_status st = validate_gemm(X, T, K, vals_row, meta_row, N, dtype, Y, epi, aux, kFwdEpis);
  if (st != SP24_OK) return st;
  if ((st = check_device()) != SP24_OK) return st;
  if (T == 0) return SP24_OK;
  return launch_gemm<true>(X, T, K, vals_row, meta_row, N, dtype, Y, epi, aux, as_stream(stream));
}

sp24_status sp24_gemm_dgrad(const void *dY, int64_t T, int64_t N, const void *vals_col, const void *meta_col,
                            int64_t K, sp24_dtype dtype, void *dX, sp24_epilogue epi, const void *aux,
                            void *stream) {
  sp24_status st = validate_gemm(dY, T, N, vals_col, meta_col, K, dtype, dX, epi, aux, kDgradEpis);
  if (st != SP24_OK) return st;
  if ((st = check_device()) != SP24_OK) return st;
  if (T == 0) return SP24_OK;
  return launch_gemm<true>(dY, T, N, vals_col, meta_col, K, dtype, dX, epi, const_cast<void *>(aux),
                          as_stream(stream));
}

sp24_status sp24_gemm_dense(const void *B, int64_t T, int64_t Kd, const void *A, int64_t M, sp24_dtype dtype,
                            void *out, sp24_epilogue epi, void *aux, void *stream) {
  sp24_status st = validate_gemm(B, T, Kd, A, A, M, dtype, out, epi, aux, kDenseEpis);
  if (st != SP24_OK) return st;
  if ((st = check_device()) != SP24_OK) return st;
  if (T == 0) return SP24_OK;
  return launch_gemm<false>(B, T, Kd, A, nullptr, M, dtype, out, epi, aux, as_stream(stream));
}

sp24_status sp24_gemm_dgrad_dense(const void *dY, int64_t T, int64_t N, const void *W, int64_t K, sp24_dtype dtype,
                                  void *dX, sp24_epilogue epi, const void *aux, void *stream) {
  sp24_status st = validate_gemm(dY, T, N, W, W, K, dtype, dX, epi, aux, kDenseDgradEpis);
  if (st != SP24_OK) return st;
  if ((st = check_device()) != SP24_OK) return st;
  if (T == 0) return SP24_OK;
  return launch_gemm<false>(dY, T, N, W, nullptr, K, dtype, dX, epi, const_cast<void *>(aux), as_stream(stream),
                            /*a_mn=*/true);
}

sp24_status sp24_transpose(const void *in, int64_t rows, int64_t cols, sp24_dtype dtype, void *out, void *stream) {
  if (rows < 0 || cols < 0) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (rows == 0 || cols == 0) return SP24_OK;
  if (!in || !out) return SP24_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(out)) return SP24_ERR_MISALIGNED;
  if (rows > INT32_MAX || cols > INT32_MAX) return SP24_ERR_UNSUPPORTED_SHAPE;
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  const dim3 grid((unsigned)((cols + kTransTile - 1) / kTransTile),
                  (unsigned)((rows + kTransTile - 1) / kTransTile < 65535 ? (rows + kTransTile - 1) / kTransTile
                                                                            : 65535));
  return launch_pdl(transpose16_kernel, grid, dim3(256), 0, as_stream(stream),
                    static_cast<const uint16_t *>(in), static_cast<uint16_t *>(out), rows, cols);
}

sp24_status sp24_mvue_sparsify(const void *dY, int64_t T, int64_t N, int64_t ldy, sp24_dtype dtype, uint64_t seed,
                               uint64_t offset, void *vals, void *meta, void *stream) {
  if (T < 0 || N < 0 || ldy < N) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (T % 16 || N % 8) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (T > INT32_MAX || N > (int64_t)65535 / 2 * 128) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (T == 0 || N == 0) return SP24_OK;
  if (!dY || !vals || !meta) return SP24_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(vals) || !aligned16(meta) || ldy % 8) return SP24_ERR_MISALIGNED;
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  // Whole metadata chunks: 128 tokens x 128 columns, two CTAs per chunk.
  const dim3 grid((unsigned)((T + kMvueTokens - 1) / kMvueTokens), (unsigned)(2 * ((N + 127) / 128)));
  cudaStream_t s = as_stream(stream);
  const uint16_t *d16 = static_cast<const uint16_t *>(dY);
  uint16_t *v16 = static_cast<uint16_t *>(vals);
  uint8_t *m8 = static_cast<uint8_t *>(meta);
  const PhiloxKeys keys = philox4x64_keys(seed, offset);
  return dtype == SP24_BF16
             ? launch_pdl(mvue_sparsify_kernel<true>, grid, dim3(kMvueThreads), 0, s, d16, T, N, ldy, keys, v16, m8)
             : launch_pdl(mvue_sparsify_kernel<false>, grid, dim3(kMvueThreads), 0, s, d16, T, N, ldy, keys, v16, m8);
}

sp24_status sp24_gemm_wgrad(const void *X, int64_t T, int64_t K, const void *vals, const void *meta, int64_t N,
                            sp24_dtype dtype, float *dW, void *stream) {
  if (T < 0 || K < 0 || N < 0) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (T % 16 || N % 16 || K % 8) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (T > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return SP24_OK;
  if (!dW || (T > 0 && (!X || !vals || !meta))) return SP24_ERR_INVALID_ARG;
  if (!aligned16(dW) || (T > 0 && (!aligned16(X) || !aligned16(vals) || !aligned16(meta)))) return SP24_ERR_MISALIGNED;
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (T == 0) {   // an empty sum over tokens
    return cudaMemsetAsync(dW, 0, (size_t)N * (size_t)K * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  }
  return dtype == SP24_BF16 ? launch_wgrad<true, true>(X, T, K, vals, meta, N, dW, s)
                            : launch_wgrad<false, true>(X, T, K, vals, meta, N, dW, s);
}

sp24_status sp24_gemm_wgrad_noalloc(const void *X, int64_t T, int64_t K, const void *vals, const void *meta,
                                    int64_t N, sp24_dtype dtype, float *dW, void *stream) {
  if (T < 0 || K < 0 || N < 0) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (T % 16 || N % 16 || K % 8) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (T > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return SP24_OK;
  if (!dW || (T > 0 && (!X || !vals || !meta))) return SP24_ERR_INVALID_ARG;
  if (!aligned16(dW) || (T > 0 && (!aligned16(X) || !aligned16(vals) || !aligned16(meta)))) return SP24_ERR_MISALIGNED;
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (T == 0) {   // an empty sum over tokens
    return cudaMemsetAsync(dW, 0, (size_t)N * (size_t)K * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  }
  SkWorkspace fixed;
  st = noalloc_scratch(&fixed);
  if (st != SP24_OK) return st;
  return dtype == SP24_BF16 ? launch_wgrad<true, true>(X, T, K, vals, meta, N, dW, s, nullptr, nullptr, 0.0f, &fixed)
                            : launch_wgrad<false, true>(X, T, K, vals, meta, N, dW, s, nullptr, nullptr, 0.0f, &fixed);
}

sp24_status sp24_gemm_wgrad_decay(const void *X, int64_t T, int64_t K, const void *vals, const void *meta,
                                  int64_t N, sp24_dtype dtype, const void *W, const uint8_t *idx, float lambda,
                                  float *dW, void *stream) {
  if (T < 0 || K < 0 || N < 0) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (T % 16 || N % 16 || K % 8) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (T > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return SP24_OK;
  if (!dW || !W || !idx || (T > 0 && (!X || !vals || !meta))) return SP24_ERR_INVALID_ARG;
  if (!aligned16(dW) || !aligned16(W) || (T > 0 && (!aligned16(X) || !aligned16(vals) || !aligned16(meta))))
    return SP24_ERR_MISALIGNED;
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (T == 0) {   // an empty sum over tokens, then the decay of the zero gradient
    if (cudaMemsetAsync(dW, 0, (size_t)N * (size_t)K * sizeof(float), s) != cudaSuccess) return SP24_ERR_CUDA;
    return sp24_masked_decay(dW, W, dtype, N, K, idx, lambda, stream);
  }
  return dtype == SP24_BF16 ? launch_wgrad<true, true>(X, T, K, vals, meta, N, dW, s, W, idx, lambda)
                            : launch_wgrad<false, true>(X, T, K, vals, meta, N, dW, s, W, idx, lambda);
}

sp24_status sp24_gemm_wgrad_dense(const void *X, int64_t T, int64_t K, const void *dY, int64_t N, sp24_dtype dtype,
                                  float *dW, void *stream) {
  if (T < 0 || K < 0 || N < 0) return SP24_ERR_INVALID_ARG;
  if (!valid_dtype(dtype)) return SP24_ERR_UNSUPPORTED_DTYPE;
  if (T % 16 || N % 16 || K % 8) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (T > INT32_MAX || K > INT32_MAX || N > INT32_MAX) return SP24_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return SP24_OK;
  if (!dW || (T > 0 && (!X || !dY))) return SP24_ERR_INVALID_ARG;
  if (!aligned16(dW) || (T > 0 && (!aligned16(X) || !aligned16(dY)))) return SP24_ERR_MISALIGNED;
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (T == 0) {   // an empty sum over tokens
    return cudaMemsetAsync(dW, 0, (size_t)N * (size_t)K * sizeof(float), s) == cudaSuccess ? SP24_OK : SP24_ERR_CUDA;
  }
  return dtype == SP24_BF16 ? launch_wgrad<true, false>(X, T, K, dY, nullptr, N, dW, s)
                            : launch_wgrad<false, false>(X, T, K, dY, nullptr, N, dW, s);
}

sp24_status sp24_masked_decay(float *grad, const void *W, sp24_dtype dtype, int64_t rows, int64_t cols,
                              const uint8_t *idx, float lambda, void *stream) {
  sp24_status st = validate_w(W, dtype, rows, cols, cols);
  if (st != SP24_OK) return st;
  if (rows > 0 && cols > 0 && (!grad || !idx)) return SP24_ERR_INVALID_ARG;
  if (rows > 0 && cols > 0 && !aligned16(grad)) return SP24_ERR_MISALIGNED;
  if ((st = check_device()) != SP24_OK) return st;
  if (rows == 0 || cols == 0) return SP24_OK;
  const int64_t strips = (cols / 4 + 255) / 256;
  const int64_t brows = rows / 4;
  const dim3 grid((unsigned)strips, (unsigned)(brows < 65535 ? brows : 65535));
  cudaStream_t s = as_stream(stream);
  const uint16_t *w16 = static_cast<const uint16_t *>(W);
  return dtype == SP24_BF16 ? launch_pdl(masked_decay_kernel<true>, grid, dim3(256), 0, s, grad, w16, idx, rows, cols, lambda)
                            : launch_pdl(masked_decay_kernel<false>, grid, dim3(256), 0, s, grad, w16, idx, rows, cols, lambda);
}

sp24_status sp24_flip_rate(const uint8_t *idx_prev, const uint8_t *idx_cur, int64_t nblocks,
                           unsigned long long *d_count, void *stream) {
  if (nblocks < 0 || !d_count || (nblocks > 0 && (!idx_prev || !idx_cur))) return SP24_ERR_INVALID_ARG;
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(d_count, 0, sizeof(unsigned long long), s) != cudaSuccess) return SP24_ERR_CUDA;
  if (nblocks == 0) return SP24_OK;
  const int64_t want = (nblocks / 16 + 255) / 256 + 1;
  const int grid = (int)(want < (int64_t)sm_count() * 8 ? want : (int64_t)sm_count() * 8);
  return launch_pdl(flip_count_kernel, dim3(grid), dim3(256), 0, s, idx_prev, idx_cur, nblocks, d_count);
}

sp24_status sp24_aux_packed_size(int64_t T, int64_t M, size_t *bytes) {
  if (T < 0 || M < 0 || !bytes) return SP24_ERR_INVALID_ARG;
  *bytes = (size_t)((T + 15) / 16) * (size_t)((M + 31) / 32) * 1024u;
  return SP24_OK;
}

sp24_status sp24_aux_pack(const void *rowmajor, int64_t T, int64_t M, void *packed) {
  if (T < 0 || M < 0 || (T > 0 && M > 0 && (!rowmajor || !packed))) return SP24_ERR_INVALID_ARG;
  const uint16_t *src = static_cast<const uint16_t *>(rowmajor);
  uint16_t *dst = static_cast<uint16_t *>(packed);
  size_t bytes = 0;
  sp24_aux_packed_size(T, M, &bytes);
  if (bytes) memset(dst, 0, bytes);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t m = 0; m < M; ++m) dst[aux_packed_offset(t, m, M)] = src[t * M + m];
  return SP24_OK;
}

sp24_status sp24_aux_unpack(const void *packed, int64_t T, int64_t M, void *rowmajor) {
  if (T < 0 || M < 0 || (T > 0 && M > 0 && (!rowmajor || !packed))) return SP24_ERR_INVALID_ARG;
  const uint16_t *src = static_cast<const uint16_t *>(packed);
  uint16_t *dst = static_cast<uint16_t *>(rowmajor);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t m = 0; m < M; ++m) dst[t * M + m] = src[aux_packed_offset(t, m, M)];
  return SP24_OK;
}

sp24_status sp24_meta_to_canonical(const void *meta_dev_layout_host, int64_t rows, int64_t cols, uint16_t *canon) {
  if (!meta_dev_layout_host || !canon || rows < 0 || cols < 0) return SP24_ERR_INVALID_ARG;
  if (rows % 4 || cols % 16) return SP24_ERR_UNSUPPORTED_SHAPE;
  const uint8_t *dev = static_cast<const uint8_t *>(meta_dev_layout_host);
  const int64_t words = cols / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t w = 0; w < words; ++w) {
      uint16_t v = 0;
      for (int e = 0; e < 4; ++e) {
        int shift = 0;
        const size_t pos = meta_nibble_pos(r, 4 * w + e, cols, &shift);
        v |= (uint16_t)(((dev[pos] >> shift) & 0xF) << (4 * e));
      }
      canon[r * words + w] = v;
    }
  return SP24_OK;
}

sp24_status sp24_meta_from_canonical(const uint16_t *canon, int64_t rows, int64_t cols, void *meta_dev_layout_host) {
  if (!meta_dev_layout_host || !canon || rows < 0 || cols < 0) return SP24_ERR_INVALID_ARG;
  if (rows % 4 || cols % 16) return SP24_ERR_UNSUPPORTED_SHAPE;
  uint8_t *dev = static_cast<uint8_t *>(meta_dev_layout_host);
  memset(dev, 0x44, meta_bytes_of(rows, cols));
  const int64_t words = cols / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t w = 0; w < words; ++w)
      for (int e = 0; e < 4; ++e) {
        int shift = 0;
        const size_t pos = meta_nibble_pos(r, 4 * w + e, cols, &shift);
        const uint8_t nib = (uint8_t)((canon[r * words + w] >> (4 * e)) & 0xF);
        dev[pos] = (uint8_t)((dev[pos] & ~(0xF << shift)) | (nib << shift));
      }
  return SP24_OK;
}

sp24_status sp24_device_status(void *stream) {
  sp24_status st = check_device();
  if (st != SP24_OK) return st;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return SP24_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess) return SP24_ERR_CUDA;
  if (word && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return SP24_ERR_CUDA;
  if (word && sk_clear_flags() != SP24_OK) return SP24_ERR_CUDA;
  return (word & kDevErrTimeout) ? SP24_ERR_TIMEOUT : SP24_OK;
}

sp24_status sp24_set_wait_budget(uint64_t cycles) {
  g_wait_budget.store(cycles);
  return SP24_OK;
}

}  // extern "C"
