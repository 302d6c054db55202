/*
 * sp24 -- 2:4 transposable-mask FFN kernels for NVIDIA B200 (sm_100a).
 *
 * C ABI of libsp24.so.  The operations come from "Accelerating Transformer
 * Pre-training with 2:4 Sparsity" (Hu, Zhao, Huang, Chen, Zhu; ICML 2024):
 *   - reproducibility table, Pseudocode row, Algorithm 1: transposable 2:4 mask
 *     search by convolving |W| at stride 4 with the candidate 4x4 patterns and
 *     taking the argmax per block;
 *   - reproducibility table, Software Dependencies row: the pruning kernel and
 *     the 2:4 sparse matrix multiplications, the masked decay kernel;
 *   - abstract: masked decay on gradients, the flip rate that monitors mask
 *     stability, and transposable masks so the backward product is 2:4 too;
 *   - Software Dependencies row: the MVUE kernel (here the minimum-variance
 *     unbiased 2:4 estimate of dY^T, sp24_mvue_sparsify) feeding the 2:4
 *     weight-gradient product (sp24_gemm_wgrad), and the GEGLU kernel (the gated
 *     epilogues of sp24_gemm_fwd / sp24_gemm_dgrad);
 *   - abstract and Experiment Setup row: dense fine-tuning for the last 1/6 of
 *     the steps (sp24_gemm_dense, sp24_gemm_dgrad_dense, sp24_gemm_wgrad_dense,
 *     sp24_transpose).
 *
 * Conventions shared by every call
 *   - Matrices are row-major.  W is [rows x cols] with leading dimension ldw
 *     (elements).  A "block" is the 4x4 tile W[4i..4i+3][4j..4j+3].
 *   - A mask is one uint8 pattern index per block, row-major
 *     [rows/4][cols/4].  Index p in 0..89 names the p-th 4x4 0/1 pattern with
 *     two ones in every row and column, in lexicographic order of the per-row
 *     column pairs (each row's pair ranked (0,1)<(0,2)<(0,3)<(1,2)<(1,3)<(2,3),
 *     row 0 most significant).  sp24_pattern_table() returns the patterns.
 *   - Device pointers (marked "device") are caller-owned device memory; host
 *     pointers (marked "host") are caller-owned host memory.  The library
 *     keeps no caller pointer after a call returns.  It allocates only the
 *     weight-gradient workspace (see sp24_gemm_wgrad): one per (device,
 *     stream), made by the first call on that stream that needs it and kept
 *     for the life of the process.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls that launch work are asynchronous and stream-ordered.
 *   - Argument checks (shapes, dtypes, alignment, null pointers) run on the
 *     host before anything is launched; a failed check launches nothing.
 *   - Weights must be finite; results for NaN/Inf weights are unspecified
 *     (never out-of-bounds accesses).
 *   - A kernel that gives up waiting (bounded spin on an mbarrier or on a
 *     counter in global memory) records it in a per-device error word and
 *     exits; sp24_device_status() reports it.
 */
#ifndef SP24_H
#define SP24_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SP24_API __attribute__((visibility("default")))
#else
#define SP24_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sp24_status {
  SP24_OK = 0,
  SP24_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum, ld < width */
  SP24_ERR_UNSUPPORTED_SHAPE = 2, /* a size is not a multiple the call needs */
  SP24_ERR_UNSUPPORTED_DTYPE = 3,
  SP24_ERR_MISALIGNED = 4,        /* a pointer or row pitch is not 16-byte aligned */
  SP24_ERR_CUDA = 5,              /* a CUDA runtime/driver call or launch failed */
  SP24_ERR_TIMEOUT = 6,           /* a kernel gave up waiting (see sp24_device_status) */
  SP24_ERR_NO_DEVICE = 7,         /* no sm_100 device is current */
  SP24_ERR_SCRATCH_TOO_SMALL = 8  /* the call needs more than a fixed scratch holds
                                     (sp24_gemm_wgrad_noalloc) */
} sp24_status;

typedef enum sp24_dtype { SP24_F16 = 0, SP24_BF16 = 1 } sp24_dtype;

typedef enum sp24_epilogue {
  SP24_EPI_NONE = 0,
  SP24_EPI_GELU = 1,  /* out = gelu(acc) (exact erf form); aux <- acc rounded to dtype */
  SP24_EPI_DGELU = 2, /* out = acc * gelu'(aux); aux holds the pre-activation */
  /* Gated GELU (abstract: gated activation functions).  The stacked weight
   * holds groups of 16 rows of W_gate and of W_up alternately (gate rows
   * 16g..16g+15 at 32g.., up rows at 32g+16..), so the accumulator columns of
   * one output feature sit 16 apart. */
  SP24_EPI_GEGLU = 3, /* out[T x N/2] = gelu(gate) * up; aux[T x N] <- acc (both halves) */
  SP24_EPI_DGEGLU = 4, /* out[T x 2K] = (acc*up*gelu'(gate), acc*gelu(gate)) interleaved as
                          aux; aux[T x 2K] holds the gated pre-activations */
  /* Derivative-saving GELU pair: the forward stores gelu'(pre-activation) as aux,
   * so the input gradient multiplies by it and evaluates no GELU'.  The same
   * product as SP24_EPI_GELU / SP24_EPI_DGELU, with the derivative rounded to the
   * dtype instead of the pre-activation.  (Value 5 is the library's own
   * weight-gradient epilogue and is not taken here.) */
  SP24_EPI_GELU_DERIV = 6, /* out = gelu(acc); aux <- gelu'(acc) rounded to dtype */
  SP24_EPI_MUL_AUX = 7,    /* out = acc * aux; aux [T x K] holds gelu'(pre-activation) */
  /* The same pair with aux in the packed chunk layout below instead of
   * row-major: the kernels write and read it straight from the registers that
   * hold the accumulator, with no staging in shared memory. */
  SP24_EPI_GELU_DERIV_PACKED = 8, /* out = gelu(acc); aux (packed) <- gelu'(acc) */
  SP24_EPI_MUL_AUX_PACKED = 9     /* out = acc * aux; aux (packed) holds gelu'(pre-activation) */
} sp24_epilogue;

/*
 * Packed chunk layout of a 16-bit [T x M] matrix (the aux of the _PACKED
 * epilogues, M the output width of the product that writes or reads it):
 * blocks of 16 tokens x 32 features, 1024 bytes each; block (t/16, m/32)
 * starts at element ((t/16) * ceil(M/32) + m/32) * 512.  In a block, element
 * (t, m) with t' = t % 16, m' = m % 32, h = m' / 16, f = m' % 16 sits at
 *   256 h + 8 (4 (f % 8) + (t' % 8) / 2) + 2 (2 (t' / 8) + f / 8) + t' % 2.
 * Blocks past T or M are part of the buffer (ceil(T/16) x ceil(M/32) blocks);
 * their padding entries are unspecified.  The buffer must be 16-byte aligned.
 */
SP24_API sp24_status sp24_aux_packed_size(int64_t T, int64_t M, size_t *bytes);

/* Host index maps of the packed layout (host memory, 16-bit elements):
 * sp24_aux_pack writes every block of packed (padding entries 0) from
 * rowmajor [T x M]; sp24_aux_unpack writes rowmajor from packed. */
SP24_API sp24_status sp24_aux_pack(const void *rowmajor, int64_t T, int64_t M, void *packed);
SP24_API sp24_status sp24_aux_unpack(const void *packed, int64_t T, int64_t M, void *rowmajor);

/* Human-readable name of a status code (static storage, never NULL). */
SP24_API const char *sp24_status_string(sp24_status status);

/* Copies the 90 candidate patterns (bit 4*i+j set <=> row i, column j kept)
 * into out[0..89] (host).  Algorithm 1's filter set m. */
SP24_API sp24_status sp24_pattern_table(uint16_t *out);

/*
 * Transposable 2:4 mask search (Algorithm 1).
 * For every block, scores each of the 90 patterns by the exact sum of the |W|
 * values it keeps and writes the index of the best one; ties go to the lowest
 * index.  The result is bit-exact (scores are exact integer sums, never
 * rounded).
 *   W    device, dtype, [rows x ldw] row-major, 16-byte aligned, ldw % 4 == 0
 *        (ldw % 8 == 0 lets every row be read with 128-bit loads)
 *   idx  device, uint8 [rows/4][cols/4]
 *   rows, cols multiples of 4 (>= 0; zero-sized calls return SP24_OK).
 */
SP24_API sp24_status sp24_mask_search(const void *W, sp24_dtype dtype, int64_t rows, int64_t cols,
                             int64_t ldw, uint8_t *idx, void *stream);

/*
 * Sizes of one compressed orientation of an [rows x cols] matrix compressed
 * along its rows (2 of every 4 values per row are kept):
 *   vals_bytes = rows * cols/2 * 2       (values, row-major [rows][cols/2])
 *   meta_bytes = ceil(rows/128) * ceil(cols/128) * 2048
 * The forward operand of W [R x C] is sp24_compressed_size(R, C); the
 * input-gradient operand (W^T compressed along its rows) is (C, R).
 */
SP24_API sp24_status sp24_compressed_size(int64_t rows, int64_t cols, sp24_dtype dtype, size_t *vals_bytes,
                                 size_t *meta_bytes);

/*
 * Pruning and compression of W with a given mask (the pruning kernel of the
 * Software Dependencies row), into the layout the sparse tensor cores read.
 *   vals_row  device [rows][cols/2]   kept values of each row, in column order
 *   meta_row  device, meta_bytes of (rows, cols): 2-bit positions, tiled in
 *             128x128 chunks of 2048 bytes in tensor-memory lane order
 *   vals_col  device [cols][rows/2]   kept values of each column of W (rows of W^T)
 *   meta_col  device, meta_bytes of (cols, rows)
 * Either orientation may be skipped by passing NULL for both of its pointers.
 * rows % 16 == 0 and cols % 16 == 0.  Every byte of the metadata buffers is
 * written (padding carries a valid code).  sp24_meta_to_canonical() maps the
 * metadata to a canonical per-row form.
 */
SP24_API sp24_status sp24_prune_compress(const void *W, sp24_dtype dtype, int64_t rows, int64_t cols,
                                int64_t ldw, const uint8_t *idx, void *vals_row, void *meta_row,
                                void *vals_col, void *meta_col, void *stream);

/*
 * One mask update in a single pass over W: search (as sp24_mask_search),
 * optionally the flip count against the previous mask (as sp24_flip_rate) and
 * optionally the compression of both orientations (as sp24_prune_compress).
 *   idx_prev, d_flip_count  both NULL or both set (device); *d_flip_count is
 *                           overwritten with the number of changed mask entries
 *   vals_row..meta_col      as sp24_prune_compress, or all NULL (search only)
 * Compression requires rows % 16 == 0 and cols % 16 == 0.
 */
SP24_API sp24_status sp24_mask_step(const void *W, sp24_dtype dtype, int64_t rows, int64_t cols, int64_t ldw,
                           uint8_t *idx, const uint8_t *idx_prev,
                           unsigned long long *d_flip_count, void *vals_row, void *meta_row,
                           void *vals_col, void *meta_col, void *stream);

/*
 * 2:4 sparse FFN forward GEMM (Software Dependencies row): Y = X * (W*m)^T.
 *   X         device [T x K] row-major, contiguous
 *   vals_row, meta_row   device, W [N x K] compressed along K (sp24_prune_compress)
 *   Y         device [T x N] row-major, contiguous
 *   epi       SP24_EPI_NONE, or SP24_EPI_GELU: Y = gelu(acc) and aux[T x N] <- acc,
 *             or SP24_EPI_GELU_DERIV: Y = gelu(acc) and aux[T x N] <- gelu'(acc),
 *             or SP24_EPI_GEGLU: Y is [T x N/2] = gelu(gate) * up for the stacked
 *             gate/up weight (N % 32 == 0) and aux[T x N] <- acc
 *   aux       device [T x N] for SP24_EPI_GELU / GEGLU / GELU_DERIV, else ignored (may be NULL)
 * fp32 accumulation; outputs rounded to dtype.  K % 16 == 0, N % 16 == 0,
 * T >= 0.  All pointers 16-byte aligned.
 */
SP24_API sp24_status sp24_gemm_fwd(const void *X, int64_t T, int64_t K, const void *vals_row,
                          const void *meta_row, int64_t N, sp24_dtype dtype, void *Y,
                          sp24_epilogue epi, void *aux, void *stream);

/*
 * 2:4 sparse FFN input-gradient GEMM: dX = dY * (W*m).  Valid as a 2:4 product
 * because the transposed mask is 2:4 as well (abstract: transposable masks).
 *   dY        device [T x N] row-major, contiguous
 *   vals_col, meta_col   device, W^T [K x N] compressed along N (sp24_prune_compress)
 *   dX        device [T x K]
 *   epi       SP24_EPI_NONE, or SP24_EPI_DGELU: dX = acc * gelu'(aux), aux [T x K],
 *             or SP24_EPI_MUL_AUX: dX = acc * aux, aux [T x K] (the derivative that
 *             SP24_EPI_GELU_DERIV stored),
 *             or SP24_EPI_DGEGLU (input gradient of the down projection of a
 *             gated FFN, acc = dH): dX is [T x 2K], the gradients of the gate
 *             and up pre-activations in the stacked layout of aux [T x 2K]
 * N % 16 == 0, K % 16 == 0.
 */
SP24_API sp24_status sp24_gemm_dgrad(const void *dY, int64_t T, int64_t N, const void *vals_col,
                            const void *meta_col, int64_t K, sp24_dtype dtype, void *dX,
                            sp24_epilogue epi, const void *aux, void *stream);

/*
 * Dense GEMM for the dense fine-tuning phase (abstract: a dense fine-tuning
 * procedure near the end of pre-training; Experiment Setup row: the last 1/6
 * of the total steps), on the same tcgen05 pipeline as the 2:4 GEMMs:
 *   out[T x M] = B[T x Kd] * A[M x Kd]^T
 * forward:        B = X  [T x K], A = W   [N x K]  (epi NONE, GELU or GELU_DERIV)
 * input gradient: B = dY [T x N], A = W^T [K x N]  (epi NONE, DGELU or MUL_AUX;
 *                 W^T from sp24_transpose)
 *   B, A, out  device, row-major, contiguous; aux as in sp24_gemm_fwd (GELU:
 *              written with the pre-activation, GELU_DERIV with gelu' of it) or
 *              sp24_gemm_dgrad (DGELU, MUL_AUX: read)
 * fp32 accumulation; outputs rounded to dtype.  Kd % 16 == 0, M % 16 == 0,
 * T >= 0.  All pointers 16-byte aligned.
 */
SP24_API sp24_status sp24_gemm_dense(const void *B, int64_t T, int64_t Kd, const void *A, int64_t M,
                            sp24_dtype dtype, void *out, sp24_epilogue epi, void *aux, void *stream);

/*
 * Dense input gradient for the dense fine-tuning phase (abstract: dense
 * fine-tuning; Experiment Setup row: the last 1/6 of the steps), with the
 * weight read as stored:
 *   dX[T x K] = dY[T x N] * W[N x K]
 * The same product as sp24_gemm_dense(dY, W^T) without forming W^T: the tensor
 * memory accelerator loads W in 64-column atoms, MN-major for the tensor cores.
 *   dY   device [T x N] row-major, contiguous (the output gradient)
 *   W    device [N x K] row-major, contiguous (the layer's weight)
 *   dX   device [T x K] row-major, contiguous, overwritten
 *   epi  NONE, DGELU or MUL_AUX; aux as in sp24_gemm_dgrad ([T x K], read)
 * fp32 accumulation; outputs rounded to dtype.  N % 16 == 0, K % 16 == 0,
 * T >= 0 (T == 0: nothing is written).  All pointers 16-byte aligned.
 */
SP24_API sp24_status sp24_gemm_dgrad_dense(const void *dY, int64_t T, int64_t N, const void *W, int64_t K,
                                  sp24_dtype dtype, void *dX, sp24_epilogue epi, const void *aux,
                                  void *stream);

/*
 * out[cols x rows] = in[rows x cols]^T for 16-bit elements (bit copy): the
 * input-gradient operand W^T of the dense fine-tuning GEMM.
 *   in, out  device, row-major, contiguous, not overlapping, 16-byte aligned;
 *            rows, cols >= 0 (any values)
 */
SP24_API sp24_status sp24_transpose(const void *in, int64_t rows, int64_t cols, sp24_dtype dtype, void *out,
                           void *stream);

/*
 * MVUE 2:4 sparsification of dY^T along tokens (the MVUE kernel of the Software
 * Dependencies row), the sparse operand of the weight-gradient GEMM.  The pages
 * name the kernel without defining it; this call computes, per column n of dY
 * and group g of four consecutive tokens, the minimum-variance unbiased
 * estimate that keeps exactly two of the four: keep probabilities
 * p_i = min(1, c |v_i|) with sum 2 and kept values v_i / p_i, drawn by
 * systematic sampling with one uniform u.  If no |v_i| reaches half the
 * group's magnitude sum S, the points u S/2 and u S/2 + S/2 on the cumulative
 * |v| sums (index order) pick two entries, kept as sign(v_i) S/2; otherwise the
 * largest |v_m| (lowest index among equal) is kept as is and the point u R on
 * the cumulative sums of the other three (sum R) picks one more, kept as
 * sign(v_k) R (R = 0: the lowest other position, as +0).  Decisions are fp64
 * operations in that order; stored values are RNE_dtype(RNE_fp32(estimate)).
 * u: the top 24 bits, times 2^-24, of the 32-bit half (g % 2) of word
 * (g % 8) / 2 of Philox4x64-10 (Salmon et al., SC 2011) at counter
 * (g / 8, n, 0, 0) and key (seed, offset): identical for a given
 * (seed, offset) on every call and device.
 *   dY    device [T x N] row-major, leading dimension ldy (ldy >= N, ldy % 8 == 0)
 *   vals, meta  device: dY^T [N x T] compressed along T, in the layout of
 *         sp24_prune_compress's row operand (sizes from
 *         sp24_compressed_size(N, T)); whole metadata chunks are written,
 *         padding with positions (0, 1)
 * T % 16 == 0, N % 8 == 0; all pointers 16-byte aligned.
 */
SP24_API sp24_status sp24_mvue_sparsify(const void *dY, int64_t T, int64_t N, int64_t ldy, sp24_dtype dtype,
                               uint64_t seed, uint64_t offset, void *vals, void *meta, void *stream);

/*
 * Weight-gradient GEMM of an FFN layer with the MVUE-sparsified output
 * gradient: dW[N x K] = Yhat[N x T] * X[T x K], Yhat = sp24_mvue_sparsify(dY)
 * (2:4 along tokens), fp32 accumulation and fp32 output in W's layout (the
 * gradient sp24_masked_decay takes).  Same tcgen05 pipeline as the other 2:4
 * GEMMs, with X read as stored (token-major) by the tensor memory accelerator.
 *   X     device [T x K] row-major, contiguous (the layer input: X for W1,
 *         the hidden activation for W2)
 *   vals, meta  device, from sp24_mvue_sparsify with the same T and N
 *   dW    device fp32 [N x K] contiguous, overwritten (zeros when T == 0)
 * T % 16 == 0, N % 16 == 0, K % 8 == 0; all pointers 16-byte aligned.
 * Tiles of 256 x 256 of dW run in waves over the device's CTA pairs (P, 74 on
 * a 148-SM B200).  When the tile count is not a multiple of P, the r tiles of
 * the last wave are split along T into s = min(P / r, 8, ceil(T / 128)) parts
 * on all P pairs; the pair with each tile's first tokens adds the other parts'
 * fp32 partial sums (in part order, so results are reproducible run to run)
 * and stores the tile.  The partial sums go through a workspace of 147,456
 * bytes per CTA plus 48 bytes of counters (2 P CTAs: about 21 MB on B200),
 * allocated with cudaMalloc by the first such call on each (device, stream)
 * and reused by later ones; a failed allocation returns SP24_ERR_CUDA.
 * Launches on one stream run in order, so they share that workspace safely.
 */
SP24_API sp24_status sp24_gemm_wgrad(const void *X, int64_t T, int64_t K, const void *vals, const void *meta,
                            int64_t N, sp24_dtype dtype, float *dW, void *stream);

/*
 * sp24_gemm_wgrad without any device allocation.  The pages have no
 * counterpart: this is a library entry point for callers that must not
 * allocate device memory inside the call, for example a process whose device
 * memory is all taken by its own allocator (a cudaMalloc there would fail), or a
 * loop that must not pay for cudaMalloc's implicit synchronization on a
 * stream's first call.  Same arguments, checks, kernel, split rule and result
 * bits as sp24_gemm_wgrad; the split tail's partial sums go through one fixed
 * scratch array in the library's static device memory instead of the
 * per-stream workspace.  It calls no cudaMalloc, cudaFree or other allocating
 * routine; it zeroes the scratch's ready counters with cudaMemsetAsync on
 * `stream` before each launch.
 *   Limit: the scratch holds the partial sums of 128 CTAs (18,874,368 bytes)
 *   and their counters (6,144 bytes).  A call whose split tail would use more,
 *   i.e. 2 * r * s > 128 for r tail tiles split s ways (see sp24_gemm_wgrad),
 *   launches nothing and returns SP24_ERR_SCRATCH_TOO_SMALL; calls without a
 *   split tail use none of it.
 *   Concurrency: every call on a device uses the same scratch, whatever its
 *   stream or host thread, so calls that overlap in time race on it and give
 *   wrong results; order them (one stream, or events between streams).
 */
SP24_API sp24_status sp24_gemm_wgrad_noalloc(const void *X, int64_t T, int64_t K, const void *vals, const void *meta,
                                    int64_t N, sp24_dtype dtype, float *dW, void *stream);

/*
 * Weight gradient and masked decay in one pass (abstract: the masked decay
 * term on gradients; Software Dependencies row: the 2:4 MMs, MVUE and masked
 * decay kernels).  dW[N x K] = Yhat * X as sp24_gemm_wgrad computes it, then,
 * in the same kernel's epilogue, dW <- dW + lambda * W where the mask of W is 0
 * (one fp32 fused multiply-add per pruned entry, as sp24_masked_decay does on
 * the stored gradient, so the result has the same bits as sp24_gemm_wgrad
 * followed by sp24_masked_decay).
 *   X, vals, meta, dW  as for sp24_gemm_wgrad (dW overwritten)
 *   W     device dtype [N x K] row-major, contiguous (the layer's weight)
 *   idx   device uint8 [N/4][K/4], the mask of W (sp24_mask_search)
 * T % 16 == 0, N % 16 == 0, K % 8 == 0; X, vals, meta, W and dW 16-byte
 * aligned.  T == 0 gives the decay of a zero gradient.  Tiles, split tail and
 * workspace as for sp24_gemm_wgrad.
 */
SP24_API sp24_status sp24_gemm_wgrad_decay(const void *X, int64_t T, int64_t K, const void *vals, const void *meta,
                                  int64_t N, sp24_dtype dtype, const void *W, const uint8_t *idx, float lambda,
                                  float *dW, void *stream);

/*
 * Dense weight-gradient GEMM for the dense fine-tuning phase (abstract: dense
 * fine-tuning; Experiment Setup row: the last 1/6 of the steps):
 * dW[N x K] = dY^T[N x T] * X[T x K], fp32 accumulation and fp32 output in W's
 * layout, on the same tcgen05 pipeline.  Both operands are read as stored (the
 * tensor memory accelerator loads them in 64-column atoms, MN-major): no
 * transpose of dY.
 *   X     device [T x K] row-major, contiguous
 *   dY    device [T x N] row-major, contiguous (the output gradient)
 *   dW    device fp32 [N x K] contiguous, overwritten (zeros when T == 0)
 * T % 16 == 0, N % 16 == 0, K % 8 == 0; all pointers 16-byte aligned.
 * Tiles, split tail and workspace as for sp24_gemm_wgrad (64 tokens per K step:
 * s <= ceil(T / 64)).
 */
SP24_API sp24_status sp24_gemm_wgrad_dense(const void *X, int64_t T, int64_t K, const void *dY, int64_t N,
                                  sp24_dtype dtype, float *dW, void *stream);

/*
 * Masked decay on gradients (abstract; masked decay kernel of the Software
 * Dependencies row): grad <- grad + lambda * W where the mask is 0, unchanged
 * where it is 1, as one fp32 fused multiply-add per pruned entry (in place).
 *   grad  device fp32 [rows x cols] contiguous;  W device dtype [rows x cols]
 *   idx   device uint8 [rows/4][cols/4];  rows % 4 == 0, cols % 4 == 0
 */
SP24_API sp24_status sp24_masked_decay(float *grad, const void *W, sp24_dtype dtype, int64_t rows,
                              int64_t cols, const uint8_t *idx, float lambda, void *stream);

/*
 * Flip count between two masks (abstract: the flip rate): *d_count is
 * overwritten with the number of the 16*nblocks mask entries that differ.
 * The flip rate is *d_count / (16 * nblocks).
 *   idx_prev, idx_cur  device uint8 [nblocks];  d_count device
 */
SP24_API sp24_status sp24_flip_rate(const uint8_t *idx_prev, const uint8_t *idx_cur, int64_t nblocks,
                           unsigned long long *d_count, void *stream);

/*
 * Maps the device metadata of an [rows x cols] matrix compressed along its
 * rows (meta_bytes from sp24_compressed_size) to the canonical form: for row
 * r, group g (columns 4g..4g+3) with kept offsets i0 < i1, the nibble
 * i0 | i1 << 2 sits at bits 4*(g % 4) of canon[r * ceil(cols/16) + g / 4].
 * Pure index permutation on host buffers; cols % 16 == 0.
 */
SP24_API sp24_status sp24_meta_to_canonical(const void *meta_dev_layout_host, int64_t rows, int64_t cols,
                                   uint16_t *canon);

/* Inverse of sp24_meta_to_canonical (host buffers); padding gets code 0x4. */
SP24_API sp24_status sp24_meta_from_canonical(const uint16_t *canon, int64_t rows, int64_t cols,
                                     void *meta_dev_layout_host);

/*
 * Synchronizes `stream`, then reads and clears the current device's error
 * word.  Returns SP24_ERR_TIMEOUT if a kernel gave up waiting since the last
 * query, SP24_ERR_CUDA if synchronization failed, else SP24_OK.  After a
 * timeout it also waits for the whole device and zeroes the counters of every
 * weight-gradient workspace of the device, which a launch that gave up may have
 * left raised; results of the calls before the query are then unspecified.
 */
SP24_API sp24_status sp24_device_status(void *stream);

/*
 * Test hook: the spin budget, in SM clock cycles, of every bounded wait in
 * the GEMM kernels on later launches (default 2^32, about 2 s).  A budget of
 * 0 makes a wait give up unless its barrier has already completed.
 */
SP24_API sp24_status sp24_set_wait_budget(uint64_t cycles);

#ifdef __cplusplus
}
#endif

#endif /* SP24_H */
