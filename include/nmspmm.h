/*
 * nmspmm.h -- C ABI of the B200 (sm_100a) N:M sparse weight x dense activation
 * GEMM library (libnmspmm.so).
 *
 * The operation is the one of "Realizable N:M Sparse Transformer Inference via
 * Search-Kernel Co-Design" (arXiv 2607.12505):
 *   - section 2.1: N:M semi-structured sparsity keeps N non-zeros in every
 *     group of M weights of the projection and FFN linears;
 *   - section 4.1: the kernel rests on three mechanisms -- weight packing for
 *     decode-friendly storage, micro-dense execution, adaptive parallelism;
 *   - section 4.2: only the N kept values of each window are materialised in
 *     dense, MMA-shaped tiles; the packed weight carries values and their
 *     in-window positions together, so no separate index load is needed.
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev are device pointers of the current CUDA device;
 *     *_host are host pointers.  The caller owns every buffer it passes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are stream-ordered and never synchronise the host unless
 *     stated.
 *   - Errors are returned as nm_status, never thrown or trapped; a message for
 *     the last failing call of the calling thread is in nm_last_error().
 *   - Layouts are row-major: W [n_out][k] (the PyTorch Linear layout),
 *     X [T][k], Y [T][n_out].
 */
#ifndef NMSPMM_H
#define NMSPMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NM_OK = 0,
    NM_ERR_INVALID = 1,     /* bad argument: null pointer, bad size, misalignment */
    NM_ERR_UNSUPPORTED = 2, /* valid request the library does not implement       */
    NM_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed                  */
    NM_ERR_OOM = 4,         /* device allocation failed                           */
    NM_ERR_TIMEOUT = 5      /* a kernel gave up a bounded wait (see nm_device_status) */
} nm_status;

typedef enum { NM_INT8 = 0, NM_FP16 = 1, NM_BF16 = 2 } nm_dtype;

/* Opaque handle holding one compressed weight; owns all device memory it allocates. */
typedef struct nm_handle nm_handle;

/*
 * nm_compress -- prune and pack one weight (paper sections 2.1 and 4.2,
 * "weight packing").
 *
 * For every row n and every group g of M consecutive k positions (aligned at
 * k = 0) keeps the N entries of largest |W|, ties to the lower position, and
 * builds two device images inside the new handle:
 *   - the canonical compressed format (see nm_export), and
 *   - the packed operand image the SpMM kernel streams: per 128-row x k-block
 *     tile, the kept values already laid out as swizzled tensor-core operand
 *     rows, followed by their 2-bit in-window positions in the layout the
 *     sparse tensor core reads.
 *
 * W_dev   [n_out][k] of dtype `dt`, 16-byte aligned.  It may be freed once the
 *         stream has passed this call.
 * (N, M)  one of (1,4), (2,4), (2,8), (4,8), or N == M with M in {4, 8}
 *         (dense pass-through).  Other pairs -> NM_ERR_UNSUPPORTED.
 * k       multiple of M (else NM_ERR_INVALID); n_out, k > 0, at most 2^24;
 *         for NM_INT8 k at most 2^17 (so that k * 128 * 127 fits the int32
 *         accumulator exactly), else NM_ERR_UNSUPPORTED.
 * out     receives the handle; *out is NULL on failure.
 * Allocates device memory (NM_ERR_OOM on failure); returns without waiting
 * for the kernels.
 */
nm_status nm_compress(const void* W_dev, int64_t n_out, int64_t k, nm_dtype dt, int N, int M,
                      void* stream, nm_handle** out);

/*
 * nm_spmm_noalloc -- the same product as nm_spmm for callers that cannot
 * allocate device memory.  (The paper has no counterpart: this is a
 * deployment variant.)  Such callers include serving engines that hand
 * nearly all of HBM to their own pool up front, so a library cudaMalloc would
 * fail, and latency-critical code that must not call cudaMalloc/cudaFree,
 * which can synchronise the device and take a process-wide lock.
 *
 * Arguments, layouts, rounding and results are those of nm_spmm.  The
 * difference is where the scratch of a global-memory split-K (partial tiles
 * and per-tile arrival counters) lives: in one fixed array inside the
 * library, 4 MiB of partials plus 1024 counters.  Every GPU that loads the
 * library holds that array until the process exits.  This call never calls
 * cudaMalloc, cudaFree or any allocating routine.
 *   - The planner's own plans never use the array: they either do not split
 *     k or reduce the splits on chip (see nm_spmm).  Only a global-memory
 *     split forced through the environment (NMSPMM_FORCE_SPLITK with
 *     NMSPMM_SPLIT_GLOBAL=1, or more than 8 splits) uses it, and only then do
 *     the size limit and the race below apply.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (set-up, once per device, with that device
 *     current); make that first call before any stream capture.
 *   - A shape whose split-K plan needs more than the array holds is rejected
 *     with NM_ERR_UNSUPPORTED and a message naming the sizes; nm_spmm handles
 *     it instead.
 *   - All calls share the array and it keeps the last call's contents; each
 *     call clears the counters it uses (an asynchronous memset on `stream`).
 *     Calls whose kernels overlap on the GPU (different streams, or different
 *     host threads) race on the array: order them.
 */
nm_status nm_spmm_noalloc(const nm_handle* h, const void* X_dev, int64_t T, void* Y_dev,
                          const float* scale_dev, void* stream);

/*
 * nm_recompress -- prune and pack a new weight of the handle's shape, dtype and
 * N:M into the handle's existing device buffers (a weight update; same rule
 * and layouts as nm_compress).  Allocates nothing; stream-ordered, so an
 * nm_spmm on the same stream afterwards sees the new weight.  W_dev element
 * aligned, [n_out][k].
 */
nm_status nm_recompress(nm_handle* h, const void* W_dev, void* stream);

/*
 * nm_spmm -- Y = X . Wm^T with Wm the masked weight of `h` (paper section 4.2,
 * micro-dense execution; section 4.1, adaptive parallelism).
 *
 * X_dev     [T][k] of the handle's dtype, 16-byte aligned, k * sizeof(dtype)
 *           a multiple of 16 bytes (else NM_ERR_UNSUPPORTED).
 * Y_dev     [T][n_out]:
 *             INT8, scale_dev == NULL : int32, exact integer result;
 *             INT8, scale_dev != NULL : float32, (float)acc * scale[n]
 *                                       (round-to-nearest, one multiply);
 *             FP16/BF16               : same dtype as X, rounded to nearest
 *                                       once from the fp32 accumulator
 *                                       (times scale[n] when given).
 *           Must be 16-byte aligned and must not overlap X.
 * scale_dev float32 [n_out] or NULL.
 * T         >= 0; T == 0 is a no-op returning NM_OK.
 * The kernel, token tile and split-K factor are chosen per (T, k, n_out,
 * N:M, dtype) so that small token counts still occupy the SMs (section 4.1,
 * mechanism 3; nm_plan_query reports the choice).  A split chosen by the
 * planner puts the k-splits of one output tile on the CTAs of one
 * thread-block cluster, which sum their partial tiles through distributed
 * shared memory: no workspace, no allocation.  A global-memory split-K
 * (forced through the environment: NMSPMM_FORCE_SPLITK with
 * NMSPMM_SPLIT_GLOBAL=1, or more than 8 splits) uses the handle's workspace:
 * calls on one handle must then not overlap on the GPU, and the first such
 * call allocates the workspace (after a device synchronisation; make it
 * before any stream capture).  Otherwise never synchronises.
 */
nm_status nm_spmm(const nm_handle* h, const void* X_dev, int64_t T, void* Y_dev,
                  const float* scale_dev, void* stream);

/*
 * Fused output stage of nm_spmm_ex.  The paper stops at the MMA (section 4.2)
 * and does not discuss the output stage; this is the library's definition.
 * Per output element, in fp32, each step rounded to nearest:
 *   v = acc                         INT8: (float)acc; FP16/BF16: the fp32 sum
 *   v = v * scale[n]                if scale != NULL
 *   v = v + bias[n]                 if bias != NULL
 *   v = v/2 * (1 + erf(v/sqrt 2))   if act == NM_ACT_GELU (erf form of GELU)
 * then stored as the output type:
 *   NM_OUT_FP32                     v
 *   NM_OUT_FP16 / NM_OUT_BF16       v rounded to nearest even
 *   NM_OUT_INT8                     clamp(round_half_even(v * out_scale), -128, 127)
 *   NM_OUT_INT32                    the raw INT8 accumulator (no scale, bias
 *                                   or activation allowed)
 *   NM_OUT_DEFAULT                  INT8: INT32 when scale, bias and act are
 *                                   all absent, else FP32; FP16/BF16: the
 *                                   input's type.
 * With act == NM_ACT_NONE and an INT8 handle the result is exactly fixed.  The
 * GELU evaluates erf by formula 7.1.26 of Abramowitz and Stegun (absolute error
 * at most 1.5e-7) with the GPU's approximate reciprocal and power of two; the
 * GELU value g of a pre-activation v is within 4e-7 |v| + 2e-6 |GELU(v)| of the
 * exact one.
 */
typedef enum {
  NM_OUT_DEFAULT = 0,
  NM_OUT_INT32 = 1,
  NM_OUT_FP32 = 2,
  NM_OUT_FP16 = 3,
  NM_OUT_BF16 = 4,
  NM_OUT_INT8 = 5
} nm_out_type;

typedef enum { NM_ACT_NONE = 0, NM_ACT_GELU = 1 } nm_act;

typedef struct nm_epilogue {
  nm_out_type out;     /* element type of Y */
  nm_act act;          /* activation after scale and bias */
  const float* scale;  /* device float32 [n_out], 4-byte aligned, or NULL */
  const float* bias;   /* device float32 [n_out], 4-byte aligned, or NULL */
  float out_scale;     /* NM_OUT_INT8 only: multiplier before rounding; finite and > 0 */
} nm_epilogue;

/*
 * nm_spmm_ex -- nm_spmm with the fused output stage above: Y = out(act(
 * (X . Wm^T) * scale + bias)).  Arguments, alignment, the no-op for T == 0,
 * the workspace rule and the never-synchronise rule are those of nm_spmm; Y_dev
 * holds elements of the chosen output type.  ep == NULL is nm_spmm with no
 * scale.
 * Errors: NM_ERR_INVALID for an unknown out/act value, NM_OUT_INT32 together
 * with scale, bias or act, a misaligned scale/bias, or NM_OUT_INT8 with an
 * out_scale that is not finite and positive; NM_ERR_UNSUPPORTED for
 * NM_OUT_INT32 or NM_OUT_INT8 on an FP16/BF16 handle.
 */
nm_status nm_spmm_ex(const nm_handle* h, const void* X_dev, int64_t T, void* Y_dev,
                     const nm_epilogue* ep, void* stream);

/*
 * nm_compress_tile -- prune and pack one weight with a pattern shared by each
 * tile of 128 consecutive output channels (the vector-wise reading of the
 * paper's section 4.2: kept values become dense MMA tiles and the activations
 * are gathered to match, which needs one set of kept positions per tile of
 * channels).
 *
 * For every tile of rows [128t, 128t + 128) (the last may be shorter) and
 * every group g of M consecutive k positions, the score of position p is
 * sum over the tile's rows of |W[n][gM + p]|, computed exactly; the N
 * positions of largest score are kept, ties to the lower position, and every
 * row of the tile keeps them.  The handle holds the canonical format (exactly
 * as nm_compress lays it out, nm_export) and a dense operand image over the
 * kept k only (K' = k * N / M per row) plus the tile's kept k list, which
 * nm_spmm_gather uses to gather rows of the activation.
 *
 * Arguments as nm_compress, except:
 *   dt      NM_INT8 or NM_FP16 (scores of bfloat16 weights are not exact in
 *           any fixed-width sum: NM_ERR_UNSUPPORTED);
 *   (N, M)  one of (1,4), (2,4), (2,8), (4,8), or N == M with M in {4, 8}.
 * nm_recompress, nm_decompress, nm_export, nm_query and nm_destroy accept the
 * handle; nm_spmm, nm_spmm_ex and nm_spmm_noalloc reject it (NM_ERR_INVALID):
 * its product is nm_spmm_gather.
 */
nm_status nm_compress_tile(const void* W_dev, int64_t n_out, int64_t k, nm_dtype dt, int N, int M,
                           void* stream, nm_handle** out);

/*
 * nm_spmm_gather -- Y = X . Wm^T for a handle made by nm_compress_tile, with
 * the activation given feature-major: Xt_dev [k][ldx] holds X[t][kk] at
 * Xt_dev[kk * ldx + t].  Per 128-channel tile the kernel gathers the kept rows
 * of Xt (16-byte asynchronous copies, eight threads per 128-byte token run)
 * into a dense operand and runs dense tensor-core MMAs over K' = k * N / M
 * only, so both the MMA work and the activation bytes read per tile shrink by
 * N / M.  Environment NMSPMM_GATHER_TMA=1 gathers with four-row tensor copies
 * instead (same results; slower on B200).
 *
 * Xt_dev    16-byte aligned; ldx >= T and ldx * sizeof(dtype) a multiple of
 *           16 bytes (else NM_ERR_INVALID).  Columns t >= T are not read.
 * Y_dev     [T][n_out], 16-byte aligned, not overlapping Xt; element type and
 *           rounding exactly as nm_spmm (INT8: int32, or float32 with scale;
 *           FP16: fp16 from the fp32 accumulator).
 * scale_dev float32 [n_out] or NULL.
 * T         >= 0; T == 0 is a no-op.
 * The default plan never splits k, so the call allocates nothing and never
 * synchronises; a split-K plan forced through NMSPMM_FORCE_SPLITK reduces in
 * global memory and uses the handle's workspace under the rules of nm_spmm
 * (the first such call allocates it, after a device synchronisation).
 */
nm_status nm_spmm_gather(const nm_handle* h, const void* Xt_dev, int64_t ldx, int64_t T, void* Y_dev,
                         const float* scale_dev, void* stream);

/*
 * nm_spmm_gather_ex -- nm_spmm_gather with the fused output stage of
 * nm_spmm_ex (nm_epilogue above): Y = out(act((X . Wm^T) * scale + bias)), the same
 * definition, element types, rounding and argument checks as nm_spmm_ex; the
 * activation arguments (Xt_dev, ldx, T) and their checks are those of
 * nm_spmm_gather.  ep == NULL is nm_spmm_gather without a scale.
 */
nm_status nm_spmm_gather_ex(const nm_handle* h, const void* Xt_dev, int64_t ldx, int64_t T, void* Y_dev,
                            const nm_epilogue* ep, void* stream);

/*
 * nm_decompress -- write the masked dense weight Wm [n_out][k] (dtype of the
 * handle) decoded from the packed operand image the SpMM kernel reads, so the
 * image can be checked against the top-N rule.  W_dev_out 16-byte aligned.
 */
nm_status nm_decompress(const nm_handle* h, void* W_dev_out, void* stream);

/*
 * nm_export -- copy the canonical compressed format to the host.  Synchronises
 * the device.
 *   values_host: [n_out][k/M][N] elements of the weight dtype, kept values in
 *                ascending in-group position (nm_export_sizes gives bytes);
 *   idx_host:    [n_out][idx_pitch] bytes, one 4-bit in-group position per
 *                kept element in the same order, two per byte, low nibble
 *                first; idx_pitch = ceil(N * k / M / 2) so rows never share a
 *                byte.  For N == M, positions are 0..M-1.
 */
nm_status nm_export(const nm_handle* h, void* values_host, uint8_t* idx_host);
nm_status nm_export_sizes(const nm_handle* h, size_t* values_bytes, size_t* idx_bytes);

/*
 * nm_plan_query -- the launch plan nm_spmm (scaled != 0: with a scale; the
 * INT8 fp32-output kernels) would use for T tokens on the current device,
 * without launching anything (section 4.1, mechanism 3, adaptive
 * parallelism).  For a handle from nm_compress_tile it is nm_spmm_gather's
 * plan.  Environment overrides (NMSPMM_FORCE_*) apply as they would to the
 * call.  T > 0, else NM_ERR_INVALID.
 */
typedef struct nm_plan_info {
  int pair;     /* 1: two-SM kernel (M = 256 per MMA, grid counts CTA pairs) */
  int bn;       /* token tile (MMA N) */
  int splits;   /* k-splits per output tile (1: none) */
  int cluster;  /* 1: the splits of a tile are one cluster, reduced on chip */
  int grid;     /* CTAs launched (CTA pairs for the two-SM kernel) */
  int units;    /* (tile, split) work units */
} nm_plan_info;
nm_status nm_plan_query(const nm_handle* h, int64_t T, int scaled, nm_plan_info* out);

/*
 * nm_plan_for_shape -- test and diagnostic hook (no counterpart in the paper):
 * the plan nm_plan_query would report for a handle of this shape (nm_compress
 * with dt, n_out, k, N, M) and T tokens on a GPU with `sms` SMs whose
 * resident-cluster capacities are given instead of queried, so the planner's
 * rules can be checked without a GPU.  Touches no device and allocates
 * nothing.
 *
 * pair_clusters    int[3]: CTA pairs of the two-SM kernel that fit on the GPU
 *                  at the token tiles 224, 192 and 128 (<= 0: that tile cannot
 *                  run); nm_plan_query queries these from the device for the
 *                  output the call would write.
 * stream_clusters  int[8]: clusters of S one-SM CTAs that fit, S = 1 .. 8
 *                  (<= 0: none).
 * The NMSPMM_FORCE_* environment overrides apply as in nm_spmm.  Errors:
 * NM_ERR_INVALID for null pointers, a bad dtype, shape, T or sms;
 * NM_ERR_UNSUPPORTED for an N:M nm_compress rejects.
 */
nm_status nm_plan_for_shape(nm_dtype dt, int64_t n_out, int64_t k, int N, int M, int64_t T, int sms,
                            const int* pair_clusters, const int* stream_clusters, nm_plan_info* out);

/* nm_query -- shape and format of a handle; any output pointer may be NULL. */
nm_status nm_query(const nm_handle* h, int64_t* n_out, int64_t* k, int* N, int* M, nm_dtype* dt);

/*
 * nm_device_status -- read (and clear) the handle's device error word, which a
 * kernel sets instead of trapping when a bounded wait runs out.  Synchronises
 * the device.  Returns NM_OK or NM_ERR_TIMEOUT.
 */
nm_status nm_device_status(const nm_handle* h);

/* nm_destroy -- free the handle and its device memory (synchronises). NULL is a no-op. */
void nm_destroy(nm_handle* h);

/* nm_last_error -- message of the calling thread's last failing call ("" if none). */
const char* nm_last_error(void);

/* nm_version -- library version string. */
const char* nm_version(void);

/*
 * Test hook (no counterpart in the paper): run nm_spmm with the SpMM kernel's
 * producer leaving pipeline stage number `skip_stage` (counted over the CTA's
 * whole run) unfilled, and every bounded wait limited to `timeout_ns`
 * (0 < timeout_ns <= 2e9).  The MMA warp's wait on that stage then runs out:
 * the kernel records the timeout in the handle's error word, drains its own
 * copies and MMAs, frees its tensor memory and returns, so the context stays
 * usable.  Exists so tests can exercise the failure path without faulting or
 * hanging a GPU; Y is left partially written.
 */
nm_status nm_test_spmm_skip_stage(const nm_handle* h, const void* X_dev, int64_t T, void* Y_dev,
                                  const float* scale_dev, void* stream, int skip_stage, int64_t timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* NMSPMM_H */
