/*
 * ar_rmsnorm.h -- C ABI of the fused "W-way reduce + residual add + RMSNorm"
 * library for NVIDIA B200 (sm_100a).
 *
 * The operation is the step that closes a tensor-parallel transformer
 * sub-layer: the all-reduce of the ranks' partial activations, the residual
 * add, and RMSNorm.  Here the W partials already sit on one GPU, so the
 * all-reduce is a W-way elementwise sum done inside the same kernel as the
 * add and the norm.
 *
 * Passages defining the operations (vLLM pull-request reports on
 * prhub.com.cn; page title, then section):
 *   - PR #54787 report (ROCm AITER fused allreduce+RMSNorm fast path),
 *     "关键源码片段": fused_allreduce_gemma_rms_norm returns
 *     (norm_out, residual_out); its fallback is all_reduce followed by
 *     GemmaRMSNorm(reduced, residual); gemma_norm selects weight bias 1.0;
 *     the one-stage predicate is capture-static (depends only on shape,
 *     dtype and world size).
 *   - PR #50802 report (AITER add-RMSNorm dead-residual fusion),
 *     "实现拆解" and "关键源码片段": the output-only pattern keeps only the
 *     RMSNorm result; the no-residual all_reduce -> rms_norm site; the
 *     per-group FP8 quantisation of the normalised output, with the bf16
 *     normalised output also kept for a second consumer.
 *   - PR #44849 report ([ROCm][MiniMax-M2] fused QK-norm + AllReduce),
 *     "关键源码片段": _minimax_qk_norm_fusion(qkv, q_weight, k_weight,
 *     q_size, kv_size, tp_rank, tp_world, eps, ...) normalises q and k over
 *     their full width across the TP shards.
 *   - PR #49673 report (token count fix for 3-D inputs), "实现拆解": the
 *     token count is numel / hidden_dim; here T is passed explicitly and
 *     callers flatten leading dimensions.
 *
 * Conventions for every entry point:
 *   - All tensor arguments are caller-owned DEVICE pointers to contiguous
 *     row-major memory on the current CUDA device.  Pointer arrays
 *     (`partials`, `qkv`, `q_out`, `k_out`) are HOST arrays of W device
 *     pointers; they are copied by value into the kernel's parameters, so the
 *     host array may be reused as soon as the call returns.
 *   - The library allocates nothing per call, never synchronises, and
 *     launches on `stream`; calls are asynchronous and may be captured in a
 *     CUDA graph once the device has been used by one call outside capture
 *     (the first call on a device reads its attributes and sets kernel
 *     attributes).
 *   - Errors are returned synchronously as ar_status and nothing is
 *     launched; there is no silent no-op and no hidden fallback.  T == 0 is
 *     valid and launches nothing.  Faults inside a kernel surface as CUDA
 *     errors on `stream`, as for any kernel.
 *   - 16-bit formats: AR_BF16 (bfloat16) or AR_FP16 (IEEE half); all 16-bit
 *     tensors of one call share `dtype`.
 *   - Arithmetic is fp32.  The W+1 terms are summed with a certificate:
 *     a plain fp32 sum is kept when its rounding-error bound is below
 *     2^-(p+2) of the result (p = 8 for bf16, 11 for fp16 outputs), and
 *     otherwise the element is recomputed with an error-free (TwoSum)
 *     compensated sum.  The FP8 variant sums exactly: the fp32 sum rounded
 *     down and rounded up agree exactly when it is exact, and elements where
 *     they differ take the compensated sum.
 *     residual_out is therefore within one unit in the last place of the
 *     rounded exact sum.  The sum of squares is combined across threads in
 *     fp64 for the FP8 variant (its scales must be within 1e-6) and in fp32
 *     otherwise.  Outputs are rounded to nearest even.
 */
#ifndef AR_RMSNORM_H
#define AR_RMSNORM_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define AR_API __attribute__((visibility("default")))
#else
#define AR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AR_OK = 0,
    AR_EINVAL = 1,        /* null required pointer, bad size or count       */
    AR_EALIGN = 2,        /* a device pointer is not 16-byte aligned         */
    AR_EUNSUPPORTED = 3,  /* device is not sm_100, or a size beyond limits   */
    AR_ECUDA = 4,         /* a CUDA runtime call or launch failed            */
    AR_ETIMEDOUT = 5      /* reserved for bounded device waits               */
} ar_status;

typedef enum { AR_BF16 = 0, AR_FP16 = 1 } ar_dtype;

/* Largest supported hidden size (elements) and number of partials. */
#define AR_MAX_H 65536
#define AR_MAX_W 16

/*
 * ar_add_rmsnorm -- two-output, output-only and no-residual forms.
 *
 *   r[t,h] = residual[t,h] + sum_{w<W} partials[w][t,h]
 *   y[t,h] = r[t,h] * rsqrt(mean_h(r[t,:]^2) + eps) * (gemma ? 1 + weight[h]
 *                                                          : weight[h])
 *   out[t,h]          = RNE_dtype(y[t,h])
 *   residual_out[t,h] = RNE_dtype(r[t,h])
 *
 * partials      host array of W device pointers, each [T, H] in `dtype`
 * residual      [T, H] or NULL (NULL: r is the plain sum, the no-residual
 *               form all_reduce -> rms_norm)
 * weight        [H]
 * out           [T, H], written
 * residual_out  [T, H] or NULL (NULL: the dead-residual / output-only form;
 *               nothing is written).  residual_out == residual (in place) is
 *               allowed; any other overlap between outputs and inputs is
 *               undefined.
 * T             tokens (rows), >= 0
 * H             hidden size, multiple of 8, 8 <= H <= AR_MAX_H
 * W             number of partials, 1 <= W <= AR_MAX_W
 * eps           finite, >= 0; added to the mean of squares inside the rsqrt
 * gemma         0: weight w;  1: weight (1 + w), the Gemma RMSNorm variant
 * dtype         AR_BF16 or AR_FP16
 * Alignment: every pointer 16-byte aligned (AR_EALIGN otherwise).
 */
AR_API int ar_add_rmsnorm(const void *const *partials, const void *residual,
                   const void *weight, void *out, void *residual_out,
                   int64_t T, int64_t H, int W, float eps, int gemma,
                   int dtype, cudaStream_t stream);

/*
 * ar_add_rmsnorm_quant_fp8_group -- the same r and y, then per-group FP8.
 * (PR #50802 report: all_reduce -> add -> RMSNorm -> per-group FP8 quant,
 * with the 16-bit normalised output kept for a second consumer.)
 *
 * For each group g of `group` consecutive elements of a row, with y in fp32:
 *   amax          = max |y| over the group
 *   scales[t,g]   = amax / 448                  (IEEE fp32 division)
 *   out_fp8[t,h]  = e4m3fn_RNE_satfinite(y[t,h] / scales[t,g]),
 *                   0 for every element when amax == 0
 * out_fp8       [T, H] bytes, OCP e4m3fn codes (1-4-3, bias 7, max 448)
 * scales        [T, H/group] fp32, row-major (any layout: the _strided call)
 * out_y         [T, H] in `dtype` (RNE of y) or NULL
 * residual_out  [T, H] in `dtype` or NULL, as in ar_add_rmsnorm
 * group         must be 128; H must be a multiple of it
 * Other arguments as in ar_add_rmsnorm.  scales needs 4-byte alignment, all
 * other pointers 16-byte alignment.
 */
AR_API int ar_add_rmsnorm_quant_fp8_group(const void *const *partials,
                                   const void *residual, const void *weight,
                                   void *out_fp8, float *scales, void *out_y,
                                   void *residual_out, int64_t T, int64_t H,
                                   int W, int group, float eps, int gemma,
                                   int dtype, cudaStream_t stream);

/*
 * ar_add_rmsnorm_quant_fp8_group_strided -- as ar_add_rmsnorm_quant_fp8_group
 * with any scales layout: scales[t, g] lives at
 *   scales[t * scale_stride_t + g * scale_stride_g]   (elements).
 * Row-major [T, H/group] is (H/group, 1); the transposed [H/group, T] layout
 * is (1, T).  The strides must be >= 0 and give every (t, g) its own slot
 * (row-major-like: stride_g >= 1 and stride_t >= (H/group) * stride_g, or
 * column-major-like: stride_t >= 1 and stride_g >= T * stride_t; one of
 * them may be anything when T or H/group is 1), else AR_EINVAL.
 */
AR_API int ar_add_rmsnorm_quant_fp8_group_strided(const void *const *partials,
                                   const void *residual, const void *weight,
                                   void *out_fp8, float *scales,
                                   int64_t scale_stride_t, int64_t scale_stride_g,
                                   void *out_y, void *residual_out, int64_t T,
                                   int64_t H, int W, int group, float eps,
                                   int gemma, int dtype, cudaStream_t stream);

/*
 * qk_norm_sharded -- MiniMax-style QK-norm over W tensor-parallel shards.
 * (PR #44849 report: q and k of each shard are normalised over the full
 * q (k) width; the only cross-shard quantity is a token's sum of squares.)
 *
 * qs = q_size / W, ks = kv_size / W.  Shard w's buffer qkv[w] is [T, qs+2ks]
 * with row layout [ q_w | k_w | v_w ].  For each token t:
 *   inv_q = rsqrt(sum_{w,j} q_w[t,j]^2 / q_size + eps)
 *   inv_k = rsqrt(sum_{w,j} k_w[t,j]^2 / kv_size + eps)
 *   q_out[w][t,j] = RNE(q_w[t,j] * inv_q * q_weight[w*qs + j])
 *   k_out[w][t,j] = RNE(k_w[t,j] * inv_k * k_weight[w*ks + j])
 * v is neither read nor written.
 *
 * qkv       host array of W device pointers, each [T, qs + 2*ks]
 * q_weight  [q_size];  k_weight [kv_size]  (full vectors; shard w uses its
 *           slice)
 * q_out     host array of W device pointers, each [T, qs], dense
 * k_out     host array of W device pointers, each [T, ks], dense
 *           In-place form: q_out[w] == qkv[w] and k_out[w] == qkv[w] + qs
 *           (elements) for every w.  The outputs then have qkv's row stride
 *           and overwrite the q and k columns; v is untouched.  A call
 *           that uses this form for some shards but not all returns
 *           AR_EINVAL.  (Each row is read completely before it is written.)
 * Requirements: 1 <= W <= AR_MAX_W, q_size and kv_size positive multiples
 * of W with qs and ks multiples of 8, qs + ks <= AR_MAX_H, pointers 16-byte
 * aligned; apart from the in-place form, outputs do not overlap inputs.
 */
AR_API int qk_norm_sharded(const void *const *qkv, const void *q_weight,
                    const void *k_weight, void *const *q_out,
                    void *const *k_out, int64_t T, int64_t q_size,
                    int64_t kv_size, int W, float eps, int dtype,
                    cudaStream_t stream);

/*
 * Dispatch plans.  Each call picks a kernel configuration ("plan") from a
 * table of measured timings keyed by (variant, dtype, W, H, T range), and
 * falls back to a built-in rule for shapes the table does not cover.  The
 * choice depends only on these arguments and the loaded table, never on
 * data or device state, so it is the same during CUDA-graph capture as
 * outside it (the PR #54787 report's "capture-static" property).
 */
typedef enum { AR_VARIANT_NORM = 0, AR_VARIANT_FP8 = 1, AR_VARIANT_QK = 2 } ar_variant;

/* Plan ids.
 *   ROWC<k>           one row per cluster of k CTAs; the sum of squares is
 *                     combined through distributed shared memory.
 *   PERSIST           one CTA of at most 256 threads per row; persistent grid
 *                     (SM count x occupancy), rows looped.  Where a thread's
 *                     share of a row fits the register budget (at most 10
 *                     16-byte packs: packs per thread x (W + 1)) the CTA's
 *                     next row is loaded into registers while the current
 *                     one is finished; otherwise it is bulk-prefetched into
 *                     L2.
 *   PERSIST_AHEAD     the same with at most 512 threads (fewer packs per
 *                     thread, so the register load-ahead applies to wider
 *                     rows).
 *   PERSIST_C2_AHEAD  PERSIST_AHEAD with each row split over a cluster of 2
 *                     CTAs; the grid is the number of clusters that fit at
 *                     once.
 *   PERSIST512        persistent, at most 512 threads, two CTAs per SM
 *                     (registers for two CTAs, so no load-ahead); each CTA's
 *                     next row is bulk-prefetched into L2.
 *   PERSIST_C2        PERSIST512 with each row split over a cluster of 2
 *                     CTAs.
 *   BULK              rows staged into shared memory by bulk asynchronous
 *                     copies.
 *   QK_C<k>           one token per cluster of k CTAs, shards split across
 *                     the cluster.
 *   QK_PERSIST        one CTA of at most 512 threads per token, persistent
 *                     grid with L2 prefetch.
 *   QK_PERSIST256     the same with at most 256 threads (more packs per
 *                     thread).
 *   QK_BULK           one persistent CTA per SM; one thread keeps up to 16
 *                     tokens in flight into a shared-memory ring with bulk
 *                     asynchronous copies (one per shard row), and whole
 *                     warps normalise one token each from it (falls back to
 *                     QK_PERSIST where two tokens and the weights do not fit
 *                     in shared memory).
 *   QK_RING           every shard of a token in one CTA of at most 256
 *                     threads, persistent, two tokens per step (one
 *                     reduction for their four sums of squares); each thread
 *                     keeps its packs of the four tokens after the current
 *                     pair in flight as 16-byte asynchronous copies into a
 *                     six-token shared-memory ring (falls back to QK_PERSIST
 *                     for tokens wider than 1024 packs). */
enum {
    AR_PLAN_AUTO = 0,
    AR_PLAN_ROWC1 = 1,
    AR_PLAN_ROWC2 = 2,
    AR_PLAN_ROWC4 = 3,
    AR_PLAN_ROWC8 = 4,
    AR_PLAN_PERSIST = 5,
    AR_PLAN_BULK = 6,
    AR_PLAN_PERSIST512 = 7,
    AR_PLAN_PERSIST_C2 = 8,
    AR_PLAN_PERSIST_AHEAD = 9,
    AR_PLAN_PERSIST_C2_AHEAD = 10,
    AR_PLAN_QK_C1 = 11,
    AR_PLAN_QK_C2 = 12,
    AR_PLAN_QK_C4 = 13,
    AR_PLAN_QK_C8 = 14,
    AR_PLAN_QK_PERSIST = 15,
    AR_PLAN_QK_PERSIST256 = 16,
    AR_PLAN_QK_BULK = 17,
    AR_PLAN_QK_RING = 18
};

/* The plan a call with these arguments would use (for QK, H = q_size + kv_size
 * per token, W the shard count).  Writes *plan_id; returns AR_EINVAL for a bad
 * variant, dtype or null plan_id. */
AR_API int ar_plan_query(int variant, int64_t T, int64_t H, int W, int dtype,
                  int *plan_id);

/* Load a plan table (JSON: {"entries": [{"variant":v, "dtype":d, "W":w,
 * "H":h, "t_lo":a, "t_hi":b, "plan":p}, ...]}).  The table replaces the
 * loaded one only if the whole file parses and every plan id is valid for
 * its variant; otherwise AR_EINVAL is returned and the previous table stays.
 * path == NULL clears the table (built-in rule only).  Not safe to call
 * concurrently with launches on other threads. */
AR_API int ar_plan_load(const char *path);

/* Force `plan_id` for every call of `variant` (AR_PLAN_AUTO clears).  For A/B
 * measurement; AR_EINVAL for an id that does not belong to the variant. */
AR_API int ar_plan_force(int variant, int plan_id);

/*
 * Device-side status.  The bulk-staged kernel (AR_PLAN_BULK) bounds every
 * wait on its copy pipeline; a wait that sees no progress for one second
 * makes the kernel record AR_ETIMEDOUT here and wind down (its outputs for
 * the affected rows are then undefined).  ar_device_status synchronises the
 * current device, returns AR_ETIMEDOUT if any launch on it recorded a timeout
 * since the last clear (AR_OK otherwise, AR_ECUDA if the device could not be
 * read), and clears the record when `clear` is non-zero.
 */
AR_API int ar_device_status(int clear);

/*
 * Test hook for the bounded waits: the next bulk-staged launch on any device
 * never issues the copies of row `row` (>= 0), so that row's consumers wait
 * out their limit; -1 (the default) disables it.  The hook resets itself
 * after one launch.  It exists so failure handling can be tested without a
 * GPU fault; production code never sets it.
 */
AR_API int ar_test_withhold_row(int64_t row);

/* Number of table entries currently loaded. */
AR_API int ar_plan_table_size(void);

/* Static description of a status code. */
AR_API const char *ar_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* AR_RMSNORM_H */
