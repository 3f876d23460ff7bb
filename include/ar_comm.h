/*
 * ar_comm.h -- C ABI of the multi-GPU form: the all-reduce of the ranks'
 * partial activations fused with the residual add and RMSNorm (and its
 * per-group FP8 output), and the sharded QK-norm, across W ranks with one
 * GPU each.
 *
 * Passages defining the operations (vLLM pull-request reports on
 * prhub.com.cn; page title, then section):
 *   - PR #54787 report (ROCm AITER fused allreduce+RMSNorm fast path):
 *     "功能与动机" -- the fused all-reduce + (Gemma)RMSNorm replaces the
 *     unfused all_reduce followed by the norm (post-attention step about
 *     12.5 us -> 7.5 us on their hardware); "实现拆解" items 1 and 4 -- a
 *     one-stage kernel for small token counts, a two-stage one beyond, the
 *     choice made from shape and world size only (capture-static) and only
 *     where it measured profitable; "评论区精华" items 3-4 -- the two-stage
 *     slowdown traced to writing the reduced slice into a temporary buffer
 *     (push), fixed by reading peers' data (pull).
 *   - PR #44849 report ([ROCm][MiniMax-M2] fused QK-norm + AllReduce),
 *     "关键源码片段": q and k of every rank's shard are normalised over the
 *     full width, the only cross-rank quantity being a token's sums of
 *     squares; the unfused fallback all-reduces them and normalises locally.
 *   - PR #50802 report: the dead-residual, no-residual and per-group FP8
 *     forms, as in ar_rmsnorm.h.
 *
 * Arithmetic.  Every rank computes r = residual + sum over ranks w = 0..W-1
 * of partial_w, in rank order, with the same certified (16-bit outputs) or
 * exact (FP8) summation as ar_add_rmsnorm, so the results are identical
 * (bit for bit) on every rank and equal to ar_add_rmsnorm's on one GPU with
 * the W partials given in rank order.  The QK form sums the ranks' partial
 * sums of squares in rank order in fp32.
 *
 * Transport.  Each rank owns one device region (allocated once, at
 * creation): arrival flags, counters, two staging slots and two gather
 * slots.  The other ranks map it through CUDA IPC handles, which the caller
 * exchanges (ar_comm_handle / ar_comm_open), e.g. with torch.distributed.
 * A call's kernel first copies this rank's partial rows into its staging
 * slot, then meets the other ranks at a barrier (per CTA: a release store
 * into each peer's flag, an acquire wait on its own flags), then reads the
 * peers' rows with plain loads over NVLink ("pull").  No bulk or TMA copy
 * and no multicast ever touches another GPU's memory.
 *   one-shot  every rank pulls all rows of every rank and normalises every
 *             row (small token counts: one barrier, replicated work);
 *   two-shot  rank r owns rows [r*ceil(T/W), (r+1)*ceil(T/W)): it pulls only
 *             those rows from every rank and normalises them
 *             (reduce-scatter + norm), leaves the results in its gather
 *             slot, meets the others again, and pulls the rows it does not
 *             own from their owners (all-gather): about 2(W-1)/W of the
 *             bytes per rank instead of (W-1).
 * Waits are bounded: a wait that sees no arrival for the communicator's
 * timeout gives up, the kernel finishes with the same control flow (its
 * outputs are then undefined) and ar_comm_status reports AR_ETIMEDOUT; the
 * communicator should then be destroyed.  No call ever hangs a GPU.
 *
 * Ordering.  The calls of one communicator must be issued in the same order
 * on every rank, with the same T, H, dtype and algorithm, each rank's calls
 * on one stream (like a collective).  Calls are asynchronous and may be
 * captured in CUDA graphs after one call outside capture.
 */
#ifndef AR_COMM_H
#define AR_COMM_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#include "ar_rmsnorm.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ar_comm ar_comm;   /* opaque */

/* Bytes of one rank's handle record (IPC handle + consistency record). */
#define AR_COMM_HANDLE_BYTES 128

typedef enum { AR_ALGO_AUTO = 0, AR_ALGO_ONESHOT = 1, AR_ALGO_TWOSHOT = 2 } ar_algo;

/*
 * ar_comm_create -- this rank's communicator on the current device.
 * rank in [0, world), 1 <= world <= AR_MAX_W.  max_elems bounds T*H of every
 * call (>= 8); the region is about 14 * max_elems bytes (two staging slots of
 * 2 bytes per element, two gather slots of 5 bytes and a scale per 128).
 * The region is allocated and zeroed here (synchronously); nothing is
 * allocated per call.  With world == 1 the communicator is ready at once;
 * otherwise exchange handles and call ar_comm_open.  *out is NULL on error.
 */
AR_API int ar_comm_create(int rank, int world, int64_t max_elems, ar_comm **out);

/* This rank's handle record (AR_COMM_HANDLE_BYTES bytes) for the others. */
AR_API int ar_comm_handle(const ar_comm *c, void *record);

/* Checks a gathered set of `world` records (rank order): each is a record
 * of this library, rank w's record says rank w, and all agree on world,
 * max_elems, region size and SM count.  AR_EINVAL otherwise.  Host only. */
AR_API int ar_comm_check_handles(const void *records, int world);

/* Maps every other rank's region from the gathered records (world *
 * AR_COMM_HANDLE_BYTES bytes, rank order; this rank's own entry is only
 * checked).  All or nothing: on failure nothing stays mapped. */
AR_API int ar_comm_open(ar_comm *c, const void *records);

/*
 * ar_comm_create_group -- W ranks in this process on the current device:
 * W regions in one allocation, each rank's "peers" being the others.  A
 * group call runs every rank's part in ONE cooperative launch (the ranks'
 * CTAs are co-resident, so their waits on each other always complete).  It
 * exercises the exact exchange protocol and kernels of the multi-GPU form on
 * one GPU; calls take per-rank arrays.  rank-form calls on a group return
 * AR_EINVAL and vice versa.
 */
AR_API int ar_comm_create_group(int world, int64_t max_elems, ar_comm **out);

/* Unmaps peers and frees the region; NULL is a no-op.  Synchronises the
 * communicator's device.  Every rank must have finished its calls (its
 * device synchronised, and the ranks met on the host) before any rank
 * destroys its communicator: another rank's last kernel may still be reading
 * this rank's region. */
AR_API int ar_comm_destroy(ar_comm *c);

/* Limit of one cross-rank wait in nanoseconds (default 2 s; >= 1 ms). */
AR_API int ar_comm_set_timeout(ar_comm *c, uint64_t ns);

/* Largest per-rank partial (T*H*2 bytes) that AR_ALGO_AUTO sends one-shot;
 * above it the two-shot form is used.  Default 1 MiB for W <= 4, 512 KiB
 * above (the crossover is a measured property; callers may load their own). */
AR_API int ar_comm_set_oneshot_max(ar_comm *c, int64_t bytes);

/* The algorithm AR_ALGO_AUTO picks for a call of T x H (depends on the
 * arguments and the communicator's settings only: capture-static). */
AR_API int ar_comm_algo(const ar_comm *c, int64_t T, int64_t H, int *algo);

/* Synchronises the device; AR_ETIMEDOUT if a cross-rank wait of this
 * communicator ran out since the last clear, else AR_OK.  clear != 0 resets
 * the record. */
AR_API int ar_comm_status(ar_comm *c, int clear);

/* Test hook: in the next launch of this communicator, rank `rank` publishes
 * no arrival, so the other ranks' bounded waits run out (-1 clears).  It
 * exists so the timeout path can be tested without a GPU fault. */
AR_API int ar_comm_test_withhold(ar_comm *c, int rank);

/*
 * ar_comm_allreduce_add_rmsnorm -- this rank's part of
 *   r = residual + sum_w partial_w,  y = r * rsqrt(mean(r^2) + eps) * w_eff
 * partial       this rank's [T, H] partial (16-bit)
 * residual      [T, H] or NULL (the no-residual form); same on every rank
 * weight        [H]
 * out           [T, H]: y (every row, on every rank)
 * residual_out  [T, H] or NULL (dead residual): r
 * T*H <= max_elems; H, eps, gemma, dtype as in ar_add_rmsnorm.
 * algo          AR_ALGO_AUTO, AR_ALGO_ONESHOT or AR_ALGO_TWOSHOT
 * All pointers 16-byte aligned device memory of the communicator's device.
 */
AR_API int ar_comm_allreduce_add_rmsnorm(ar_comm *c, const void *partial, const void *residual,
                                         const void *weight, void *out, void *residual_out,
                                         int64_t T, int64_t H, float eps, int gemma, int dtype,
                                         int algo, cudaStream_t stream);

/* The same with per-group FP8 output, as ar_add_rmsnorm_quant_fp8_group
 * (scales row-major [T, H/128]; out_y and residual_out nullable). */
AR_API int ar_comm_allreduce_add_rmsnorm_quant_fp8_group(
    ar_comm *c, const void *partial, const void *residual, const void *weight, void *out_fp8,
    float *scales, void *out_y, void *residual_out, int64_t T, int64_t H, int group, float eps,
    int gemma, int dtype, int algo, cudaStream_t stream);

/*
 * ar_comm_qk_norm_sharded -- this rank's shard of the sharded QK-norm.
 * qkv       this rank's [T, qs + 2 ks] (qs = q_size / W, ks = kv_size / W)
 * q_weight  [q_size], k_weight [kv_size]: full vectors (rank r uses its slice)
 * q_out     [T, qs] dense, or qkv itself (in place: k_out == qkv + qs
 *           elements; outputs then take qkv's row stride; v untouched)
 * k_out     [T, ks] dense, or qkv + qs
 * T * 4 <= max_elems; other requirements as in qk_norm_sharded.
 */
AR_API int ar_comm_qk_norm_sharded(ar_comm *c, const void *qkv, const void *q_weight,
                                   const void *k_weight, void *q_out, void *k_out, int64_t T,
                                   int64_t q_size, int64_t kv_size, float eps, int dtype,
                                   cudaStream_t stream);

/* Group forms: the same calls for every rank of a group at once; each
 * per-rank argument is a host array of W device pointers (residual and
 * residual_out arrays may be NULL, or hold NULL entries consistently). */
AR_API int ar_group_allreduce_add_rmsnorm(ar_comm *g, const void *const *partial,
                                          const void *const *residual, const void *weight,
                                          void *const *out, void *const *residual_out, int64_t T,
                                          int64_t H, float eps, int gemma, int dtype, int algo,
                                          cudaStream_t stream);

AR_API int ar_group_allreduce_add_rmsnorm_quant_fp8_group(
    ar_comm *g, const void *const *partial, const void *const *residual, const void *weight,
    void *const *out_fp8, float *const *scales, void *const *out_y, void *const *residual_out,
    int64_t T, int64_t H, int group, float eps, int gemma, int dtype, int algo,
    cudaStream_t stream);

AR_API int ar_group_qk_norm_sharded(ar_comm *g, const void *const *qkv, const void *q_weight,
                                    const void *k_weight, void *const *q_out, void *const *k_out,
                                    int64_t T, int64_t q_size, int64_t kv_size, float eps,
                                    int dtype, cudaStream_t stream);

/*
 * ar_group_qk_norm_sharded_static -- ar_group_qk_norm_sharded (W ranks of
 * one GPU, one cooperative launch) for callers that cannot allocate device
 * memory: it calls no cudaMalloc, cudaFree or allocating library routine.
 * Some callers cannot call cudaMalloc: a plugin that only receives buffers
 * from its host application, an engine that reserved all free device
 * memory at start-up (a further allocation would fail), or code that must
 * not take the device-wide synchronisation cudaMalloc may imply.  The
 * papers describe no such form: it has no counterpart there.
 *
 * The exchange regions live in one file-scope device array of
 * AR_STATIC_QK_MAX_W regions of 8 * AR_STATIC_QK_MAX_T * 2 bytes plus the
 * flag area (about 2 MiB), which every GPU that loads the library holds
 * until the process exits.  The first call on a device looks up the array's
 * device address on that device (once); make that first call before any
 * stream capture.  Every call shares the array: each call first clears the
 * flags and counters of the regions it uses (an asynchronous memset on
 * `stream`), so calls in one stream are ordered, and calls that overlap on
 * the GPU (other streams, other threads) race and give undefined results.
 * 1 <= W <= AR_STATIC_QK_MAX_W and T <= AR_STATIC_QK_MAX_T (else AR_EINVAL /
 * AR_EUNSUPPORTED); other arguments as in ar_group_qk_norm_sharded, with
 * per-rank host arrays of W device pointers.
 */
#define AR_STATIC_QK_MAX_T 4096
#define AR_STATIC_QK_MAX_W 16
AR_API int ar_group_qk_norm_sharded_static(int W, const void *const *qkv, const void *q_weight,
                                           const void *k_weight, void *const *q_out,
                                           void *const *k_out, int64_t T, int64_t q_size,
                                           int64_t kv_size, float eps, int dtype,
                                           cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AR_COMM_H */
