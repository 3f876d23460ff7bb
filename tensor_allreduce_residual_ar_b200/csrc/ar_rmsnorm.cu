// ar_rmsnorm.cu -- C ABI entry points: argument validation, plan dispatch,
// launch geometry and kernel launch on the caller's stream.
//
// Error behaviour follows two lessons of the vLLM reports: never a silent
// no-op on an unsupported size (PR #54787 report, section 风险与影响, item 1),
// and no try/except-style fallback that hides a failure (PR #44849 report,
// section 评论区精华).  Every rejection is a status code, and nothing is
// launched after a rejection.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <mutex>

#include "ar_rmsnorm.h"
#include "host_util.h"
#include "kernels.cuh"
#include "plan.h"

using namespace arn;

namespace arn {

constexpr int kMaxDevices = 64;

DevInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

// Device facts, read once per device.  sm_100a code runs only on compute
// capability 10.0 (B200); anything else is AR_EUNSUPPORTED.
int device_info(DevInfo &out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return AR_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return AR_EUNSUPPORTED;
    std::call_once(g_dev_once[dev], [dev] {
        int major = 0, minor = 0, sms = 0, optin = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
            g_dev[dev].status = AR_ECUDA;
            return;
        }
        g_dev[dev].status = (major == 10 && minor == 0) ? AR_OK : AR_EUNSUPPORTED;
        g_dev[dev].sm_count = sms;
        g_dev[dev].smem_optin = optin;
    });
    out = g_dev[dev];
    return out.status;
}

bool split_threads(int packs, int max_threads, int &threads, int &ppt_idx) {
    for (int i = 0; i < kPptVariants; ++i) {
        const int ppt = 1 << i;
        const int t = (packs + ppt - 1) / ppt;
        if (t <= max_threads) {
            threads = ((t + 31) / 32) * 32;
            ppt_idx = i;
            return true;
        }
    }
    return false;
}

namespace {
struct OccKey { const void *fn; int threads; int dev; };
struct OccSlot { OccKey key; int occ; };
std::mutex g_occ_mutex;
OccSlot g_occ[512];
int g_occ_n = 0;
struct ClusterOccSlot { OccKey key; int C; int n; };
ClusterOccSlot g_cocc[256];
int g_cocc_n = 0;
}  // namespace

int occupancy(const void *fn, int threads, int dev) {
    std::lock_guard<std::mutex> lk(g_occ_mutex);
    for (int i = 0; i < g_occ_n; ++i)
        if (g_occ[i].key.fn == fn && g_occ[i].key.threads == threads && g_occ[i].key.dev == dev)
            return g_occ[i].occ;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, 0) != cudaSuccess || occ < 1)
        occ = 1;
    if (g_occ_n < 512) g_occ[g_occ_n++] = {{fn, threads, dev}, occ};
    return occ;
}

int cluster_occupancy(const void *fn, int threads, int C, int dev, int sm_count) {
    {
        std::lock_guard<std::mutex> lk(g_occ_mutex);
        for (int i = 0; i < g_cocc_n; ++i)
            if (g_cocc[i].key.fn == fn && g_cocc[i].key.threads == threads &&
                g_cocc[i].key.dev == dev && g_cocc[i].C == C)
                return g_cocc[i].n;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C, 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)C;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        n = sm_count * occupancy(fn, threads, dev) / C;
    }
    if (n < 1) n = 1;
    std::lock_guard<std::mutex> lk(g_occ_mutex);
    if (g_cocc_n < 256) g_cocc[g_cocc_n++] = {{fn, threads, dev}, C, n};
    return n;
}

// Programmatic dependent launch is on unless AR_RMSNORM_PDL=0 in the
// environment when the library first launches.
bool pdl_enabled() {
    static const bool on = [] {
        const char *e = std::getenv("AR_RMSNORM_PDL");
        return !(e && e[0] == '0');
    }();
    return on;
}

}  // namespace arn

namespace {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// ---------------------------------------------------------------------------
// launch tables
// ---------------------------------------------------------------------------

using NormKernel = void (*)(const NormParams);
using QKKernel = void (*)(const QKParams);

template <typename Elt, bool FP8, int MODE>
NormKernel norm_kernel_for(int wb, int ppt_idx) {
#define ARN_K(WB, PPT) &norm_rows_kernel<Elt, WB, PPT, FP8, MODE>
    static const NormKernel tab[4][kPptVariants] = {
        {ARN_K(2, 1), ARN_K(2, 2), ARN_K(2, 4)},
        {ARN_K(4, 1), ARN_K(4, 2), ARN_K(4, 4)},
        {ARN_K(8, 1), ARN_K(8, 2), ARN_K(8, 4)},
        {ARN_K(16, 1), ARN_K(16, 2), ARN_K(16, 4)},
    };
#undef ARN_K
    return tab[wb][ppt_idx];
}

template <int MODE>
NormKernel pick_norm_kernel_mode(int dtype, bool fp8, int wb, int ppt_idx) {
    if (dtype == AR_BF16)
        return fp8 ? norm_kernel_for<__nv_bfloat16, true, MODE>(wb, ppt_idx)
                   : norm_kernel_for<__nv_bfloat16, false, MODE>(wb, ppt_idx);
    return fp8 ? norm_kernel_for<__half, true, MODE>(wb, ppt_idx)
               : norm_kernel_for<__half, false, MODE>(wb, ppt_idx);
}

// The kernel compiled for a plan's grid shape (see kModeRow and friends).
NormKernel pick_norm_kernel(int dtype, bool fp8, int wb, int ppt_idx, const Geometry &g) {
    if (g.minb == 2) return pick_norm_kernel_mode<kModePersist512>(dtype, fp8, wb, ppt_idx);
    if (g.persistent) return pick_norm_kernel_mode<kModePersist>(dtype, fp8, wb, ppt_idx);
    return pick_norm_kernel_mode<kModeRow>(dtype, fp8, wb, ppt_idx);
}

// Bulk-staged kernels: one slot of EPT elements per consumer thread.
// EPT 4 with up to 1024 consumers (rows up to 4096 elements), EPT 8 with up
// to 640 consumers (rows up to 5120 elements).
constexpr int kBulkMaxT4 = 1024;
constexpr int kBulkMaxT8 = 640;

template <typename Elt, bool FP8>
NormKernel bulk_kernel_for(int wb, int ept) {
#define ARN_B(WB) ept == 4 ? &norm_bulk_kernel<Elt, WB, 4, FP8, kBulkMaxT4> \
                           : &norm_bulk_kernel<Elt, WB, 8, FP8, kBulkMaxT8>
    switch (wb) {
    case 0: return ARN_B(2);
    case 1: return ARN_B(4);
    case 2: return ARN_B(8);
    default: return ARN_B(16);
    }
#undef ARN_B
}

NormKernel pick_bulk_kernel(int dtype, bool fp8, int wb, int ept) {
    if (dtype == AR_BF16)
        return fp8 ? bulk_kernel_for<__nv_bfloat16, true>(wb, ept)
                   : bulk_kernel_for<__nv_bfloat16, false>(wb, ept);
    return fp8 ? bulk_kernel_for<__half, true>(wb, ept) : bulk_kernel_for<__half, false>(wb, ept);
}

// Opt a kernel into `bytes` of dynamic shared memory (once per kernel and
// size class; kernel attributes are per device context, so the first call on
// every device sets them).
std::mutex g_attr_mutex;
struct AttrSlot { const void *fn; int dev; int bytes; };
AttrSlot g_attr[512];
int g_attr_n = 0;

int ensure_smem(const void *fn, int dev, int bytes) {
    std::lock_guard<std::mutex> lk(g_attr_mutex);
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr[i].fn == fn && g_attr[i].dev == dev && g_attr[i].bytes >= bytes) return AR_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return AR_ECUDA;
    if (g_attr_n < 512) g_attr[g_attr_n++] = {fn, dev, bytes};
    return AR_OK;
}

std::atomic<int64_t> g_withhold_row{-1};

QKKernel pick_qk_kernel(int dtype, int ppt_idx, int minb) {
    static const QKKernel bf[2][kPptVariants] = {
        {&qk_norm_kernel<__nv_bfloat16, 1, 1>, &qk_norm_kernel<__nv_bfloat16, 2, 1>,
         &qk_norm_kernel<__nv_bfloat16, 4, 1>},
        {&qk_norm_kernel<__nv_bfloat16, 1, 2>, &qk_norm_kernel<__nv_bfloat16, 2, 2>,
         &qk_norm_kernel<__nv_bfloat16, 4, 2>}};
    static const QKKernel hf[2][kPptVariants] = {
        {&qk_norm_kernel<__half, 1, 1>, &qk_norm_kernel<__half, 2, 1>, &qk_norm_kernel<__half, 4, 1>},
        {&qk_norm_kernel<__half, 1, 2>, &qk_norm_kernel<__half, 2, 2>, &qk_norm_kernel<__half, 4, 2>}};
    const int m = minb == 2 ? 1 : 0;
    return dtype == AR_BF16 ? bf[m][ppt_idx] : hf[m][ppt_idx];
}

template <typename Params>
int launch(void (*fn)(const Params), const Params &p, int64_t clusters, int C, int threads,
           cudaStream_t stream, size_t smem = 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(clusters * C), 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (C > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)C;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl_enabled()) {
        // may start while the previous kernel in the stream finishes; the
        // kernel waits for it (griddepcontrol.wait) before any memory access
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, fn, p) == cudaSuccess ? AR_OK : AR_ECUDA;
}

// Grid size in clusters: one per row, or capped for persistent plans.
int64_t grid_clusters(int64_t rows, const Geometry &g, const void *fn, int threads, int dev,
                      int sm_count) {
    int64_t cap = (int64_t)0x7FFFFFFF / g.C;
    if (g.persistent)
        cap = g.C > 1 ? (int64_t)cluster_occupancy(fn, threads, g.C, dev, sm_count)
                      : (int64_t)sm_count * occupancy(fn, threads, dev);
    if (cap < 1) cap = 1;
    return rows < cap ? rows : cap;
}

int validate_norm_common(const void *const *partials, const void *residual, const void *weight,
                         void *residual_out, int64_t T, int64_t H, int W, float eps, int dtype) {
    if (partials == nullptr || weight == nullptr) return AR_EINVAL;
    if (W < 1 || W > AR_MAX_W) return AR_EINVAL;
    if (T < 0 || H < 8 || H % 8 != 0) return AR_EINVAL;
    if (H > AR_MAX_H) return AR_EUNSUPPORTED;
    if (dtype != AR_BF16 && dtype != AR_FP16) return AR_EINVAL;
    if (!std::isfinite(eps) || eps < 0.f) return AR_EINVAL;
    for (int w = 0; w < W; ++w) {
        if (partials[w] == nullptr) return AR_EINVAL;
        if (!aligned(partials[w], 16)) return AR_EALIGN;
    }
    if (!aligned(weight, 16)) return AR_EALIGN;
    if (residual && !aligned(residual, 16)) return AR_EALIGN;
    if (residual_out && !aligned(residual_out, 16)) return AR_EALIGN;
    return AR_OK;
}

int run_norm(const void *const *partials, const void *residual, const void *weight, void *out,
             void *residual_out, uint8_t *out_fp8, float *scales, int64_t s_row, int64_t s_grp,
             int64_t T, int64_t H, int W, float eps, int gemma, int dtype, bool fp8,
             cudaStream_t stream) {
    DevInfo di;
    int st = device_info(di);
    if (st != AR_OK) return st;
    int dev = 0;
    cudaGetDevice(&dev);

    NormParams p = {};
    for (int w = 0; w < W; ++w) p.partials[w] = partials[w];
    p.residual = residual;
    p.weight = weight;
    p.out = out;
    p.residual_out = residual_out;
    p.out_fp8 = out_fp8;
    p.scales = scales;
    p.s_row = s_row;
    p.s_grp = s_grp;
    p.T = T;
    p.P = (int)(H / 8);
    p.W = W;
    p.inv_H = 1.0 / (double)H;
    p.eps = (double)eps;
    p.inv_Hf = (float)p.inv_H;
    p.epsf = eps;
    p.gemma = gemma ? 1 : 0;

    p.withhold_row = -1;
    // certified fast sum for outputs with p significand bits (bf16 8,
    // fp16 11): accept s when |s| >= u (2^(p+2) + 1) sum_k |s_k|, with a 1%
    // margin for the (1 + O(Wu)) factors and the fp32 evaluation of the test
    {
        const int pbits = dtype == AR_BF16 ? 8 : 11;
        p.kcert = (float)(std::ldexp(1.0, -24) * (std::ldexp(1.0, pbits + 2) + 1.0) * 1.01);
    }
    const int variant = fp8 ? AR_VARIANT_FP8 : AR_VARIANT_NORM;
    int plan = plan_lookup(variant, T, H, W, dtype, di.sm_count);

    if (plan == AR_PLAN_BULK) {
        // one row of every stream per stage, at least two stages in shared
        // memory, one slot of 4 (or else 8) elements per consumer thread;
        // otherwise the persistent register-resident plan
        const int NS = W + (residual ? 1 : 0);
        const size_t stage_bytes = (size_t)NS * (size_t)H * 2;
        const size_t budget = (size_t)di.smem_optin > 4096 ? (size_t)di.smem_optin - 4096 : 0;
        int stages = (int)(budget / stage_bytes);
        if (stages > kBulkMaxStages) stages = kBulkMaxStages;
        int ept = 0;
        if ((H / 8 + 31) / 32 * 32 <= kBulkMaxT8) ept = 8;
        else if ((H / 4 + 31) / 32 * 32 <= kBulkMaxT4) ept = 4;
        if (stages >= 2 && ept != 0) {
            const int consumers = (int)(((H / ept) + 31) / 32 * 32);
            p.C = 1;
            p.ppc = p.P;
            p.prefetch = 0;
            p.stages = stages;
            p.consumers = consumers;
            p.withhold_row = g_withhold_row.exchange(-1);
            NormKernel fn = pick_bulk_kernel(dtype, fp8, wb_bucket(W), ept);
            const int smem = (int)(stages * stage_bytes);
            int st2 = ensure_smem((const void *)fn, dev, smem);
            if (st2 != AR_OK) return st2;
            const int64_t grid = T < di.sm_count ? T : di.sm_count;
            return launch(fn, p, grid, 1, consumers, stream, (size_t)smem);
        }
        plan = AR_PLAN_PERSIST;
    }
    Geometry g = plan_geometry(plan);
    // never split a row into slices narrower than one FP8 group
    while (g.C > 1 && (p.P + g.C - 1) / g.C < kGroupPacks) g.C /= 2;
    int ppc = 0, threads = 0, ppt_idx = 0;
    for (;;) {
        ppc = (p.P + g.C - 1) / g.C;
        if (fp8) ppc = ((ppc + kGroupPacks - 1) / kGroupPacks) * kGroupPacks;
        if (split_threads(ppc, g.max_threads, threads, ppt_idx) ||
            split_threads(ppc, kMaxThreads, threads, ppt_idx))
            break;
        // a row too wide for this plan's cluster: widen the cluster
        if (g.C >= 8) return AR_EUNSUPPORTED;
        g.C *= 2;
        g.persistent = false;
    }
    p.C = g.C;
    p.ppc = ppc;
    p.prefetch = g.persistent ? 1 : 0;
    NormKernel fn = pick_norm_kernel(dtype, fp8, wb_bucket(W), ppt_idx, g);
    const int64_t clusters = grid_clusters(T, g, (const void *)fn, threads, dev, di.sm_count);
    return launch(fn, p, clusters, g.C, threads, stream);
}

}  // namespace

extern "C" {

int ar_add_rmsnorm(const void *const *partials, const void *residual, const void *weight, void *out,
                   void *residual_out, int64_t T, int64_t H, int W, float eps, int gemma, int dtype,
                   cudaStream_t stream) {
    int st = validate_norm_common(partials, residual, weight, residual_out, T, H, W, eps, dtype);
    if (st != AR_OK) return st;
    if (out == nullptr) return AR_EINVAL;
    if (!aligned(out, 16)) return AR_EALIGN;
    if (T == 0) return AR_OK;
    return run_norm(partials, residual, weight, out, residual_out, nullptr, nullptr, 0, 0, T, H, W,
                    eps, gemma, dtype, false, stream);
}

int ar_add_rmsnorm_quant_fp8_group_strided(const void *const *partials, const void *residual,
                                           const void *weight, void *out_fp8, float *scales,
                                           int64_t scale_stride_t, int64_t scale_stride_g,
                                           void *out_y, void *residual_out, int64_t T, int64_t H,
                                           int W, int group, float eps, int gemma, int dtype,
                                           cudaStream_t stream) {
    int st = validate_norm_common(partials, residual, weight, residual_out, T, H, W, eps, dtype);
    if (st != AR_OK) return st;
    if (out_fp8 == nullptr || scales == nullptr) return AR_EINVAL;
    if (group != 128 || H % group != 0) return AR_EINVAL;
    // every (row, group) must own a distinct scale slot
    {
        const __int128 G = H / group, st_t = scale_stride_t, st_g = scale_stride_g;
        if (st_t < 0 || st_g < 0) return AR_EINVAL;
        bool ok;
        if (G == 1 && T <= 1) ok = true;
        else if (G == 1) ok = st_t >= 1;
        else if (T <= 1) ok = st_g >= 1;
        else ok = (st_g >= 1 && st_t >= G * st_g) || (st_t >= 1 && st_g >= (__int128)T * st_t);
        if (!ok) return AR_EINVAL;
    }
    if (!aligned(out_fp8, 16) || !aligned(scales, 4)) return AR_EALIGN;
    if (out_y && !aligned(out_y, 16)) return AR_EALIGN;
    if (T == 0) return AR_OK;
    return run_norm(partials, residual, weight, out_y, residual_out, (uint8_t *)out_fp8, scales,
                    scale_stride_t, scale_stride_g, T, H, W, eps, gemma, dtype, true, stream);
}

int ar_add_rmsnorm_quant_fp8_group(const void *const *partials, const void *residual,
                                   const void *weight, void *out_fp8, float *scales, void *out_y,
                                   void *residual_out, int64_t T, int64_t H, int W, int group,
                                   float eps, int gemma, int dtype, cudaStream_t stream) {
    const int64_t groups = group > 0 ? H / group : 0;
    return ar_add_rmsnorm_quant_fp8_group_strided(partials, residual, weight, out_fp8, scales,
                                                  groups, 1, out_y, residual_out, T, H, W, group,
                                                  eps, gemma, dtype, stream);
}

int qk_norm_sharded(const void *const *qkv, const void *q_weight, const void *k_weight,
                    void *const *q_out, void *const *k_out, int64_t T, int64_t q_size,
                    int64_t kv_size, int W, float eps, int dtype, cudaStream_t stream) {
    if (qkv == nullptr || q_out == nullptr || k_out == nullptr || q_weight == nullptr ||
        k_weight == nullptr)
        return AR_EINVAL;
    if (W < 1 || W > AR_MAX_W || T < 0) return AR_EINVAL;
    if (q_size <= 0 || kv_size <= 0 || q_size % W != 0 || kv_size % W != 0) return AR_EINVAL;
    const int64_t qs = q_size / W, ks = kv_size / W;
    if (qs % 8 != 0 || ks % 8 != 0) return AR_EINVAL;
    if (qs + ks > AR_MAX_H) return AR_EUNSUPPORTED;
    if (dtype != AR_BF16 && dtype != AR_FP16) return AR_EINVAL;
    if (!std::isfinite(eps) || eps < 0.f) return AR_EINVAL;
    for (int w = 0; w < W; ++w) {
        if (qkv[w] == nullptr || q_out[w] == nullptr || k_out[w] == nullptr) return AR_EINVAL;
        if (!aligned(qkv[w], 16) || !aligned(q_out[w], 16) || !aligned(k_out[w], 16)) return AR_EALIGN;
    }
    if (!aligned(q_weight, 16) || !aligned(k_weight, 16)) return AR_EALIGN;
    // in-place form: q_out[w] == qkv[w] and k_out[w] == qkv[w] + qs elements
    // for every shard; the outputs then have qkv's row stride
    const bool inplace = q_out[0] == qkv[0];
    for (int w = 0; w < W; ++w) {
        const char *base = static_cast<const char *>(qkv[w]);
        const bool ip = q_out[w] == qkv[w] && static_cast<const char *>(k_out[w]) == base + qs * 2;
        if (ip != inplace) return AR_EINVAL;
    }
    if (T == 0) return AR_OK;

    DevInfo di;
    int st = device_info(di);
    if (st != AR_OK) return st;
    int dev = 0;
    cudaGetDevice(&dev);

    QKParams p = {};
    for (int w = 0; w < W; ++w) {
        p.qkv[w] = qkv[w];
        p.q_out[w] = q_out[w];
        p.k_out[w] = k_out[w];
    }
    p.q_weight = q_weight;
    p.k_weight = k_weight;
    p.T = T;
    p.W = W;
    p.qsp = (int)(qs / 8);
    p.ksp = (int)(ks / 8);
    p.row_packs = p.qsp + 2 * p.ksp;
    p.q_stride = inplace ? p.row_packs : p.qsp;
    p.k_stride = inplace ? p.row_packs : p.ksp;
    p.inv_q = (float)(1.0 / (double)q_size);
    p.inv_k = (float)(1.0 / (double)kv_size);
    p.eps = eps;

    int plan = plan_lookup(AR_VARIANT_QK, T, q_size + kv_size, W, dtype, di.sm_count);
    if (plan == AR_PLAN_QK_BULK) {
        // weights plus at least two tokens in the shared-memory ring, else
        // the persistent register-resident plan
        const size_t tok_bytes = (size_t)W * (size_t)(qs + ks) * 2;
        const size_t w_bytes = (size_t)(q_size + kv_size) * 2;
        const size_t budget = (size_t)di.smem_optin > 4096 ? (size_t)di.smem_optin - 4096 : 0;
        int fit = budget > w_bytes ? (int)((budget - w_bytes) / tok_bytes) : 0;
        if (fit > kQKMaxStages) fit = kQKMaxStages;
        if (fit >= 4) {
            // NW consumer warps with SPW stages each (stages = NW * SPW)
            const int nw = fit < kMaxWarps - 1 ? fit : kMaxWarps - 1;
            const int spw = fit / nw;
            p.C = 1;
            p.stages = nw * spw;
            QKKernel fn = dtype == AR_BF16 ? &qk_bulk_kernel<__nv_bfloat16> : &qk_bulk_kernel<__half>;
            const int smem = (int)(w_bytes + (size_t)p.stages * tok_bytes);
            int st2 = ensure_smem((const void *)fn, dev, smem);
            if (st2 != AR_OK) return st2;
            const int64_t grid = T < di.sm_count ? T : di.sm_count;
            return launch(fn, p, grid, 1, 32 * (nw + 1), stream, (size_t)smem);
        }
        plan = AR_PLAN_QK_PERSIST;
    }
    if (plan == AR_PLAN_QK_RING) {
        // one token per CTA at a time, every shard of it (at most 256
        // threads, 1, 2 or 4 packs each), the next tokens' copies in a
        // shared-memory ring; otherwise the persistent register plan
        int threads = 0, ppt_idx = 0;
        if (split_threads(W * (p.qsp + p.ksp), 256, threads, ppt_idx)) {
            p.C = 1;
            p.spc = W;
            static const QKKernel bf[kPptVariants] = {&qk_ring_kernel<__nv_bfloat16, 1>,
                                                      &qk_ring_kernel<__nv_bfloat16, 2>,
                                                      &qk_ring_kernel<__nv_bfloat16, 4>};
            static const QKKernel hf[kPptVariants] = {&qk_ring_kernel<__half, 1>, &qk_ring_kernel<__half, 2>,
                                                      &qk_ring_kernel<__half, 4>};
            QKKernel fn = dtype == AR_BF16 ? bf[ppt_idx] : hf[ppt_idx];
            const int smem = kQKRingStages * (1 << ppt_idx) * threads * 16;
            int st2 = ensure_smem((const void *)fn, dev, smem);
            if (st2 != AR_OK) return st2;
            int occ = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, (size_t)smem) != cudaSuccess ||
                occ < 1) {
                (void)cudaGetLastError();
                occ = 1;
            }
            const int64_t cap = (int64_t)di.sm_count * occ;
            return launch(fn, p, T < cap ? T : cap, 1, threads, stream, (size_t)smem);
        }
        plan = AR_PLAN_QK_PERSIST;
    }
    Geometry g = plan_geometry(plan);
    while (g.C > 1 && W % g.C != 0) g.C /= 2;
    int threads = 0, ppt_idx = 0;
    for (;;) {
        p.spc = W / g.C;
        const int npk = p.spc * (p.qsp + p.ksp);
        if (split_threads(npk, g.max_threads, threads, ppt_idx) ||
            split_threads(npk, kMaxThreads, threads, ppt_idx))
            break;
        // a token too wide for this plan's cluster: split it over more CTAs
        if (g.C >= 8 || W % (2 * g.C) != 0) return AR_EUNSUPPORTED;
        g.C *= 2;
        g.persistent = false;
    }
    p.C = g.C;
    p.prefetch = g.persistent ? 1 : 0;
    QKKernel fn = pick_qk_kernel(dtype, ppt_idx, g.minb);
    const int64_t clusters = grid_clusters(T, g, (const void *)fn, threads, dev, di.sm_count);
    return launch(fn, p, clusters, g.C, threads, stream);
}

int ar_plan_query(int variant, int64_t T, int64_t H, int W, int dtype, int *plan_id) {
    if (plan_id == nullptr || variant < 0 || variant > 2) return AR_EINVAL;
    if (dtype != AR_BF16 && dtype != AR_FP16) return AR_EINVAL;
    if (W < 1 || W > AR_MAX_W || T < 0 || H < 8) return AR_EINVAL;
    int sms = 148;
    DevInfo di;
    if (device_info(di) == AR_OK) sms = di.sm_count;
    *plan_id = plan_lookup(variant, T, H, W, dtype, sms);
    return AR_OK;
}

int ar_plan_load(const char *path) { return plan_load_file(path); }

int ar_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return AR_ECUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, arn::g_ar_device_status, sizeof v) != cudaSuccess) return AR_ECUDA;
    if (clear && v) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(arn::g_ar_device_status, &zero, sizeof zero) != cudaSuccess) return AR_ECUDA;
    }
    return v ? AR_ETIMEDOUT : AR_OK;
}

int ar_test_withhold_row(int64_t row) {
    if (row < -1) return AR_EINVAL;
    g_withhold_row.store(row);
    return AR_OK;
}

int ar_plan_force(int variant, int plan_id) { return plan_force(variant, plan_id); }

int ar_plan_table_size(void) { return plan_table_size(); }

const char *ar_status_string(int status) {
    switch (status) {
    case AR_OK: return "AR_OK: success";
    case AR_EINVAL: return "AR_EINVAL: invalid argument (null pointer, size or count)";
    case AR_EALIGN: return "AR_EALIGN: pointer not aligned (16 bytes; 4 for scales)";
    case AR_EUNSUPPORTED: return "AR_EUNSUPPORTED: device is not sm_100 or size beyond limits";
    case AR_ECUDA: return "AR_ECUDA: CUDA runtime call or kernel launch failed";
    case AR_ETIMEDOUT: return "AR_ETIMEDOUT: bounded device wait expired";
    default: return "unknown ar_status";
    }
}

}  // extern "C"
