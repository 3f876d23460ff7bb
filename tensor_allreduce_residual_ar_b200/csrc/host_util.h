// host_util.h -- launch helpers shared by the library's host code (device
// facts, thread splits, occupancy, programmatic dependent launch).
#pragma once

#include <cuda_runtime_api.h>
#include <stdint.h>

namespace arn {

struct DevInfo {
    int sm_count = 0;
    int smem_optin = 0;   // largest dynamic shared memory per block
    int status = 0;       // ar_status of the device check
};

// Facts of the current device, read once per device; AR_EUNSUPPORTED unless
// it is compute capability 10.0.
int device_info(DevInfo &out);

// Threads per CTA and packs per thread for `packs` packs per CTA: the
// fewest packs per thread (1, 2, 4) that fit within max_threads.
constexpr int kPptVariants = 3;
bool split_threads(int packs, int max_threads, int &threads, int &ppt_idx);

// Resident CTAs per SM of a kernel at a block size (cached).
int occupancy(const void *fn, int threads, int dev);

// Clusters of C CTAs of a kernel that fit on the device at once (cached).
int cluster_occupancy(const void *fn, int threads, int C, int dev, int sm_count);

// Whether launches use programmatic dependent launch (AR_RMSNORM_PDL=0 off).
bool pdl_enabled();

// W -> partial-count bucket of the kernels' unrolled loops (2, 4, 8, 16).
inline int wb_bucket(int W) { return W <= 2 ? 0 : W <= 4 ? 1 : W <= 8 ? 2 : 3; }

}  // namespace arn
