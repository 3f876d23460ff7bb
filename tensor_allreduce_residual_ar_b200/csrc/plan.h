// plan.h -- per-shape kernel choice ("plan") for the fused norm library.
//
// A plan names a kernel configuration (cluster size, persistent grid or
// not).  The choice comes from a table of measured timings keyed by
// (variant, dtype, W, H, T range), loaded from JSON, with a built-in rule
// for shapes the table does not cover.  It depends only on those arguments
// and the loaded table, so it is identical inside and outside CUDA-graph
// capture: the "capture-static" property of the one-stage predicate in the
// vLLM PR #54787 report (section 实现拆解, item 1).
#pragma once

#include <stdint.h>

namespace arn {

struct Geometry {
    int C;            // CTAs per row / token (cluster size)
    bool persistent;  // grid capped at SM count x occupancy, rows looped
    int max_threads;  // upper bound on threads per CTA
    int minb;         // CTAs per SM the kernel's registers are sized for (1 or 2)
};

bool plan_valid_for(int variant, int plan_id);
Geometry plan_geometry(int plan_id);

// Plan for a call; never fails for valid arguments.
int plan_lookup(int variant, int64_t T, int64_t H, int W, int dtype, int sm_count);

int plan_load_file(const char *path);     // ar_status
int plan_force(int variant, int plan_id);  // ar_status
int plan_table_size();

}  // namespace arn
