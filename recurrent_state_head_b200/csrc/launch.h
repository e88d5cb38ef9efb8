// launch.h -- internal: launch configuration and dispatch of the kernels.
#pragma once

#include <cuda_runtime.h>

#include "kernels.cuh"

namespace dl {

// Value tile and CTA size per head shape.  A CTA covers TV value columns
// of all d_k rows of one head: TV / 4 threads per row, 16-byte loads.
template <int DK, int DV>
struct LaunchCfg {
    static constexpr int TV = 32;
    static constexpr int NT = 128;
};

using append_fn = cudaError_t (*)(const AppendParams &, cudaStream_t);
using merge_fn = cudaError_t (*)(const MergeParams &, cudaStream_t);
using eager_fn = cudaError_t (*)(const EagerParams &, cudaStream_t);

// Return the launcher for (op, dk, dv), or nullptr for an unsupported shape.
append_fn get_append(int op, int dk, int dv);
merge_fn get_merge(int op, int dk, int dv);
eager_fn get_eager(int op, int dk, int dv);

}  // namespace dl

// Instantiate a launcher table for one kernel family.
#define DL_DIM_INDEX(d) ((d) == 64 ? 0 : ((d) == 128 ? 1 : -1))
