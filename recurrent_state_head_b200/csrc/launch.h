// launch.h -- internal: launch planning and dispatch of the kernels.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "kernels.cuh"

namespace dl {

using append_fn = cudaError_t (*)(const AppendParams &, cudaStream_t);
using merge_fn = cudaError_t (*)(const MergeParams &, cudaStream_t);
using eager_fn = cudaError_t (*)(const EagerParams &, cudaStream_t);

// Return the launcher for (op, dk, dv), or nullptr for an unsupported shape.
append_fn get_append(int op, int dk, int dv);
merge_fn get_merge(int op, int dk, int dv);
eager_fn get_eager(int op, int dk, int dv);

constexpr int MAX_STAGES = 3;        // pipeline depth of the persistent kernels
constexpr int MAX_CTAS_PER_SM = 4;

// Device facts used by the launch plans (cached per device).
struct DeviceFacts {
    int sms = 0;
    int smem_optin = 0;              // max dynamic + static shared memory per block
};
cudaError_t device_facts(DeviceFacts *f);

// Value-tile width for a kernel over NH heads of width DV: a whole head per
// unit unless that leaves fewer than two units per SM, then halve (>= 32).
inline int pick_tile(long long NH, int DV, int sms) {
    int tv = DV;
    while (tv > 32 && NH * (DV / tv) < 2LL * sms) tv /= 2;
    return tv;
}

// Launch plan of a persistent kernel, cached per (kernel, device, stage size).
struct Plan {
    int ns = 0;        // stages
    size_t smem = 0;   // dynamic shared memory per CTA
    int per_sm = 0;    // resident CTAs per SM
};

class PlanCache {
   public:
    template <typename Kernel>
    cudaError_t get(Kernel kern, int nt, size_t stage_bytes, Plan *out) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        std::lock_guard<std::mutex> lock(mu_);
        for (int i = 0; i < n_; ++i)
            if (keys_[i].dev == dev && keys_[i].stage == stage_bytes) {
                *out = plans_[i];
                return cudaSuccess;
            }
        DeviceFacts f;
        if ((e = device_facts(&f)) != cudaSuccess) return e;
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
        const size_t room = (size_t)f.smem_optin - fa.sharedSizeBytes;
        if (!attr_done_[dev & 63]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)room);
            if (e != cudaSuccess) return e;
            attr_done_[dev & 63] = true;
        }
        Plan p;
        p.ns = MAX_STAGES;
        while (p.ns > 1 && (size_t)p.ns * stage_bytes > room) --p.ns;
        if ((size_t)p.ns * stage_bytes > room) return cudaErrorInvalidConfiguration;
        p.smem = (size_t)p.ns * stage_bytes;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p.per_sm, kern, nt, p.smem);
        if (e != cudaSuccess) return e;
        if (p.per_sm < 1) return cudaErrorInvalidConfiguration;
        p.per_sm = std::min(p.per_sm, MAX_CTAS_PER_SM);
        if (n_ < kSlots) {
            keys_[n_] = {dev, stage_bytes};
            plans_[n_] = p;
            ++n_;
        }
        *out = p;
        return cudaSuccess;
    }

   private:
    static constexpr int kSlots = 128;
    struct Key {
        int dev;
        size_t stage;
    };
    std::mutex mu_;
    Key keys_[kSlots];
    Plan plans_[kSlots];
    bool attr_done_[64] = {};
    int n_ = 0;
};

}  // namespace dl

#define DL_DIM_INDEX(d) ((d) == 64 ? 0 : ((d) == 128 ? 1 : -1))
