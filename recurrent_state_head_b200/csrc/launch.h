// launch.h -- internal: launch planning and dispatch of the kernels.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "kernels.cuh"

namespace dl {

// fold = true launches the merge-token variant of the append kernel.
using append_fn = cudaError_t (*)(const AppendParams &, bool fold, cudaStream_t);
using merge_fn = cudaError_t (*)(const MergeParams &, cudaStream_t);
using eager_fn = cudaError_t (*)(const EagerParams &, cudaStream_t);

// Return the launcher for (op, dk, dv), or nullptr for an unsupported shape.
append_fn get_append(int op, int dk, int dv);
merge_fn get_merge(int op, int dk, int dv);
eager_fn get_eager(int op, int dk, int dv);

// Number of SMs of the current device (cached per device).
cudaError_t sm_count(int *sms);

// Value-tile width for NH heads of width DV: 64 columns (or the whole head
// when narrower) while that still gives at least four CTAs per SM, else the
// widest tile that does (>= 32 columns).
inline int pick_tile(long long NH, int DV, int sms) {
    int tv = DV < 64 ? DV : 64;
    while (tv > 32 && NH * (DV / tv) < 4LL * sms) tv /= 2;
    return tv;
}

// Pipeline depth (stages) of the persistent append kernel per tile width.
template <int TV>
struct Pipe {
    static constexpr int NS = (TV == 32) ? 3 : 2;
};

// Resident CTAs per SM of a kernel at a given dynamic shared-memory size,
// cached per (device, size).
class OccupancyCache {
   public:
    template <typename Kernel>
    cudaError_t get(Kernel kern, int nt, size_t smem, int *per_sm) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        {
            std::lock_guard<std::mutex> lock(mu_);
            for (int i = 0; i < n_; ++i)
                if (dev_[i] == dev && smem_[i] == smem) {
                    *per_sm = occ_[i];
                    return cudaSuccess;
                }
        }
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, nt, smem);
        if (e != cudaSuccess) return e;
        if (occ < 1) return cudaErrorInvalidConfiguration;
        std::lock_guard<std::mutex> lock(mu_);
        if (n_ < kSlots) {
            dev_[n_] = dev;
            smem_[n_] = smem;
            occ_[n_] = occ;
            ++n_;
        }
        *per_sm = occ;
        return cudaSuccess;
    }

   private:
    static constexpr int kSlots = 64;
    std::mutex mu_;
    int dev_[kSlots] = {};
    size_t smem_[kSlots] = {};
    int occ_[kSlots] = {};
    int n_ = 0;
};

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename Kernel>
cudaError_t allow_smem(std::atomic<unsigned long long> &done, Kernel kern, size_t bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_relaxed) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

}  // namespace dl

#define DL_DIM_INDEX(d) ((d) == 64 ? 0 : ((d) == 128 ? 1 : -1))
