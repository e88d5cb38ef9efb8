// launch.h -- internal: launch planning and dispatch of the kernels.
#pragma once

#include <cuda_runtime.h>

#include <atomic>

#include "kernels.cuh"

namespace dl {

// fold = true launches the merge-token variant of the append kernel.
using append_fn = cudaError_t (*)(const AppendParams &, bool fold, cudaStream_t);
using merge_fn = cudaError_t (*)(const MergeParams &, cudaStream_t);
using eager_fn = cudaError_t (*)(const EagerParams &, cudaStream_t);

// The same over a list of slots, each at its own log length; p.L is the
// longest length in the list.  In the append list, entries [0, nfold) take
// the merge-token.
using append_slots_fn = cudaError_t (*)(const AppendParams &, const SlotList &, cudaStream_t);
using merge_slots_fn = cudaError_t (*)(const MergeParams &, const SlotList &, cudaStream_t);

// Return the launcher for (op, dk, dv), or nullptr for an unsupported shape.
append_fn get_append(int op, int dk, int dv);
merge_fn get_merge(int op, int dk, int dv);
eager_fn get_eager(int op, int dk, int dv);
append_slots_fn get_append_slots(int op, int dk, int dv);
merge_slots_fn get_merge_slots(int op, int dk, int dv);

// Number of SMs of the current device (cached per device).
cudaError_t sm_count(int *sms);

// Value-tile width for NH heads of width DV: 64 columns (or the whole head
// when narrower) while that still gives at least four CTAs per SM, else 32.
// Measured on B200 for d = 64 and 128: 64-column tiles beat 32 (more per-CTA
// work to amortise the prologue) and 128 (fewer, longer CTAs: worse overlap
// of their serial phases), so 128-column tiles are not built.
inline int pick_tile(long long NH, int DV, int sms) {
    int tv = DV < 64 ? DV : 64;
    while (tv > 32 && NH * (DV / tv) < 4LL * sms) tv /= 2;
    return tv;
}

// Threads of a CTA over a TV-column tile of d_k rows: TV/4 threads per row
// (one 16-byte column group each) and d_k/8 row groups, so that every thread
// streams 8 rows of its column group.
template <int DK, int TV>
struct CtaShape {
    static constexpr int NT = (TV / 4) * (DK / 8);
};

// The append and the merge-token stream 16 rows per thread where that still
// leaves a thread per key row and per value column: at most 96 registers a
// thread, so 5 CTAs of 128 threads fit an SM and 160 KB of the base is in
// flight per SM instead of 128 KB (the merge-token folds its log four
// entries at a time, so that only four value factors a thread are held in
// registers).  Measured on B200 in four-layer merge cycles against 8 rows per
// thread: append GDN -4.2 %, KDA -4.9 %, RWKV6 (d = 64) -0.3 % per token;
// merge-token GDN C8 53.3 -> 48.8 us, KDA C8 99.3 -> 91.9 us (cycles GDN
// -0.8 %, KDA -1.2 %, RWKV6 C4 -3.8 %, RWKV6 C8 +1.4 %).
template <int DK, int TV, bool FOLD>
struct AppendShape {
    static constexpr int NT16 = (TV / 4) * (DK / 16);
    static constexpr int NT = (NT16 >= (DK > TV ? DK : TV)) ? NT16 : CtaShape<DK, TV>::NT;
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

// CTAs of `kern` resident per SM on the current device at `threads`
// threads and `smem` bytes of dynamic shared memory, computed once per
// device (callers pass the largest size they launch with, so that the
// answer does not depend on which launch came first).
template <typename Kernel>
cudaError_t resident_ctas(std::atomic<int> (&cache)[64], Kernel kern, int threads, size_t smem, int *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
        if (e != cudaSuccess) return e;
        n = n > 0 ? n : 1;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    *out = n;
    return cudaSuccess;
}

}  // namespace dl

#define DL_DIM_INDEX(d) ((d) == 64 ? 0 : ((d) == 128 ? 1 : -1))
