// merge_launch.cuh -- internal: launch templates of the merge / materialise
// kernel, for one shared log length (NoSlots) or a list of slots with their
// own lengths (SlotList).
#pragma once

#include "launch.h"

namespace dl {
namespace merge_detail {

template <bool SLOTS>
long long launch_heads(const MergeParams &p, const SlotArg<SLOTS> &sl) {
    if constexpr (SLOTS)
        return (long long)sl.n * p.H;
    else
        return p.NH;
}

// p.L is the shared length, or for a slot list the longest length in it.
// The thread count is the append's: 16 rows a thread where that leaves a
// thread per key row and value column (at most 96 registers, 5 CTAs of 128
// threads per SM).
template <int OP, int DK, int DV, int TV, bool SLOTS>
cudaError_t launch_tv(const MergeParams &p, const SlotArg<SLOTS> &sl, cudaStream_t s) {
    constexpr int NT = AppendShape<DK, TV, true>::NT;
    static std::atomic<unsigned long long> smem_ok{0};
    auto kern = merge_kernel<OP, DK, DV, TV, NT, SLOTS>;
    const int ie = p.in_bf16 ? 2 : 4;
    const size_t smem = op_layout<OP, DK, TV>(p.L, ie, false, true).bytes;
    cudaError_t e = allow_smem(smem_ok, kern, op_layout<OP, DK, TV>(MAXC, 4, false, true).bytes);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(launch_heads<SLOTS>(p, sl) * (DV / TV));
    kern<<<grid, NT, smem, s>>>(p, sl);
    return cudaGetLastError();
}

template <int OP, int DK, int DV, bool SLOTS>
cudaError_t launch(const MergeParams &p, const SlotArg<SLOTS> &sl, cudaStream_t s) {
    int sms = 0;
    cudaError_t e = sm_count(&sms);
    if (e != cudaSuccess) return e;
    switch (pick_tile(launch_heads<SLOTS>(p, sl), DV, sms)) {
        case 64: return launch_tv<OP, DK, DV, 64, SLOTS>(p, sl, s);
        default: break;
    }
    return launch_tv<OP, DK, DV, 32, SLOTS>(p, sl, s);
}

}  // namespace merge_detail
}  // namespace dl
