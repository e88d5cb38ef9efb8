// append_launch.cuh -- internal: launch templates of the append + read-out
// kernel and its merge-token variant, for one log length shared by every
// head (append_kernel) or a list of slots with their own lengths
// (append_slots_kernel).
#pragma once

#include "launch.h"

namespace dl {
namespace append_detail {

// The first wave's CTAs of an SM start spread over a window (slot i of n
// resident CTAs at i * window / n): 2 us for d_k = 128, 4 us for d_k = 64.
// Measured on B200 in four-layer merge cycles, per token, 4 us against no
// offset: GDN -2.3 %, KDA -1.3 %, RWKV6 -4.2 % (C = 8 and C = 4); 2 us
// against 4 us: GDN -0.7 % (isolated append -1 %), KDA -0.2 %, RWKV6 +2.4 %.
template <int DK>
constexpr int stagger_window_ns() { return DK > 64 ? 2000 : 4000; }
constexpr bool kStaggerFold = true;

// Plain launch, or a programmatic dependent launch when p.early (it may
// start while the previous kernel of the stream finishes; the kernel orders
// itself with griddepcontrol).
template <typename Kernel, typename... Args>
cudaError_t launch_kernel(Kernel kern, unsigned grid, int threads, size_t smem, bool early,
                          cudaStream_t s, const Args &...args) {
    if (!early) {
        kern<<<grid, threads, smem, s>>>(args...);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int OP, int DK, int DV, int TV, bool FOLD, int LX = -1>
cudaError_t launch_one(const AppendParams &p, cudaStream_t s) {
    constexpr int NT = AppendShape<DK, TV, FOLD>::NT;
    static std::atomic<unsigned long long> smem_ok{0};
    static std::atomic<int> resident[64];
    auto kern = append_kernel<OP, DK, DV, TV, NT, FOLD, LX>;
    const int ie = p.in_bf16 ? 2 : 4;
    const size_t smem = op_layout<OP, DK, TV>(p.L, ie, true, FOLD).bytes;
    const size_t smem_max = op_layout<OP, DK, TV>(MAXC - 1, 4, true, FOLD).bytes;
    cudaError_t e = allow_smem(smem_ok, kern, smem_max);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((long long)p.NH * (DV / TV));
    Stagger st{0, 0, 0};
    if (!FOLD || kStaggerFold) {
        int slots = 1;
        e = resident_ctas(resident, kern, NT, smem_max, &slots);
        if (e != cudaSuccess) return e;
        e = sm_count(&st.sms);
        if (e != cudaSuccess) return e;
        st.slots = slots;
        st.ns = stagger_window_ns<DK>() / slots;
    }
    return launch_kernel(kern, grid, NT, smem, p.early != 0, s, p, st);
}

// The merge-token sees L = C - 1: the log lengths of C = 4 and 8 have
// kernels of their own (measured on B200: merge-token GDN C8 61.3 -> 54.6
// us, KDA C8 117 -> 104 us), the others take the length at run time.  A
// kernel of its own for L = 1 (C = 2) is not built: its first launch raised
// "an illegal instruction was encountered" in two of four runs, for a cause
// not found in its source.
template <int OP, int DK, int DV, int TV, bool FOLD>
cudaError_t launch_tv(const AppendParams &p, cudaStream_t s) {
    if constexpr (FOLD) {
        if (p.L == 3) return launch_one<OP, DK, DV, TV, true, 3>(p, s);
        if (p.L == 7) return launch_one<OP, DK, DV, TV, true, 7>(p, s);
    }
    return launch_one<OP, DK, DV, TV, FOLD>(p, s);
}

template <int OP, int DK, int DV, bool FOLD>
cudaError_t launch_fold(const AppendParams &p, cudaStream_t s) {
    int sms = 0;
    cudaError_t e = sm_count(&sms);
    if (e != cudaSuccess) return e;
    switch (pick_tile(p.NH, DV, sms)) {
        case 64: return launch_tv<OP, DK, DV, 64, FOLD>(p, s);
        default: break;
    }
    return launch_tv<OP, DK, DV, 32, FOLD>(p, s);
}

// Slot list: p.L is the longest length in the list; the merge-token
// entries (the first sl.nfold) are all at that length, one short of full.
// For d_k = 128 the merge-token units take 32-column tiles (8 rows a thread
// at the append's thread count), for d_k = 64 the append's own tile.
// Measured on B200, cycles with the slots at staggered lengths, 32-column vs
// the append's tile: GDN d128 C8 26.1 vs 28.7 us/token, KDA d128 C8 52.0 vs
// 55.7; RWKV6 d64 C8 15.7 vs 14.4, C4 16.3 vs 15.6.
template <int OP, int DK, int DV, int TVA, int LX = -1>
cudaError_t launch_slots_one(const AppendParams &p, const SlotList &sl, cudaStream_t s) {
    constexpr int TVF = DK > 64 ? 32 : TVA;
    constexpr int NT = AppendShape<DK, TVA, false>::NT;
    static_assert(TVF <= NT && DK <= NT, "merge-token tile shape");
    static std::atomic<unsigned long long> smem_ok{0};
    auto kern = append_slots_kernel<OP, DK, DV, TVA, TVF, NT, LX>;
    const int ie = p.in_bf16 ? 2 : 4;
    const size_t sa = op_layout<OP, DK, TVA>(p.L, ie, true, false).bytes;
    const size_t sf = op_layout<OP, DK, TVF>(p.L, ie, true, true).bytes;
    const size_t smem = sl.nfold > 0 && sf > sa ? sf : sa;
    const size_t ma = op_layout<OP, DK, TVA>(MAXC - 1, 4, true, false).bytes;
    const size_t mf = op_layout<OP, DK, TVF>(MAXC - 1, 4, true, true).bytes;
    cudaError_t e = allow_smem(smem_ok, kern, ma > mf ? ma : mf);
    if (e != cudaSuccess) return e;
    const long long units = (long long)sl.nfold * p.H * (DV / TVF) + (long long)(sl.n - sl.nfold) * p.H * (DV / TVA);
    return launch_kernel(kern, (unsigned)units, NT, smem, p.early != 0, s, p, sl);
}

template <int OP, int DK, int DV, int TVA>
cudaError_t launch_slots_tv(const AppendParams &p, const SlotList &sl, cudaStream_t s) {
    // the merge-token entries' length is p.L: kernels of their own as in launch_tv
    if (sl.nfold > 0 && p.L == 3) return launch_slots_one<OP, DK, DV, TVA, 3>(p, sl, s);
    if (sl.nfold > 0 && p.L == 7) return launch_slots_one<OP, DK, DV, TVA, 7>(p, sl, s);
    return launch_slots_one<OP, DK, DV, TVA>(p, sl, s);
}

template <int OP, int DK, int DV>
cudaError_t launch_slots(const AppendParams &p, const SlotList &sl, cudaStream_t s) {
    int sms = 0;
    cudaError_t e = sm_count(&sms);
    if (e != cudaSuccess) return e;
    switch (pick_tile((long long)sl.n * p.H, DV, sms)) {
        case 64: return launch_slots_tv<OP, DK, DV, 64>(p, sl, s);
        default: break;
    }
    return launch_slots_tv<OP, DK, DV, 32>(p, sl, s);
}

}  // namespace append_detail
}  // namespace dl
