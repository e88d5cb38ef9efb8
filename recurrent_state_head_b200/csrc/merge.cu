// merge.cu -- launchers of the merge / materialise kernel (all ops and shapes).
#include "launch.h"

namespace dl {
namespace {
template <int OP, int DK, int DV, int TV, int LB>
cudaError_t launch_lb(const MergeParams &p, cudaStream_t s) {
    constexpr int NT = CtaShape<DK, TV>::NT;
    static std::atomic<unsigned long long> smem_ok{0};
    auto kern = merge_kernel<OP, DK, DV, TV, NT, LB>;
    const int ie = p.in_bf16 ? 2 : 4;
    const size_t smem = op_layout<OP, DK, TV>(p.L, ie, false, true).bytes;
    cudaError_t e = allow_smem(smem_ok, kern, op_layout<OP, DK, TV>(MAXC, 4, false, true).bytes);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)p.NH * (DV / TV);
    kern<<<grid, NT, smem, s>>>(p);
    return cudaGetLastError();
}

// The logged value factors stay in registers for logs of up to 8 entries.
template <int OP, int DK, int DV, int TV>
cudaError_t launch_tv(const MergeParams &p, cudaStream_t s) {
    if (p.L <= 4) return launch_lb<OP, DK, DV, TV, 4>(p, s);
    if (p.L <= 8) return launch_lb<OP, DK, DV, TV, 8>(p, s);
    return launch_lb<OP, DK, DV, TV, 0>(p, s);
}

template <int OP, int DK, int DV>
cudaError_t launch(const MergeParams &p, cudaStream_t s) {
    int sms = 0;
    cudaError_t e = sm_count(&sms);
    if (e != cudaSuccess) return e;
    switch (pick_tile(p.NH, DV, sms)) {
        case 128: if constexpr (DV >= 128) return launch_tv<OP, DK, DV, 128>(p, s); break;
        case 64: return launch_tv<OP, DK, DV, 64>(p, s);
        default: break;
    }
    return launch_tv<OP, DK, DV, 32>(p, s);
}

#define ROW(OP) {{launch<OP, 64, 64>, launch<OP, 64, 128>}, {launch<OP, 128, 64>, launch<OP, 128, 128>}}
const merge_fn table[3][2][2] = {ROW(OP_GDN), ROW(OP_KDA), ROW(OP_RWKV6)};
#undef ROW
}  // namespace

merge_fn get_merge(int op, int dk, int dv) {
    const int a = DL_DIM_INDEX(dk), b = DL_DIM_INDEX(dv);
    if (op < 0 || op > 2 || a < 0 || b < 0) return nullptr;
    return table[op][a][b];
}
}  // namespace dl
