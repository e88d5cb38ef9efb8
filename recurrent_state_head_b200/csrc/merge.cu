// merge.cu -- launchers of the merge / materialise kernel (all ops and
// shapes) for one log length shared by every head.
#include "merge_launch.cuh"

namespace dl {
namespace {
template <int OP, int DK, int DV>
cudaError_t launch(const MergeParams &p, cudaStream_t s) {
    const NoSlots none{};
    return merge_detail::launch<OP, DK, DV, false>(p, none, s);
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
