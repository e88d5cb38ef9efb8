// append_slots.cu -- launchers of the append + read-out kernel over a list
// of slots, each at its own log length (continuous batching), the slots
// whose log the token completes taking the merge-token in the same launch.
#include "append_launch.cuh"

namespace dl {
namespace {
template <int OP, int DK, int DV>
cudaError_t launch(const AppendParams &p, const SlotList &sl, cudaStream_t s) {
    return append_detail::launch_slots<OP, DK, DV>(p, sl, s);
}

#define ROW(OP) {{launch<OP, 64, 64>, launch<OP, 64, 128>}, {launch<OP, 128, 64>, launch<OP, 128, 128>}}
const append_slots_fn table[3][2][2] = {ROW(OP_GDN), ROW(OP_KDA), ROW(OP_RWKV6)};
#undef ROW
}  // namespace

append_slots_fn get_append_slots(int op, int dk, int dv) {
    const int a = DL_DIM_INDEX(dk), b = DL_DIM_INDEX(dv);
    if (op < 0 || op > 2 || a < 0 || b < 0) return nullptr;
    return table[op][a][b];
}
}  // namespace dl
