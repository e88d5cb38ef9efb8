// append.cu -- launchers of the append + read-out kernel (all ops and shapes).
#include "launch.h"

namespace dl {
namespace {
template <int OP, int DK, int DV>
cudaError_t launch(const AppendParams &p, cudaStream_t s) {
    using LC = LaunchCfg<DK, DV>;
    const unsigned grid = (unsigned)p.NH * (DV / LC::TV);
    append_kernel<OP, DK, DV, LC::TV, LC::NT><<<grid, LC::NT, 0, s>>>(p);
    return cudaGetLastError();
}
#define ROW(OP) {{launch<OP, 64, 64>, launch<OP, 64, 128>}, {launch<OP, 128, 64>, launch<OP, 128, 128>}}
const append_fn table[3][2][2] = {ROW(OP_GDN), ROW(OP_KDA), ROW(OP_RWKV6)};
#undef ROW
}  // namespace

append_fn get_append(int op, int dk, int dv) {
    const int a = DL_DIM_INDEX(dk), b = DL_DIM_INDEX(dv);
    if (op < 0 || op > 2 || a < 0 || b < 0) return nullptr;
    return table[op][a][b];
}
}  // namespace dl
