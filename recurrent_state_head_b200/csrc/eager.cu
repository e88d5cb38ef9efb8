// eager.cu -- launchers of the eager dense-update kernel (all ops and shapes).
#include "launch.h"

namespace dl {
namespace {
template <int OP, int DK, int DV>
cudaError_t launch(const EagerParams &p, cudaStream_t s) {
    // one CTA per (head, 32-column tile), tile held in registers
    constexpr int TV = 32, NT = CtaShape<DK, TV>::NT;
    const unsigned grid = (unsigned)p.NH * (DV / TV);
    eager_kernel<OP, DK, DV, TV, NT><<<grid, NT, 0, s>>>(p);
    return cudaGetLastError();
}
#define ROW(OP) {{launch<OP, 64, 64>, launch<OP, 64, 128>}, {launch<OP, 128, 64>, launch<OP, 128, 128>}}
const eager_fn table[3][2][2] = {ROW(OP_GDN), ROW(OP_KDA), ROW(OP_RWKV6)};
#undef ROW
}  // namespace

eager_fn get_eager(int op, int dk, int dv) {
    const int a = DL_DIM_INDEX(dk), b = DL_DIM_INDEX(dv);
    if (op < 0 || op > 2 || a < 0 || b < 0) return nullptr;
    return table[op][a][b];
}
}  // namespace dl
