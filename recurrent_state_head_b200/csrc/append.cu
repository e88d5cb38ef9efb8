// append.cu -- launchers of the append + read-out kernel and its merge-token
// variant (all ops and shapes) for one log length shared by every head.
#include <mutex>

#include "append_launch.cuh"

namespace dl {
namespace {
template <int OP, int DK, int DV>
cudaError_t launch(const AppendParams &p, bool fold, cudaStream_t s) {
    return fold ? append_detail::launch_fold<OP, DK, DV, true>(p, s)
                : append_detail::launch_fold<OP, DK, DV, false>(p, s);
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

cudaError_t sm_count(int *sms) {
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        e = cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    *sms = cache[dev];
    return cudaSuccess;
}
}  // namespace dl
