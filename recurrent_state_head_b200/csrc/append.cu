// append.cu -- launchers of the append + read-out kernel and its merge-token
// variant (all ops and shapes).
#include <mutex>

#include "launch.h"

namespace dl {
namespace {
template <int OP, int DK, int DV, int TV, bool FOLD, int LB>
cudaError_t launch_lb(const AppendParams &p, cudaStream_t s) {
    constexpr int NT = CtaShape<DK, TV>::NT;
    static std::atomic<unsigned long long> smem_ok{0};
    auto kern = append_kernel<OP, DK, DV, TV, NT, FOLD, LB>;
    const int ie = p.in_bf16 ? 2 : 4;
    const size_t smem = op_layout<OP, DK, TV>(p.L, ie, true, FOLD).bytes;
    cudaError_t e = allow_smem(smem_ok, kern, op_layout<OP, DK, TV>(MAXC - 1, 4, true, FOLD).bytes);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)p.NH * (DV / TV);
    if (!p.early) {
        kern<<<grid, NT, smem, s>>>(p);
        return cudaGetLastError();
    }
    // programmatic dependent launch: may start while the previous kernel of
    // the stream finishes (the kernel orders itself with griddepcontrol)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// The merge-token keeps the logged value factors in registers while the log
// is short (up to 8 entries); longer logs are read from shared memory.
template <int OP, int DK, int DV, int TV, bool FOLD>
cudaError_t launch_tv(const AppendParams &p, cudaStream_t s) {
    if constexpr (FOLD) {
        if (p.L <= 4) return launch_lb<OP, DK, DV, TV, true, 4>(p, s);
        if (p.L <= 8) return launch_lb<OP, DK, DV, TV, true, 8>(p, s);
    }
    return launch_lb<OP, DK, DV, TV, FOLD, 0>(p, s);
}

template <int OP, int DK, int DV, bool FOLD>
cudaError_t launch_fold(const AppendParams &p, cudaStream_t s) {
    int sms = 0;
    cudaError_t e = sm_count(&sms);
    if (e != cudaSuccess) return e;
    switch (pick_tile(p.NH, DV, sms)) {
        case 128: if constexpr (DV >= 128) return launch_tv<OP, DK, DV, 128, FOLD>(p, s); break;
        case 64: return launch_tv<OP, DK, DV, 64, FOLD>(p, s);
        default: break;
    }
    return launch_tv<OP, DK, DV, 32, FOLD>(p, s);
}

template <int OP, int DK, int DV>
cudaError_t launch(const AppendParams &p, bool fold, cudaStream_t s) {
    return fold ? launch_fold<OP, DK, DV, true>(p, s) : launch_fold<OP, DK, DV, false>(p, s);
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
