// kernels.cuh -- sm_100a kernels of DeltaLog decode (append + read-out, merge /
// materialise, eager) for the GDN, KDA and RWKV6 recurrences.
//
// Method: "DeltaLog: Deferred Materialization of Recurrent States for Linear
// Attention Decoding" (arXiv 2608.15533), gist.science technical summary:
// base + bounded log ("Meccanismo Core: Base + Log"), value-tile parallelism
// with shared key-side metadata and the ReplayPrep / AppendDecode stages
// ("Implementazione del Kernel"), operators GDN / KDA / RWKV6.
//
// Decomposition.  A work unit is one head, or one value tile of a head when
// there are too few heads to fill the GPU (the paper's value-tile split): TV
// value columns of all d_k rows, so the key-side contractions S^T x reduce
// inside the CTA.  TV/4 threads per row, each owning a 16-byte column group,
// and RPT rows per thread held in registers: 16 for the append, the
// merge-token and the merge, 8 for the eager kernel (the launchers pick NT;
// Tile derives the rest).  The eager kernel always uses 32-column tiles.  Nothing here is
// a dense contraction worth a tensor core: per state element the append does
// 2 FMAs and the merge at most C = 16, against 4 to 8 bytes of HBM traffic.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace dl {

constexpr int OP_GDN = 0, OP_KDA = 1, OP_RWKV6 = 2;
constexpr int MAXC = 16;

// ----------------------------------------------------------- parameters --

struct AppendParams {
    const float *base;        // [NH, DK, DV]
    void *logK;               // [NH, C, DK]  in dtype
    void *logU;               // [NH, C, DV]  f32 (GDN/KDA) or in dtype (RWKV6)
    float *logLam;            // [NH, C, m]
    const void *q, *k, *v;    // [NH, DK], [NH, DK], [NH, DV] in dtype
    const float *beta;        // [NH]
    const float *g;           // [NH, m]
    const float *bonus;       // [H, DK]
    void *out;                // [NH, DV] out dtype
    int NH, H, C, L;
    float scale;
    int in_bf16, out_bf16;
    int early;                // 1: stream the base before waiting for the
                              // previous kernel (launch is a programmatic
                              // dependent and the previous kernel does not
                              // write this base)
};

// Start offsets of the first wave's CTAs: CTA b < slots * sms starts
// (b / sms) * ns nanoseconds late (slots = CTAs resident per SM).
struct Stagger {
    int ns, slots, sms;
};

struct MergeParams {
    const float *base;        // [NH, DK, DV]
    float *dst;               // [NH, DK, DV]  (== base for the in-place merge)
    const void *logK;
    const void *logU;
    const float *logLam;
    int NH, H, C, L;
    int in_bf16;
};

// The slots of one launch when log lengths differ between slots (continuous
// batching): list entry i is slot id[i] -- heads id[i] * H .. id[i] * H + H - 1
// -- at log length L[i].  The grid then covers n * H heads instead of all NH,
// and every head-indexed address (base, log, inputs, output) goes through
// the list.  Merge launches with one shared length take NoSlots instead.
constexpr int MAXSEL = 512;
struct SlotList {
    int n;
    int nfold;                       // append kernel: entries [0, nfold) take the merge-token
    unsigned short id[MAXSEL];
    unsigned char L[MAXSEL];
};
struct NoSlots {};
template <bool SLOTS>
using SlotArg = typename std::conditional<SLOTS, SlotList, NoSlots>::type;

// Head index (in [0, NH)) and log length of launch-local head `lh`.
template <bool SLOTS>
__device__ __forceinline__ void slot_head(const SlotArg<SLOTS> &sl, int lh, int H, int L0,
                                          int &head, int &L) {
    if constexpr (SLOTS) {
        const int i = lh / H;
        head = (int)sl.id[i] * H + (lh - i * H);
        L = sl.L[i];
    } else {
        head = lh;
        L = L0;
    }
}

struct EagerParams {
    float *S;                 // [NH, DK, DV] read and rewritten
    const void *q, *k, *v;
    const float *beta, *g, *bonus;
    void *out;
    int NH, H;
    float scale;
    int in_bf16, out_bf16;
};

// -------------------------------------------------------------- helpers --

__device__ __forceinline__ float4 ld_state(const float *p) {
    // state tile that this kernel also writes back (coherent path)
    return *reinterpret_cast<const float4 *>(p);
}

__device__ __forceinline__ void st_state(float *p, float4 v) {
    *reinterpret_cast<float4 *>(p) = v;
}

__device__ __forceinline__ float ld_in(const void *p, size_t i, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ void st_out(void *p, size_t i, float x, int bf16) {
    if (bf16)
        reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
    else
        reinterpret_cast<float *>(p)[i] = x;
}

// element i of a raw vector in shared (or global) memory, either dtype
__device__ __forceinline__ float ld_raw(const void *p, int i, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

// Asynchronous global -> shared copies (sm_80+ cp.async; completion is
// awaited with cp.async.wait_all, a hardware wait).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa), "l"(gmem) : "memory");
}

// L2 eviction priorities (createpolicy + .L2::cache_hint), used by the
// append kernel: the read-once base stream is marked evict-first, so that it
// does not push out of L2 what the next decode token reads again -- the log
// entries, written and read evict-last while the log is live.  The
// merge-token reads its log evict-first (the log is dropped after it) and
// its base tile, read and written back, without a policy.  Measured on B200
// in a four-layer merge cycle: 1.4 % (GDN) to 3.7 % (RWKV6) faster than
// without hints; the kernels that read and write the state tile (merge,
// merge-token) are faster without hints on it.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ float4 ld_stream_hint(const float *p, uint64_t pol) {
    float4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p), "l"(pol));
    return r;
}

__device__ __forceinline__ void st_f32_hint(float *p, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_b16_hint(void *p, uint16_t v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(p), "h"(v), "l"(pol) : "memory");
}

// element copy into the log (input dtype), with an L2 policy
__device__ __forceinline__ void copy_raw_hint(void *dst, size_t di, const void *src, int si, int bf16,
                                              uint64_t pol) {
    if (bf16)
        st_b16_hint(reinterpret_cast<uint16_t *>(dst) + di, reinterpret_cast<const uint16_t *>(src)[si], pol);
    else
        st_f32_hint(reinterpret_cast<float *>(dst) + di, reinterpret_cast<const float *>(src)[si], pol);
}

__device__ __forceinline__ void cp_async16_hint(void *smem, const void *gmem, uint64_t pol) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void cp_async4_hint(void *smem, const void *gmem, uint64_t pol) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 4, %2;" ::"r"(sa), "l"(gmem), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// acc += w * s on four lanes as two paired fp32 FMAs (sm_100 FFMA2; each
// lane is one correctly rounded fused multiply-add, as fmaf)
__device__ __forceinline__ void fma4(float4 &acc, float w, const float4 &s) {
    const float2 ww = make_float2(w, w);
    const float2 lo = __ffma2_rn(ww, make_float2(s.x, s.y), make_float2(acc.x, acc.y));
    const float2 hi = __ffma2_rn(ww, make_float2(s.z, s.w), make_float2(acc.z, acc.w));
    acc = make_float4(lo.x, lo.y, hi.x, hi.y);
}

// s + w * t on four lanes
__device__ __forceinline__ float4 fma4_ret(const float4 &s, float w, const float4 &t) {
    float4 o = s;
    fma4(o, w, t);
    return o;
}

// a * s + b * t on four lanes
__device__ __forceinline__ float4 fma4_2(float a, const float4 &s, float b, const float4 &t) {
    const float2 aa = make_float2(a, a), bb = make_float2(b, b);
    const float2 lo = __ffma2_rn(aa, make_float2(s.x, s.y), __fmul2_rn(bb, make_float2(t.x, t.y)));
    const float2 hi = __ffma2_rn(aa, make_float2(s.z, s.w), __fmul2_rn(bb, make_float2(t.z, t.w)));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Tile geometry shared by the kernels.
template <int DK, int DV, int TV, int NT>
struct Tile {
    static constexpr int NVT = DV / TV;      // value tiles per head
    static constexpr int TPR = TV / 4;       // threads per row (one float4 each)
    static constexpr int RG = NT / TPR;      // row groups
    static constexpr int RPT = DK / RG;      // rows per thread
    static constexpr int NW = NT / 32;       // warps
    static constexpr int RG_PER_WARP = 32 / TPR;
    static_assert(DV % TV == 0, "value tile must divide d_v");
    static_assert(TV % 4 == 0 && TPR <= 32 && 32 % TPR == 0, "bad value tile");
    static_assert(NT % 32 == 0 && NT % TPR == 0, "bad thread count");
    static_assert(DK % RG == 0, "row groups must divide d_k");
};

// Reduce NA per-thread partial float4 sums over all row groups of the CTA.
// On return xs[a][c] (c < TV) holds the full column sums.  `red` must hold
// NA * NW * TV floats.  Ends with __syncthreads().
template <int NA, int TV, int NT>
__device__ __forceinline__ void reduce_rows(float4 (&acc)[NA], float *red, float *xs) {
    constexpr int TPR = TV / 4;
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int a = 0; a < NA; ++a) {
#pragma unroll
        for (int o = TPR; o < 32; o <<= 1) {
            acc[a].x += __shfl_xor_sync(0xffffffffu, acc[a].x, o);
            acc[a].y += __shfl_xor_sync(0xffffffffu, acc[a].y, o);
            acc[a].z += __shfl_xor_sync(0xffffffffu, acc[a].z, o);
            acc[a].w += __shfl_xor_sync(0xffffffffu, acc[a].w, o);
        }
    }
    if (lane < TPR) {
#pragma unroll
        for (int a = 0; a < NA; ++a)
            *reinterpret_cast<float4 *>(&red[(a * NW + warp) * TV + lane * 4]) = acc[a];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < NA * TV; idx += NT) {
        const int a = idx / TV, c = idx % TV;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) s += red[(a * NW + w) * TV + c];
        xs[a * TV + c] = s;
    }
    __syncthreads();
}

// The same partial sums, left with the threads below TV: thread c gets
// column c's sums in xs[a] (the other threads' xs are not set).  One barrier
// instead of two: the sums go straight to the value side.
template <int NA, int TV, int NT>
__device__ __forceinline__ void reduce_cols(float4 (&acc)[NA], float *red, float (&xs)[NA]) {
    constexpr int TPR = TV / 4;
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int a = 0; a < NA; ++a) {
#pragma unroll
        for (int o = TPR; o < 32; o <<= 1) {
            acc[a].x += __shfl_xor_sync(0xffffffffu, acc[a].x, o);
            acc[a].y += __shfl_xor_sync(0xffffffffu, acc[a].y, o);
            acc[a].z += __shfl_xor_sync(0xffffffffu, acc[a].z, o);
            acc[a].w += __shfl_xor_sync(0xffffffffu, acc[a].w, o);
        }
    }
    if (lane < TPR) {
#pragma unroll
        for (int a = 0; a < NA; ++a)
            *reinterpret_cast<float4 *>(&red[(a * NW + warp) * TV + lane * 4]) = acc[a];
    }
    __syncthreads();
    if ((int)threadIdx.x < TV) {
#pragma unroll
        for (int a = 0; a < NA; ++a) {
            float t = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) t += red[(a * NW + w) * TV + threadIdx.x];
            xs[a] = t;
        }
    }
}

// ===================================================== operand staging ==
//
// The append, merge-token and merge kernels hold their base tile in
// registers (16-byte loads issued first, so they are in flight while
// everything else happens) and stage the small operands -- the token's rows,
// its decay, beta or bonus, and the L logged entries -- in dynamic shared
// memory with cp.async issued by warp 0 alone, waited for with
// cp.async.wait_all (a hardware wait) and published with __syncthreads.

__host__ __device__ constexpr int up16(int x) { return (x + 15) & ~15; }
__host__ __device__ constexpr int up4(int x) { return (x + 3) & ~3; }

// Byte offsets of the staged operands (all 16-byte aligned).
struct OpLayout {
    int kin, qin, vin, g, beta, bonus, K, lam, U, A, bytes;
};

// token: stage the token's k, q (r), v tile, g, beta / bonus.  A: room for
// the [DK][up4(L) + 4] fp32 table of per-row replay factors (merge,
// merge-token).
template <int OP, int DK, int TV>
__host__ __device__ inline OpLayout op_layout(int L, int ie, bool token, bool table) {
    const int M = (OP == OP_GDN) ? 1 : DK;
    const int ue = (OP == OP_RWKV6) ? ie : 4;
    OpLayout s{};
    int o = 0;
    s.kin = o; o += token ? up16(DK * ie) : 0;
    s.qin = o; o += token ? up16(DK * ie) : 0;
    s.vin = o; o += token ? up16(TV * ie) : 0;
    s.g = o; o += token ? up16(M * 4) : 0;
    s.beta = o; o += token ? 16 : 0;
    s.bonus = o; o += (token && OP == OP_RWKV6) ? DK * 4 : 0;
    s.K = o; o += up16(L * DK * ie);
    s.lam = o; o += up16(L * M * 4);
    s.U = o; o += up16(L * TV * ue);
    s.A = o; o += table ? DK * (up4(L) + 4) * 4 : 0;
    s.bytes = o;
    return s;
}

// warp-level copy of `bytes` (a multiple of 16; 16-byte aligned addresses)
__device__ __forceinline__ void warp_copy(unsigned char *dst, const void *src, int bytes, int lane) {
    const char *g = static_cast<const char *>(src);
    for (int o = lane * 16; o < bytes; o += 32 * 16) cp_async16(dst + o, g + o);
}

// cp.async of 16 / 4 bytes with an L2 policy (HINT) or without one
template <bool HINT>
__device__ __forceinline__ void cp16(void *smem, const void *gmem, uint64_t pol) {
    if constexpr (HINT)
        cp_async16_hint(smem, gmem, pol);
    else
        cp_async16(smem, gmem);
}
template <bool HINT>
__device__ __forceinline__ void cp4(void *smem, const void *gmem, uint64_t pol) {
    if constexpr (HINT)
        cp_async4_hint(smem, gmem, pol);
    else
        cp_async4(smem, gmem);
}
template <bool HINT>
__device__ __forceinline__ void warp_copy_pol(unsigned char *dst, const void *src, int bytes, int lane,
                                              uint64_t pol) {
    const char *g = static_cast<const char *>(src);
    for (int o = lane * 16; o < bytes; o += 32 * 16) cp16<HINT>(dst + o, g + o, pol);
}

// Sources of one head's staged operands.
struct OpSources {
    const void *k, *q, *v;          // token rows (NULL: not staged)
    const float *g, *beta, *bonus;
    const void *logK, *logU;
    const float *logLam;
};

// Stage one unit's operands (warp 0 only), then wait for them.  The log
// entries are read with the L2 policy log_pol when HINT is set.
template <int OP, int DK, int DV, int TV, bool HINT>
__device__ __forceinline__ void stage_ops(unsigned char *sm, const OpLayout &lay, const OpSources &src,
                                          int head, int vt, int L, int C, int H, int ie, bool token,
                                          uint64_t log_pol) {
    constexpr int M = (OP == OP_GDN) ? 1 : DK;
    const int ue = (OP == OP_RWKV6) ? ie : 4;
    const int lane = threadIdx.x & 31;
    if (token) {
        warp_copy(sm + lay.kin, static_cast<const char *>(src.k) + (size_t)head * DK * ie, DK * ie, lane);
        warp_copy(sm + lay.qin, static_cast<const char *>(src.q) + (size_t)head * DK * ie, DK * ie, lane);
        warp_copy(sm + lay.vin, static_cast<const char *>(src.v) + ((size_t)head * DV + vt * TV) * ie,
                  TV * ie, lane);
        if (OP == OP_GDN) {
            if (lane == 0) cp_async4(sm + lay.g, src.g + head);
        } else {
            warp_copy(sm + lay.g, src.g + (size_t)head * DK, DK * 4, lane);
        }
        if (OP == OP_RWKV6)
            warp_copy(sm + lay.bonus, src.bonus + (size_t)(head % H) * DK, DK * 4, lane);
        else if (lane == 1)
            cp_async4(sm + lay.beta, src.beta + head);
    }
    warp_copy_pol<HINT>(sm + lay.K, static_cast<const char *>(src.logK) + (size_t)head * C * DK * ie,
                        L * DK * ie, lane, log_pol);
    const float *lamh = src.logLam + (size_t)head * C * M;
    if (OP == OP_GDN) {
        for (int j = lane; j < L; j += 32) cp4<HINT>(sm + lay.lam + 4 * j, lamh + j, log_pol);
    } else {
        warp_copy_pol<HINT>(sm + lay.lam, lamh, L * DK * 4, lane, log_pol);
    }
    const char *lU = static_cast<const char *>(src.logU) + ((size_t)head * C * DV + vt * TV) * ue;
    const int cpr = TV * ue / 16;
    for (int idx = lane; idx < L * cpr; idx += 32) {
        const int j = idx / cpr, c = idx - j * cpr;
        cp16<HINT>(sm + lay.U + j * TV * ue + c * 16, lU + (size_t)j * DV * ue + c * 16, log_pol);
    }
    cp_async_wait_all();
}

// Four consecutive elements of a raw vector in shared memory as fp32.
__device__ __forceinline__ float4 ld_raw4(const unsigned char *p, int i, int bf16) {
    if (bf16) {
        const uint2 w = *reinterpret_cast<const uint2 *>(p + 2 * i);
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
    }
    return *reinterpret_cast<const float4 *>(p + 4 * i);
}

// Replay-factor table A[i][j] = exp(lam[i] - Lambda_j[i]) k_j[i] for j < L
// (pitch up4(L) + 4 floats) and the base decay gam[i] = exp(lam[i]), where
// lam is Lambda_L (merge) or Lambda_t (merge-token).  All NT threads.
template <int OP, int DK, int NT>
__device__ __forceinline__ void replay_table(float *A, float *gam, const float *lam_row,
                                             const unsigned char *sK, const float *slam, int L, int bf16) {
    constexpr int M = (OP == OP_GDN) ? 1 : DK;
    const int AP = up4(L) + 4;
    for (int idx = threadIdx.x; idx < DK * (L + 1); idx += NT) {
        const int i = idx % DK, j = idx / DK;           // j == L -> base decay
        const int x = (OP == OP_GDN) ? 0 : i;
        if (j == L)
            gam[i] = expf(lam_row[x]);
        else
            A[i * AP + j] = expf(lam_row[x] - slam[j * M + x]) * ld_raw(sK, j * DK + i, bf16);
    }
}

// ============================================ append + read-out (+ fold) ==
//
// One CTA per unit (a head, or a TV-column value tile of a head).
// ReplayPrep (once per CTA): decay point Lambda_t = Lambda_{L-1} + g_t
// (RWKV6 reads at Lambda_{t-1}), read-out weights Gamma * k, Gamma * q (RWKV6:
// Gamma * r), replay coefficients c_j = sum_i k_i k_j[i] e^{Lam[i] - Lam_j[i]}
// (d_j with q) and the self term k.q (RWKV6: r.(bonus*k)).  AppendDecode:
// x = Sbar^T w over the register tile (the one base read), value-side replay,
// delta correction, output.
// ("Fase di Append"): u_t, k_t and Lambda_t go to log slot L; the base is
// not written.
//
// append_unit does one unit (head, value tile vt) at log length L;
// append_kernel runs it (or merge_token_unit, below) over all heads at the
// shared length p.L, and append_slots_kernel over a slot list whose first
// nfold entries take the merge-token and the rest the append (one launch per
// step however the slots' lengths are spread).  nap > 0 holds the unit for
// nap nanoseconds once its base loads have gone out (a first-wave start
// offset taken there; see append_kernel).
template <int OP, int DK, int DV, int TV, int NT>
__device__ __forceinline__ void append_unit(const AppendParams &p, const int head, const int vt,
                                            const int L, const unsigned nap = 0u) {
    using T = Tile<DK, DV, TV, NT>;
    constexpr int M = (OP == OP_GDN) ? 1 : DK;
    constexpr int NA = (OP == OP_RWKV6) ? 1 : 2;
    static_assert(TV <= NT && DK <= NT, "one thread per key row and per value column");

    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ float s_lt[DK];           // Lambda_t
    __shared__ float s_lr[DK];           // decay point of read-out and replay
    __shared__ float s_k[DK];
    __shared__ float s_q[DK];
    __shared__ float s_w[NA][DK];        // read-out weights
    __shared__ float s_bk[OP == OP_RWKV6 ? DK : 1];
    __shared__ float s_coef[NA][MAXC];   // replay coefficients (c_j, d_j)
    __shared__ float s_self;             // k.q (GDN/KDA) or r.(bonus*k) (RWKV6)
    __shared__ __align__(16) float s_red[NA * T::NW * TV];

    const int tid = threadIdx.x;
    const int C = p.C;
    const int ie = p.in_bf16 ? 2 : 4;
    const int col4 = tid % T::TPR, rg = tid / T::TPR;
    const int c4 = col4 * 4;
    const OpLayout lay = op_layout<OP, DK, TV>(L, ie, true, false);

    // 1. the base stream: RPT rows x 16 bytes per thread.  As a programmatic
    //    dependent launch (merge cycles over several layers) the stream
    //    starts before the previous kernel -- another layer's -- has
    //    finished; everything else this kernel reads or writes comes after
    //    griddepcontrol.wait (a no-op for an ordinary launch).
    float *bh = const_cast<float *>(p.base) + (size_t)head * DK * DV + vt * TV + c4;
    const uint64_t pol_first = l2_evict_first(), pol_last = l2_evict_last();
    float4 s[T::RPT];
    auto load_base = [&]() {
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) s[r] = ld_stream_hint(bh + (size_t)(rg + r * T::RG) * DV, pol_first);
    };
    if (p.early) load_base();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!p.early) load_base();
    if (nap) __nanosleep(nap);

    // 2. small operands, staged by warp 0 while the base loads are in flight
    if (tid < 32) {
        const OpSources src{p.k, p.q, p.v, p.g, p.beta, p.bonus, p.logK, p.logU, p.logLam};
        stage_ops<OP, DK, DV, TV, true>(dsm, lay, src, head, vt, L, C, p.H, ie, true, pol_last);
    }
    __syncthreads();
    const float *sg = reinterpret_cast<const float *>(dsm + lay.g);
    const float *slam = reinterpret_cast<const float *>(dsm + lay.lam);

    // 3. key side: decay point, read-out weights (append: k_t, Lambda_t to slot L)
    if (tid < DK) {
        const int i = tid;
        const int x = (OP == OP_GDN) ? 0 : i;
        const float lprev = L > 0 ? slam[(L - 1) * M + x] : 0.f;
        const float lt = lprev + sg[x];
        const float lr = (OP == OP_RWKV6) ? lprev : lt;
        const float kf = ld_raw(dsm + lay.kin, i, p.in_bf16);
        const float qf = ld_raw(dsm + lay.qin, i, p.in_bf16);
        const float gam = expf(lr);
        s_lt[i] = lt;
        s_lr[i] = lr;
        s_k[i] = kf;
        s_q[i] = qf;
        if (OP == OP_RWKV6) {
            s_w[0][i] = gam * qf;
            s_bk[i] = reinterpret_cast<const float *>(dsm + lay.bonus)[i] * kf;
        } else {
            s_w[0][i] = gam * kf;
            s_w[NA - 1][i] = gam * qf;
        }
        if (vt == 0) {
            copy_raw_hint(p.logK, ((size_t)head * C + L) * DK + i, dsm + lay.kin, i, p.in_bf16, pol_last);
            if (OP != OP_GDN || i == 0) st_f32_hint(p.logLam + ((size_t)head * C + L) * M + x, lt, pol_last);
        }
    }
    __syncthreads();

    // replay coefficients: task tau < L is log entry tau, tau == L the self term
    {
        const int lane = tid & 31, warp = tid >> 5;
        for (int tau = warp; tau <= L; tau += T::NW) {
            float a0 = 0.f, a1 = 0.f;
            if (tau < L) {
                const float gdec = (OP == OP_GDN) ? expf(s_lr[0] - slam[tau]) : 1.f;
#pragma unroll
                for (int i = lane; i < DK; i += 32) {
                    const float kj = ld_raw(dsm + lay.K, tau * DK + i, p.in_bf16);
                    const float e = (OP == OP_GDN) ? kj : expf(s_lr[i] - slam[tau * M + i]) * kj;
                    if (OP == OP_RWKV6) {
                        a0 = fmaf(s_q[i], e, a0);
                    } else {
                        a0 = fmaf(s_k[i], e, a0);
                        a1 = fmaf(s_q[i], e, a1);
                    }
                }
                a0 = warp_sum(a0) * gdec;
                if (NA == 2) a1 = warp_sum(a1) * gdec;
                if (lane == 0) {
                    s_coef[0][tau] = a0;
                    if (NA == 2) s_coef[NA - 1][tau] = a1;
                }
            } else {
#pragma unroll
                for (int i = lane; i < DK; i += 32)
                    a0 = fmaf(s_q[i], (OP == OP_RWKV6) ? s_bk[i] : s_k[i], a0);
                a0 = warp_sum(a0);
                if (lane == 0) s_self = a0;
            }
        }
    }
    __syncthreads();

    // 4. base read-out: x_a[c] = sum_i w_a[i] * Sbar[i][c]
    float xc[NA];
    {
        float4 acc[NA];
#pragma unroll
        for (int a = 0; a < NA; ++a) acc[a] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const int row = rg + r * T::RG;
#pragma unroll
            for (int a = 0; a < NA; ++a) {
                const float w = s_w[a][row];
                fma4(acc[a], w, s[r]);
            }
        }
        reduce_cols<NA, TV, NT>(acc, s_red, xc);
    }

    // 5. value side: log replay, delta correction, output, append of u
    if (tid < TV) {
        const int c = tid;
        const int col = vt * TV + c;
        const size_t ub = (size_t)head * C * DV + col;
        const float vv = ld_raw(dsm + lay.vin, c, p.in_bf16);
        if (OP == OP_RWKV6) {
            float rr = 0.f;
            for (int j = 0; j < L; ++j)
                rr = fmaf(s_coef[0][j], ld_raw(dsm + lay.U, j * TV + c, p.in_bf16), rr);
            const float o = p.scale * (xc[0] + rr + s_self * vv);
            st_out(p.out, (size_t)head * DV + col, o, p.out_bf16);
            copy_raw_hint(p.logU, ub + (size_t)L * DV, dsm + lay.vin, c, p.in_bf16, pol_last);
        } else {
            const float *U = reinterpret_cast<const float *>(dsm + lay.U);
            float rk = 0.f, rq = 0.f;
            for (int j = 0; j < L; ++j) {
                const float uj = U[j * TV + c];
                rk = fmaf(s_coef[0][j], uj, rk);
                rq = fmaf(s_coef[1][j], uj, rq);
            }
            const float beta = *reinterpret_cast<const float *>(dsm + lay.beta);
            const float u = beta * (vv - xc[0] - rk);
            const float o = p.scale * (xc[NA - 1] + rq + s_self * u);
            st_out(p.out, (size_t)head * DV + col, o, p.out_bf16);
            st_f32_hint(reinterpret_cast<float *>(p.logU) + ub + (size_t)L * DV, u, pol_last);
        }
    }
}

// ====================================================== merge-token ==
//
// The token that completes the log ("Fase di Merge"): the logical state
// after this token is written over the base tile, which is read once and
// written once; the log is left for the caller to reset (L = 0).  Since the
// whole log has to be replayed into the tile anyway, the tile is folded
// first -- base decayed to the decay point plus every logged factor,
// S' = D(e^{Lambda_r}) Sbar + sum_j D(e^{Lambda_r - Lambda_j}) k_j u_j^T, with
// Lambda_r = Lambda_t (GDN/KDA) or Lambda_{t-1} (RWKV6) -- and read out from
// there, so the replay coefficients and the value-side replay of the append
// are not needed:
//   GDN/KDA  x_k = S'^T k, x_q = S'^T q, u = beta (v - x_k),
//            o = scale (x_q + (k.q) u),  S_t = S' + k u^T
//   RWKV6    o = scale (S'^T r + (r.(bonus*k)) v),  S_t = D(e^{g_t}) S' + k v^T
// LX >= 0 fixes the log length at compile time (L = LX, the common
// capacities), so that the table and fold loops have constant trip counts.
// nap as for append_unit.
template <int OP, int DK, int DV, int TV, int NT, int LX = -1>
__device__ __forceinline__ void merge_token_unit(const AppendParams &p, const int head, const int vt,
                                                 const int Lrt, const unsigned nap = 0u) {
    const int L = LX >= 0 ? LX : Lrt;
    using T = Tile<DK, DV, TV, NT>;
    constexpr int M = (OP == OP_GDN) ? 1 : DK;
    constexpr int NA = (OP == OP_RWKV6) ? 1 : 2;
    static_assert(TV <= NT && DK <= NT, "one thread per key row and per value column");

    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ float s_gam[DK];          // decay of the base to the decay point
    __shared__ float s_w[NA][DK];        // read-out weights: k, q (GDN/KDA) or r (RWKV6)
    __shared__ float s_k[DK];
    __shared__ float s_a[OP == OP_RWKV6 ? DK : 1];   // RWKV6: this token's decay e^{g_t}
    __shared__ float s_self;             // k.q (GDN/KDA) or r.(bonus*k) (RWKV6)
    __shared__ __align__(16) float s_red[NA * T::NW * TV];
    __shared__ __align__(16) float s_u[TV];

    const int tid = threadIdx.x;
    const int ie = p.in_bf16 ? 2 : 4;
    const int col4 = tid % T::TPR, rg = tid / T::TPR;
    const int c4 = col4 * 4;
    const OpLayout lay = op_layout<OP, DK, TV>(L, ie, true, true);

    // 1. the base tile (read and written back: coherent loads, no L2 policy
    //    -- an evict-first hint on this read-write tile measured 2-4 % slower
    //    on B200), streamed before the wait on the previous kernel when that
    //    one cannot be writing this base (see append_unit)
    float *bh = const_cast<float *>(p.base) + (size_t)head * DK * DV + vt * TV + c4;
    const uint64_t pol_first = l2_evict_first();
    float4 s[T::RPT];
    auto load_base = [&]() {
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) s[r] = ld_state(bh + (size_t)(rg + r * T::RG) * DV);
    };
    if (p.early) load_base();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!p.early) load_base();
    if (nap) __nanosleep(nap);

    // 2. small operands and the log, staged by warp 0 (read once: evict-first)
    if (tid < 32) {
        const OpSources src{p.k, p.q, p.v, p.g, p.beta, p.bonus, p.logK, p.logU, p.logLam};
        stage_ops<OP, DK, DV, TV, true>(dsm, lay, src, head, vt, L, p.C, p.H, ie, true, pol_first);
    }
    __syncthreads();
    const float *sg = reinterpret_cast<const float *>(dsm + lay.g);
    const float *slam = reinterpret_cast<const float *>(dsm + lay.lam);
    float *A = reinterpret_cast<float *>(dsm + lay.A);
    const int AP = up4(L) + 4;

    // 3. replay-factor table A[i][j] = e^{Lambda_r[i] - Lambda_j[i]} k_j[i],
    //    base decay, read-out weights (all threads); the self term (warp 0)
#pragma unroll
    for (int idx = tid; idx < DK * (L + 1); idx += NT) {
        const int i = idx % DK, j = idx / DK;
        const int x = (OP == OP_GDN) ? 0 : i;
        const float lprev = L > 0 ? slam[(L - 1) * M + x] : 0.f;
        const float lr = (OP == OP_RWKV6) ? lprev : lprev + sg[x];
        if (j < L) {
            A[i * AP + j] = expf(lr - slam[j * M + x]) * ld_raw(dsm + lay.K, j * DK + i, p.in_bf16);
        } else {
            const float kf = ld_raw(dsm + lay.kin, i, p.in_bf16);
            const float qf = ld_raw(dsm + lay.qin, i, p.in_bf16);
            s_gam[i] = expf(lr);
            s_k[i] = kf;
            s_w[0][i] = (OP == OP_RWKV6) ? qf : kf;
            s_w[NA - 1][i] = qf;
            if (OP == OP_RWKV6) s_a[i] = expf(sg[i]);
        }
    }
    if (tid < 32) {
        float a0 = 0.f;
#pragma unroll
        for (int i = tid; i < DK; i += 32) {
            const float kf = ld_raw(dsm + lay.kin, i, p.in_bf16);
            const float other = (OP == OP_RWKV6) ? reinterpret_cast<const float *>(dsm + lay.bonus)[i] * kf : kf;
            a0 = fmaf(ld_raw(dsm + lay.qin, i, p.in_bf16), other, a0);
        }
        a0 = warp_sum(a0);
        if (tid == 0) s_self = a0;
    }
    __syncthreads();

    // 4. fold the log into the tile, four logged entries at a time (their
    //    value factors for the thread's columns in registers, the rows swept
    //    once per four entries), then read out x_a[c] = sum_i w_a[i] S'[i][c]
    //    in a pass of its own, so that factors and accumulators are not live
    //    together
    const int ubf = (OP == OP_RWKV6) ? p.in_bf16 : 0;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        const float g = s_gam[rg + r * T::RG];
        const float2 g2 = make_float2(g, g);
        const float2 lo = __fmul2_rn(g2, make_float2(s[r].x, s[r].y)), hi = __fmul2_rn(g2, make_float2(s[r].z, s[r].w));
        s[r] = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    auto fold_chunk = [&](const int j0) {
        float4 ur[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            ur[jj] = (j0 + jj < L) ? ld_raw4(dsm + lay.U, (j0 + jj) * TV + c4, ubf) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const float4 cf4 = *reinterpret_cast<const float4 *>(A + (rg + r * T::RG) * AP + j0);
            const float cf[4] = {cf4.x, cf4.y, cf4.z, cf4.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                if (j0 + jj < L) fma4(s[r], cf[jj], ur[jj]);
        }
    };
    if constexpr (LX >= 0) {
#pragma unroll
        for (int j0 = 0; j0 < LX; j0 += 4) fold_chunk(j0);
    } else {
        for (int j0 = 0; j0 < L; j0 += 4) fold_chunk(j0);
    }
    float xc[NA];
    {
        float4 acc[NA];
#pragma unroll
        for (int a = 0; a < NA; ++a) acc[a] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const int row = rg + r * T::RG;
#pragma unroll
            for (int a = 0; a < NA; ++a) fma4(acc[a], s_w[a][row], s[r]);
        }
        reduce_cols<NA, TV, NT>(acc, s_red, xc);
    }

    // 5. value side: delta correction (GDN/KDA), output
    if (tid < TV) {
        const int c = tid;
        const int col = vt * TV + c;
        const float vv = ld_raw(dsm + lay.vin, c, p.in_bf16);
        if (OP == OP_RWKV6) {
            st_out(p.out, (size_t)head * DV + col, p.scale * (xc[0] + s_self * vv), p.out_bf16);
            s_u[c] = vv;
        } else {
            const float beta = *reinterpret_cast<const float *>(dsm + lay.beta);
            const float u = beta * (vv - xc[0]);
            st_out(p.out, (size_t)head * DV + col, p.scale * (xc[NA - 1] + s_self * u), p.out_bf16);
            s_u[c] = u;
        }
    }
    __syncthreads();

    // 6. the state after this token over the base tile
    const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[c4]);
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        const int row = rg + r * T::RG;
        const float4 o = (OP == OP_RWKV6) ? fma4_2(s_a[row], s[r], s_k[row], u4) : fma4_ret(s[r], s_k[row], u4);
        st_state(bh + (size_t)row * DV, o);
    }
}

template <int OP, int DK, int DV, int TV, int NT, bool FOLD, int LX = -1>
__global__ void __launch_bounds__(NT, 640 / NT)
append_kernel(const AppendParams p, const Stagger st) {
    using T = Tile<DK, DV, TV, NT>;
    // The first wave's CTAs of an SM would otherwise run their serial phases
    // in step, with none of them loading meanwhile; starting them a fraction
    // of a CTA's lifetime apart keeps part of the SM streaming throughout.
    // In a programmatic dependent launch with d_k = 128 the offset is taken
    // after the base loads have gone out and the previous kernel has
    // finished, so that the early stream still overlaps that kernel's tail;
    // otherwise before anything.  Measured on B200 in four-layer merge
    // cycles against the offset taken first: GDN -2.0 %, KDA -2.0 % per
    // token, isolated launches unchanged.  For d_k = 64 (RWKV6) the offset
    // after the loads gave +4 % per token, or -2 % (C = 8) with only the
    // append's moved at +3 % isolated, so d_k = 64 keeps it first.
    const unsigned nap = (st.ns > 0 && (int)blockIdx.x < st.slots * st.sms)
                             ? (unsigned)((int)blockIdx.x / st.sms) * (unsigned)st.ns : 0u;
    const bool late = DK > 64 && p.early;
    if (nap && !late) __nanosleep(nap);
    const int lh = (int)blockIdx.x / T::NVT;
    if constexpr (FOLD)
        merge_token_unit<OP, DK, DV, TV, NT, LX>(p, lh, (int)blockIdx.x - lh * T::NVT, p.L, late ? nap : 0u);
    else
        append_unit<OP, DK, DV, TV, NT>(p, lh, (int)blockIdx.x - lh * T::NVT, p.L, late ? nap : 0u);
}

// The same step over a slot list, each slot at its own log length: list
// entries [0, nfold) take the merge-token, the rest the append, in one
// launch whatever the spread of lengths.  The append units run on
// TVA-column tiles at the append's own shape (16 rows a thread where that
// leaves a thread per key row and value column), the merge-token units on
// TVF-column tiles at the same thread count NT (the launcher picks TVF).
// For d_k = 128 (TVF = 32, half the append's tile) a merge-token unit moves
// about as many bytes per CTA lifetime as an append unit (half the tile,
// read and written), and the two kinds are spread
// evenly over the grid: block b is merge-token unit floor(b F / N) when that
// count steps at b (F merge-token units of N), else append unit
// b - floor(b F / N), so every wave keeps the launch's mix in flight.  For
// d_k = 64 the merge-token units come first.  Measured on B200, cycles with
// the slots at staggered lengths, spread vs first: GDN d128 C8 27.2 vs
// 28.8 us/token, KDA d128 C8 53.2 vs 57.3, RWKV6 d64 C8 17.2 vs 16.0, RWKV6
// d64 C4 16.8 vs 17.0.
template <int OP, int DK, int DV, int TVA, int TVF, int NT, int LX = -1>
__global__ void __launch_bounds__(NT, 640 / NT)
append_slots_kernel(const AppendParams p, const SlotList sl) {
    constexpr bool SPREAD = DK > 64;
    const long long F = (long long)sl.nfold * p.H * (DV / TVF);
    const long long N = F + (long long)(sl.n - sl.nfold) * p.H * (DV / TVA);
    const long long b = blockIdx.x;
    const long long f0 = SPREAD ? b * F / N : (b < F ? b : F);
    if (SPREAD ? (b + 1) * F / N > f0 : b < F) {
        constexpr int NVT = DV / TVF;
        const int u = (int)f0, lh = u / NVT, i = lh / p.H;
        merge_token_unit<OP, DK, DV, TVF, NT, LX>(p, (int)sl.id[i] * p.H + (lh - i * p.H), u - lh * NVT,
                                                      sl.L[i]);
    } else {
        constexpr int NVT = DV / TVA;
        const int u = (int)(b - f0), lh = u / NVT + sl.nfold * p.H, i = lh / p.H;
        append_unit<OP, DK, DV, TVA, NT>(p, (int)sl.id[i] * p.H + (lh - i * p.H), u - (u / NVT) * NVT,
                                         sl.L[i]);
    }
}

// ================================================= merge / materialise ==
//
// dst[i][c] = exp(Lambda_L[i]) base[i][c] + sum_{j<L} exp(Lambda_L[i] - Lambda_j[i]) k_j[i] u_j[c]
// (Lambda_L = the last entry's snapshot; L = 0 copies the base).  In place
// (dst == base) it is the merge; into another buffer it is materialise.
// One CTA per unit; the register tile is loaded first, the log staged by
// warp 0, the replay-factor table built once per CTA, and the log folded
// into the tile four entries at a time as in the merge-token (the four value
// factors of the thread's columns in registers, each row's four
// coefficients one 16-byte shared load).
template <int OP, int DK, int DV, int TV, int NT, bool SLOTS = false>
__global__ void __launch_bounds__(NT, 640 / NT)
merge_kernel(const MergeParams p, const SlotArg<SLOTS> sl) {
    using T = Tile<DK, DV, TV, NT>;
    constexpr int M = (OP == OP_GDN) ? 1 : DK;

    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ float s_gam[DK];
    __shared__ float s_lL[M];

    const int unit = blockIdx.x;
    const int lh = unit / T::NVT, vt = unit - lh * T::NVT;
    int head, L;
    slot_head<SLOTS>(sl, lh, p.H, p.L, head, L);
    const int tid = threadIdx.x;
    const int C = p.C;
    const int ie = p.in_bf16 ? 2 : 4;
    const int col4 = tid % T::TPR, rg = tid / T::TPR;
    const int c4 = col4 * 4;
    const OpLayout lay = op_layout<OP, DK, TV>(L, ie, false, true);

    const float *bh = p.base + (size_t)head * DK * DV + vt * TV + c4;
    float *dh = p.dst + (size_t)head * DK * DV + vt * TV + c4;
    float4 s[T::RPT];
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) s[r] = ld_state(bh + (size_t)(rg + r * T::RG) * DV);

    if (tid < 32) {
        const OpSources src{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, p.logK, p.logU, p.logLam};
        stage_ops<OP, DK, DV, TV, false>(dsm, lay, src, head, vt, L, C, 1, ie, false, 0);
    }
    __syncthreads();
    const float *slam = reinterpret_cast<const float *>(dsm + lay.lam);
    for (int x = tid; x < M; x += NT) s_lL[x] = L > 0 ? slam[(L - 1) * M + x] : 0.f;
    __syncthreads();
    replay_table<OP, DK, NT>(reinterpret_cast<float *>(dsm + lay.A), s_gam, s_lL, dsm + lay.K, slam, L,
                             p.in_bf16);
    __syncthreads();

    const float *A = reinterpret_cast<const float *>(dsm + lay.A);
    const int AP = up4(L) + 4;
    const int ubf = (OP == OP_RWKV6) ? p.in_bf16 : 0;
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        const float g = s_gam[rg + r * T::RG];
        const float2 g2 = make_float2(g, g);
        const float2 lo = __fmul2_rn(g2, make_float2(s[r].x, s[r].y)), hi = __fmul2_rn(g2, make_float2(s[r].z, s[r].w));
        s[r] = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    for (int j0 = 0; j0 < L; j0 += 4) {
        float4 ur[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            ur[jj] = (j0 + jj < L) ? ld_raw4(dsm + lay.U, (j0 + jj) * TV + c4, ubf) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const float4 cf4 = *reinterpret_cast<const float4 *>(A + (rg + r * T::RG) * AP + j0);
            const float cf[4] = {cf4.x, cf4.y, cf4.z, cf4.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                if (j0 + jj < L) fma4(s[r], cf[jj], ur[jj]);
        }
    }
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) st_state(dh + (size_t)(rg + r * T::RG) * DV, s[r]);
}

// ================================================================ eager ==
//
// The dense baseline: materialise and write back the full state every token.
// GDN/KDA: x_k = S^T (a*k), x_q = S^T (a*q) from one read of S; then
// u = beta (v - x_k), o = scale (x_q + (k.q) u), S <- D(a) S + k u^T.
// RWKV6: o = scale (S^T r + (r.(bonus*k)) v), S <- D(w) S + k v^T.
template <int OP, int DK, int DV, int TV, int NT>
__global__ void __launch_bounds__(NT)
eager_kernel(const EagerParams p) {
    using T = Tile<DK, DV, TV, NT>;
    constexpr int M = (OP == OP_GDN) ? 1 : DK;
    constexpr int NA = (OP == OP_RWKV6) ? 1 : 2;

    __shared__ float s_a[DK];         // decay per key row
    __shared__ float s_k[DK];
    __shared__ float s_w[NA][DK];     // read-out weights
    __shared__ float s_self;
    __shared__ __align__(16) float s_red[NA * T::NW * TV];
    __shared__ float s_x[NA * TV];
    __shared__ __align__(16) float s_u[TV];

    const int unit = blockIdx.x;
    const int head = unit / T::NVT;
    const int vt = unit - head * T::NVT;
    const int tid = threadIdx.x;
    const int col4 = tid % T::TPR, rg = tid / T::TPR;
    const int col0 = vt * TV + col4 * 4;

    float *Sh = p.S + (size_t)head * DK * DV;
    float4 s[T::RPT];
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) s[r] = ld_state(Sh + (size_t)(rg + r * T::RG) * DV + col0);

    const size_t kq_off = (size_t)head * DK;
    for (int i = tid; i < DK; i += NT) {
        const int x = (OP == OP_GDN) ? 0 : i;
        const float a = expf(p.g[(size_t)head * M + x]);
        const float kf = ld_in(p.k, kq_off + i, p.in_bf16);
        const float qf = ld_in(p.q, kq_off + i, p.in_bf16);
        s_a[i] = a;
        s_k[i] = kf;
        if (OP == OP_RWKV6) {
            s_w[0][i] = qf;
        } else {
            s_w[0][i] = a * kf;
            s_w[NA - 1][i] = a * qf;
        }
    }
    __syncthreads();
    if (tid < 32) {
        float a0 = 0.f;
        for (int i = tid; i < DK; i += 32) {
            if (OP == OP_RWKV6)
                a0 += s_w[0][i] * p.bonus[(size_t)(head % p.H) * DK + i] * s_k[i];
            else
                a0 += s_k[i] * ld_in(p.q, kq_off + i, p.in_bf16);
        }
        a0 = warp_sum(a0);
        if (tid == 0) s_self = a0;
    }

    float4 acc[NA];
#pragma unroll
    for (int a = 0; a < NA; ++a) acc[a] = make_float4(0.f, 0.f, 0.f, 0.f);

    if constexpr (OP == OP_RWKV6) {
        // the update does not depend on the read-out: write back as we go
        const size_t vo = (size_t)head * DV + col0;
        const float4 v4 = make_float4(ld_in(p.v, vo, p.in_bf16), ld_in(p.v, vo + 1, p.in_bf16),
                                      ld_in(p.v, vo + 2, p.in_bf16), ld_in(p.v, vo + 3, p.in_bf16));
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const int row = rg + r * T::RG;
            const float w = s_w[0][row], a = s_a[row], kr = s_k[row];
            fma4(acc[0], w, s[r]);
            st_state(Sh + (size_t)row * DV + col0, fma4_2(a, s[r], kr, v4));
        }
        reduce_rows<NA, TV, NT>(acc, s_red, s_x);
        for (int c = tid; c < TV; c += NT) {
            const int col = vt * TV + c;
            const float vv = ld_in(p.v, (size_t)head * DV + col, p.in_bf16);
            st_out(p.out, (size_t)head * DV + col, p.scale * (s_x[c] + s_self * vv), p.out_bf16);
        }
    } else {
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const int row = rg + r * T::RG;
#pragma unroll
            for (int a = 0; a < NA; ++a) {
                const float w = s_w[a][row];
                fma4(acc[a], w, s[r]);
            }
        }
        reduce_rows<NA, TV, NT>(acc, s_red, s_x);
        for (int c = tid; c < TV; c += NT) {
            const int col = vt * TV + c;
            const float vv = ld_in(p.v, (size_t)head * DV + col, p.in_bf16);
            const float u = p.beta[head] * (vv - s_x[c]);
            s_u[c] = u;
            st_out(p.out, (size_t)head * DV + col, p.scale * (s_x[TV + c] + s_self * u), p.out_bf16);
        }
        __syncthreads();
        const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[col4 * 4]);
#pragma unroll
        for (int r = 0; r < T::RPT; ++r) {
            const int row = rg + r * T::RG;
            const float a = s_a[row], kr = s_k[row];
            st_state(Sh + (size_t)row * DV + col0, fma4_2(a, s[r], kr, u4));
        }
    }
}

}  // namespace dl
