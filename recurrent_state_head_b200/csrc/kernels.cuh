// kernels.cuh -- sm_100a kernels of DeltaLog decode (append + read-out, merge /
// materialise, eager) for the GDN, KDA and RWKV6 recurrences.
//
// Method: "DeltaLog: Deferred Materialization of Recurrent States for Linear
// Attention Decoding" (arXiv 2608.15533), gist.science technical summary:
// base + bounded log ("Meccanismo Core: Base + Log"), value-tile parallelism
// with shared key-side metadata and the ReplayPrep / AppendDecode stages
// ("Implementazione del Kernel"), operators GDN / KDA / RWKV6.
//
// Decomposition (all kernels): one CTA per (head, value tile).  The CTA owns
// every key row i of its TV value columns, so the key-side contractions
// S^T x reduce inside the CTA: each thread streams RPT rows of one 16-byte
// column group with 128-bit loads (a warp covers 32/TPR consecutive rows of
// TV contiguous floats), folds its rows into per-column partial sums, then a
// shuffle pass and a shared-memory pass finish the reduction.  Nothing here
// is a dense contraction worth a tensor core: per state element the append
// does 2 FMAs and the merge at most C = 16, against 4 to 8 bytes of HBM.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
};

struct MergeParams {
    const float *base;        // [NH, DK, DV]
    float *dst;               // [NH, DK, DV]  (== base for the in-place merge)
    const void *logK;
    const void *logU;
    const float *logLam;
    int NH, C, L;
    int in_bf16;
};

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

__device__ __forceinline__ float4 ld_stream(const float *p) {
    // read-once state stream: bypass L1, keep the default L2 policy
    float4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

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

// raw copy of one element of an input vector (bit-exact, either dtype)
__device__ __forceinline__ void copy_in(void *dst, size_t di, const void *src, size_t si,
                                        int bf16) {
    if (bf16)
        reinterpret_cast<uint16_t *>(dst)[di] = reinterpret_cast<const uint16_t *>(src)[si];
    else
        reinterpret_cast<float *>(dst)[di] = reinterpret_cast<const float *>(src)[si];
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

// ====================================================== append + read-out ==
//
// ReplayPrep (prologue, every CTA of the head): the token's key-side read-out
// weights Gamma_t * k and Gamma_t * q (RWKV6: Gamma_{t-1} * r), the replay
// coefficients of the L logged entries and the self term.
// AppendDecode: x = Sbar^T w over the CTA's value tile (one base read), log
// replay on the value side, delta correction, output, append of u.
template <int OP, int DK, int DV, int TV, int NT>
__global__ void __launch_bounds__(NT)
append_kernel(const AppendParams p) {
    using T = Tile<DK, DV, TV, NT>;
    constexpr int M = (OP == OP_GDN) ? 1 : DK;
    constexpr int NA = (OP == OP_RWKV6) ? 1 : 2;

    __shared__ float s_k[DK];            // k
    __shared__ float s_q[DK];            // q (RWKV6: r)
    __shared__ float s_lam[DK];          // Lambda used by the replay (t, or t-1 for RWKV6)
    __shared__ float s_w[NA][DK];        // read-out weights
    __shared__ float s_coef[NA][MAXC];   // replay coefficients (c_j, d_j)
    __shared__ float s_self;             // k.q (GDN/KDA) or r.(bonus*k) (RWKV6)
    __shared__ __align__(16) float s_red[NA * T::NW * TV];
    __shared__ float s_x[NA * TV];

    const int unit = blockIdx.x;
    const int head = unit / T::NVT;
    const int vt = unit - head * T::NVT;
    const int tid = threadIdx.x;
    const int L = p.L, C = p.C;
    const int col4 = tid % T::TPR, rg = tid / T::TPR;
    const int col0 = vt * TV + col4 * 4;

    // 1. start the base stream: RPT rows x 16 bytes per thread, in flight
    //    while the prologue runs
    const float *bh = p.base + (size_t)head * DK * DV;
    float4 s[T::RPT];
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) s[r] = ld_stream(bh + (size_t)(rg + r * T::RG) * DV + col0);

    // 2. ReplayPrep: per-key quantities of this token
    const size_t kq_off = (size_t)head * DK;
    const float *lamh = p.logLam + (size_t)head * C * M;
    for (int i = tid; i < DK; i += NT) {
        const int x = (OP == OP_GDN) ? 0 : i;
        const float lprev = L > 0 ? lamh[(size_t)(L - 1) * M + x] : 0.f;
        const float lt = lprev + p.g[(size_t)head * M + x];
        const float kf = ld_in(p.k, kq_off + i, p.in_bf16);
        const float qf = ld_in(p.q, kq_off + i, p.in_bf16);
        s_k[i] = kf;
        s_q[i] = qf;
        if (OP == OP_RWKV6) {
            s_lam[i] = lprev;
            s_w[0][i] = expf(lprev) * qf;
        } else {
            s_lam[i] = lt;
            const float gam = expf(lt);
            s_w[0][i] = gam * kf;
            s_w[NA - 1][i] = gam * qf;
        }
        if (vt == 0) {
            // append the key factor and the decay snapshot at slot L
            copy_in(p.logK, ((size_t)head * C + L) * DK + i, p.k, kq_off + i, p.in_bf16);
            if (OP != OP_GDN || i == 0) p.logLam[((size_t)head * C + L) * M + x] = lt;
        }
    }
    __syncthreads();

    // replay coefficients: task tau < L is log entry tau, tau == L the self term
    {
        const int lane = tid & 31, warp = tid >> 5;
        const float *Kf = reinterpret_cast<const float *>(p.logK);
        const __nv_bfloat16 *Kb = reinterpret_cast<const __nv_bfloat16 *>(p.logK);
        for (int tau = warp; tau <= L; tau += T::NW) {
            float a0 = 0.f, a1 = 0.f;
            if (tau < L) {
                const size_t kb = ((size_t)head * C + tau) * DK;
                const float *lj = lamh + (size_t)tau * M;
                const float gdec = (OP == OP_GDN) ? expf(s_lam[0] - lj[0]) : 1.f;
                for (int i = lane; i < DK; i += 32) {
                    const float kj = p.in_bf16 ? __bfloat162float(Kb[kb + i]) : Kf[kb + i];
                    const float e = (OP == OP_GDN) ? kj : expf(s_lam[i] - lj[i]) * kj;
                    if (OP == OP_RWKV6) {
                        a0 += s_q[i] * e;
                    } else {
                        a0 += s_k[i] * e;
                        a1 += s_q[i] * e;
                    }
                }
                a0 = warp_sum(a0) * gdec;
                a1 = warp_sum(a1) * gdec;
                if (lane == 0) {
                    s_coef[0][tau] = a0;
                    if (NA == 2) s_coef[NA - 1][tau] = a1;
                }
            } else {
                for (int i = lane; i < DK; i += 32) {
                    if (OP == OP_RWKV6)
                        a0 += s_q[i] * p.bonus[(size_t)(head % p.H) * DK + i] * s_k[i];
                    else
                        a0 += s_k[i] * s_q[i];
                }
                a0 = warp_sum(a0);
                if (lane == 0) s_self = a0;
            }
        }
    }
    __syncthreads();

    // 3. base read-out: x_a[c] = sum_i w_a[i] * Sbar[i][c]
    float4 acc[NA];
#pragma unroll
    for (int a = 0; a < NA; ++a) acc[a] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        const int row = rg + r * T::RG;
#pragma unroll
        for (int a = 0; a < NA; ++a) {
            const float w = s_w[a][row];
            acc[a].x = fmaf(w, s[r].x, acc[a].x);
            acc[a].y = fmaf(w, s[r].y, acc[a].y);
            acc[a].z = fmaf(w, s[r].z, acc[a].z);
            acc[a].w = fmaf(w, s[r].w, acc[a].w);
        }
    }
    reduce_rows<NA, TV, NT>(acc, s_red, s_x);

    // 4. value side: log replay, delta correction, output, append of u
    for (int c = tid; c < TV; c += NT) {
        const int col = vt * TV + c;
        const size_t ub = (size_t)head * C * DV + col;
        const float vv = ld_in(p.v, (size_t)head * DV + col, p.in_bf16);
        if (OP == OP_RWKV6) {
            float rr = 0.f;
            for (int j = 0; j < L; ++j)
                rr = fmaf(s_coef[0][j], ld_in(p.logU, ub + (size_t)j * DV, p.in_bf16), rr);
            const float o = p.scale * (s_x[c] + rr + s_self * vv);
            st_out(p.out, (size_t)head * DV + col, o, p.out_bf16);
            copy_in(p.logU, ub + (size_t)L * DV, p.v, (size_t)head * DV + col, p.in_bf16);
        } else {
            const float *U = reinterpret_cast<const float *>(p.logU);
            float rk = 0.f, rq = 0.f;
            for (int j = 0; j < L; ++j) {
                const float uj = U[ub + (size_t)j * DV];
                rk = fmaf(s_coef[0][j], uj, rk);
                rq = fmaf(s_coef[1][j], uj, rq);
            }
            const float u = p.beta[head] * (vv - s_x[c] - rk);
            const float o = p.scale * (s_x[TV + c] + rq + s_self * u);
            st_out(p.out, (size_t)head * DV + col, o, p.out_bf16);
            reinterpret_cast<float *>(p.logU)[ub + (size_t)L * DV] = u;
        }
    }
}

// ================================================= merge / materialise ==
//
// dst[i][c] = exp(Lambda_L[i]) base[i][c] + sum_{j<L} exp(Lambda_L[i] - Lambda_j[i]) k_j[i] u_j[c]
// (Lambda_L = the last entry's snapshot; L = 0 copies the base).  In place
// (dst == base) it is the merge; into another buffer it is materialise.
template <int OP, int DK, int DV, int TV, int NT>
__global__ void __launch_bounds__(NT)
merge_kernel(const MergeParams p) {
    using T = Tile<DK, DV, TV, NT>;
    constexpr int M = (OP == OP_GDN) ? 1 : DK;

    __shared__ float s_gam[DK];
    __shared__ float s_coef[DK][MAXC + 1];   // [row][entry], padded against bank conflicts

    const int unit = blockIdx.x;
    const int head = unit / T::NVT;
    const int vt = unit - head * T::NVT;
    const int tid = threadIdx.x;
    const int L = p.L, C = p.C;
    const int col4 = tid % T::TPR, rg = tid / T::TPR;
    const int col0 = vt * TV + col4 * 4;

    const float *lamh = p.logLam + (size_t)head * C * M;
    // per-row decay of the base and replay coefficients
    for (int idx = tid; idx < DK * (L + 1); idx += NT) {
        const int i = idx % DK, j = idx / DK;          // j == L -> base decay
        const int x = (OP == OP_GDN) ? 0 : i;
        const float lL = L > 0 ? lamh[(size_t)(L - 1) * M + x] : 0.f;
        if (j == L) {
            s_gam[i] = expf(lL);
        } else {
            const float kj = ld_in(p.logK, ((size_t)head * C + j) * DK + i, p.in_bf16);
            s_coef[i][j] = expf(lL - lamh[(size_t)j * M + x]) * kj;
        }
    }
    // value factors of this thread's four columns, every logged entry
    float4 uu[MAXC];
    const size_t ub = (size_t)head * C * DV + col0;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
        if (j < L) {
            if (OP == OP_RWKV6 && p.in_bf16) {
                const __nv_bfloat16 *Ub = reinterpret_cast<const __nv_bfloat16 *>(p.logU);
                const size_t o = ub + (size_t)j * DV;
                uu[j] = make_float4(__bfloat162float(Ub[o]), __bfloat162float(Ub[o + 1]),
                                    __bfloat162float(Ub[o + 2]), __bfloat162float(Ub[o + 3]));
            } else {
                uu[j] = *reinterpret_cast<const float4 *>(
                    reinterpret_cast<const float *>(p.logU) + ub + (size_t)j * DV);
            }
        } else {
            uu[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();

    const float *bh = p.base + (size_t)head * DK * DV;
    float *dh = p.dst + (size_t)head * DK * DV;
    float4 s[T::RPT];
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) s[r] = ld_state(bh + (size_t)(rg + r * T::RG) * DV + col0);
#pragma unroll
    for (int r = 0; r < T::RPT; ++r) {
        const int row = rg + r * T::RG;
        const float gm = s_gam[row];
        float4 o = make_float4(gm * s[r].x, gm * s[r].y, gm * s[r].z, gm * s[r].w);
#pragma unroll
        for (int j = 0; j < MAXC; ++j) {
            if (j < L) {
                const float cf = s_coef[row][j];
                o.x = fmaf(cf, uu[j].x, o.x);
                o.y = fmaf(cf, uu[j].y, o.y);
                o.z = fmaf(cf, uu[j].z, o.z);
                o.w = fmaf(cf, uu[j].w, o.w);
            }
        }
        st_state(dh + (size_t)row * DV + col0, o);
    }
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
            acc[0].x = fmaf(w, s[r].x, acc[0].x);
            acc[0].y = fmaf(w, s[r].y, acc[0].y);
            acc[0].z = fmaf(w, s[r].z, acc[0].z);
            acc[0].w = fmaf(w, s[r].w, acc[0].w);
            st_state(Sh + (size_t)row * DV + col0,
                     make_float4(fmaf(a, s[r].x, kr * v4.x), fmaf(a, s[r].y, kr * v4.y),
                                 fmaf(a, s[r].z, kr * v4.z), fmaf(a, s[r].w, kr * v4.w)));
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
                acc[a].x = fmaf(w, s[r].x, acc[a].x);
                acc[a].y = fmaf(w, s[r].y, acc[a].y);
                acc[a].z = fmaf(w, s[r].z, acc[a].z);
                acc[a].w = fmaf(w, s[r].w, acc[a].w);
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
            st_state(Sh + (size_t)row * DV + col0,
                     make_float4(fmaf(a, s[r].x, kr * u4.x), fmaf(a, s[r].y, kr * u4.y),
                                 fmaf(a, s[r].z, kr * u4.z), fmaf(a, s[r].w, kr * u4.w)));
        }
    }
}

}  // namespace dl
