// deltalog.cu -- host side of libdeltalog.so: argument checks, the decode
// handle with its log-length schedule (append while L < C, merge when the
// log is full), and the graph-captured merge cycle.
//
// Method: "DeltaLog: Deferred Materialization of Recurrent States for Linear
// Attention Decoding" (arXiv 2608.15533): append / merge phases (gist.science
// technical summary, "Meccanismo Core: Base + Log"; signal-papers page,
// Fig. 4 caption) and CUDA-Graph replay of one merge cycle (Fig. 9 caption).
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <new>
#include <vector>

#include "../../include/deltalog.h"
#include "launch.h"

namespace {

thread_local char g_err[512] = "";

dl_status fail(dl_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

dl_status ok() {
    g_err[0] = '\0';
    return DL_OK;
}

dl_status cuda_fail(cudaError_t e, const char *what) {
    return fail(DL_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool dim_ok(int d) { return d == 64 || d == 128; }
size_t esize(int dt) { return dt == DL_BF16 ? 2 : 4; }
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

dl_status check_config(const dl_config *c, bool need_log) {
    if (!c) return fail(DL_EINVAL, "config is NULL");
    if (c->op < DL_GDN || c->op > DL_RWKV6) return fail(DL_EINVAL, "op %d is not GDN/KDA/RWKV6", c->op);
    if (c->B < 0 || c->H < 1) return fail(DL_EINVAL, "need B >= 0 and H >= 1 (B=%d H=%d)", c->B, c->H);
    if ((long long)c->B * c->H > (1LL << 24))
        return fail(DL_EINVAL, "B*H = %lld heads is above the supported 2^24", (long long)c->B * c->H);
    if (!dim_ok(c->dk) || !dim_ok(c->dv))
        return fail(DL_EINVAL, "d_k, d_v must be 64 or 128 (d_k=%d d_v=%d)", c->dk, c->dv);
    if (need_log && (c->C < 1 || c->C > dl::MAXC))
        return fail(DL_EINVAL, "log capacity C=%d outside [1, %d]", c->C, dl::MAXC);
    if ((c->in_dtype != DL_F32 && c->in_dtype != DL_BF16) ||
        (c->out_dtype != DL_F32 && c->out_dtype != DL_BF16))
        return fail(DL_EINVAL, "dtypes must be DL_F32 or DL_BF16");
    if (!std::isfinite(c->scale)) return fail(DL_EINVAL, "scale is not finite");
    if (need_log && (c->auto_merge < DL_MERGE_OFF || c->auto_merge > DL_MERGE_SEPARATE))
        return fail(DL_EINVAL, "auto_merge must be 0, 1 or 2");
    return DL_OK;
}

struct Layout {
    size_t K, U, Lam, total;
};

Layout log_layout(const dl_config *c) {
    const size_t nh = (size_t)c->B * c->H, C = (size_t)c->C;
    const size_t m = c->op == DL_GDN ? 1 : (size_t)c->dk;
    const size_t ue = c->op == DL_RWKV6 ? esize(c->in_dtype) : 4;
    Layout l;
    l.K = 0;
    l.U = up256(l.K + nh * C * c->dk * esize(c->in_dtype));
    l.Lam = up256(l.U + nh * C * c->dv * ue);
    l.total = up256(l.Lam + nh * C * m * 4);
    return l;
}

// Pointers of one decode step.  The kernels copy q, k, v (and the per-key
// log-decay rows) with 16-byte asynchronous copies.
dl_status check_step_ptrs(const dl_config *c, const void *q, const void *k, const void *v,
                          const float *beta, const float *g, const void *out) {
    const size_t oe = esize(c->out_dtype);
    if (!q || !k || !v || !g || !out) return fail(DL_EINVAL, "q/k/v/g/out must not be NULL");
    if (c->op != DL_RWKV6 && !beta) return fail(DL_EINVAL, "beta must not be NULL for GDN/KDA");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16))
        return fail(DL_EINVAL, "q/k/v must be 16-byte aligned");
    if (!aligned(g, c->op == DL_GDN ? 4 : 16))
        return fail(DL_EINVAL, "g must be 4-byte (GDN) or 16-byte (KDA/RWKV6) aligned");
    if (!aligned(out, oe) || (beta && !aligned(beta, 4)))
        return fail(DL_EINVAL, "out must be element aligned, beta 4-byte aligned");
    return DL_OK;
}

}  // namespace

struct dl_handle {
    dl_config cfg;
    float *base;
    char *log;
    Layout lay;
    const float *bonus;
    int L;
    int NH;
};

struct dl_cycle {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    std::vector<dl_handle *> layers;
    int kernels;
};

namespace {

dl::AppendParams append_params(const dl_handle *h, const dl_step_io &io, int L) {
    dl::AppendParams p;
    p.base = h->base;
    p.logK = h->log + h->lay.K;
    p.logU = h->log + h->lay.U;
    p.logLam = reinterpret_cast<float *>(h->log + h->lay.Lam);
    p.q = io.q;
    p.k = io.k;
    p.v = io.v;
    p.beta = io.beta;
    p.g = io.g;
    p.bonus = h->bonus;
    p.out = io.out;
    p.NH = h->NH;
    p.H = h->cfg.H;
    p.C = h->cfg.C;
    p.L = L;
    p.scale = h->cfg.scale;
    p.in_bf16 = h->cfg.in_dtype == DL_BF16;
    p.out_bf16 = h->cfg.out_dtype == DL_BF16;
    p.early = 0;
    return p;
}

dl::MergeParams merge_params(const dl_handle *h, float *dst, int L) {
    dl::MergeParams p;
    p.base = h->base;
    p.dst = dst;
    p.logK = h->log + h->lay.K;
    p.logU = h->log + h->lay.U;
    p.logLam = reinterpret_cast<const float *>(h->log + h->lay.Lam);
    p.NH = h->NH;
    p.C = h->cfg.C;
    p.L = L;
    p.in_bf16 = h->cfg.in_dtype == DL_BF16;
    return p;
}

// fold: the merge-token variant (the token that completes the log writes
// the merged state over the base instead of appending).
// early: launch as a programmatic dependent that streams its base before the
// previous kernel of the stream has finished -- only where that kernel cannot
// be writing this base (a merge cycle over several layers with distinct
// bases).
cudaError_t launch_append(const dl_handle *h, const dl_step_io &io, int L, bool fold, cudaStream_t s,
                          bool early = false) {
    if (h->NH == 0) return cudaSuccess;
    dl::AppendParams p = append_params(h, io, L);
    p.early = early ? 1 : 0;
    return dl::get_append(h->cfg.op, h->cfg.dk, h->cfg.dv)(p, fold, s);
}

// Do the layers' base states occupy pairwise disjoint memory?
bool disjoint_bases(dl_handle *const *layers, int n) {
    for (int a = 0; a < n; ++a)
        for (int b = a + 1; b < n; ++b) {
            const char *pa = reinterpret_cast<const char *>(layers[a]->base);
            const char *pb = reinterpret_cast<const char *>(layers[b]->base);
            const size_t na = (size_t)layers[a]->NH * layers[a]->cfg.dk * layers[a]->cfg.dv * 4;
            const size_t nb = (size_t)layers[b]->NH * layers[b]->cfg.dk * layers[b]->cfg.dv * 4;
            if (na && nb && pa < pb + nb && pb < pa + na) return false;
        }
    return true;
}

cudaError_t launch_merge(const dl_handle *h, float *dst, int L, cudaStream_t s) {
    if (h->NH == 0) return cudaSuccess;
    return dl::get_merge(h->cfg.op, h->cfg.dk, h->cfg.dv)(merge_params(h, dst, L), s);
}

}  // namespace

extern "C" {

size_t dl_log_bytes(const dl_config *cfg) {
    if (check_config(cfg, true) != DL_OK) return 0;
    return log_layout(cfg).total;
}

dl_status dl_log_layout(const dl_config *cfg, size_t *off_K, size_t *off_U, size_t *off_Lam) {
    dl_status s = check_config(cfg, true);
    if (s != DL_OK) return s;
    const Layout l = log_layout(cfg);
    if (off_K) *off_K = l.K;
    if (off_U) *off_U = l.U;
    if (off_Lam) *off_Lam = l.Lam;
    return ok();
}

dl_status dl_create(const dl_config *cfg, float *base, void *log_ws, const float *bonus,
                    dl_handle **out) {
    if (!out) return fail(DL_EINVAL, "out handle pointer is NULL");
    *out = nullptr;
    dl_status s = check_config(cfg, true);
    if (s != DL_OK) return s;
    const int NH = cfg->B * cfg->H;
    if (NH > 0) {
        if (!base || !log_ws) return fail(DL_EINVAL, "base and log workspace must not be NULL");
        if (!aligned(base, 16) || !aligned(log_ws, 16))
            return fail(DL_EINVAL, "base and log workspace must be 16-byte aligned");
        if (cfg->op == DL_RWKV6 && (!bonus || !aligned(bonus, 16)))
            return fail(DL_EINVAL, "RWKV6 needs a 16-byte aligned bonus [H, d_k]");
    }
    dl_handle *h = new (std::nothrow) dl_handle;
    if (!h) return fail(DL_ENOMEM, "host allocation of the handle failed");
    h->cfg = *cfg;
    h->base = base;
    h->log = static_cast<char *>(log_ws);
    h->lay = log_layout(cfg);
    h->bonus = cfg->op == DL_RWKV6 ? bonus : nullptr;
    h->L = 0;
    h->NH = NH;
    *out = h;
    return ok();
}

dl_status dl_decode_step(dl_handle *h, const void *q, const void *k, const void *v,
                         const float *beta, const float *g, void *out, void *stream) {
    if (!h) return fail(DL_EINVAL, "handle is NULL");
    if (h->NH > 0) {
        dl_status s = check_step_ptrs(&h->cfg, q, k, v, beta, g, out);
        if (s != DL_OK) return s;
    }
    if (h->L >= h->cfg.C)
        return fail(DL_ESTATE, "log is full (L = C = %d) and auto_merge is off: merge first", h->cfg.C);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const dl_step_io io = {q, k, v, beta, g, out};
    if (h->cfg.auto_merge == DL_MERGE_FOLD && h->L == h->cfg.C - 1) {
        // the token that completes the log: one kernel reads the base once
        // and writes the merged logical state back
        cudaError_t e = launch_append(h, io, h->L, true, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge-token kernel launch");
        h->L = 0;
        return ok();
    }
    cudaError_t e = launch_append(h, io, h->L, false, st);
    if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
    h->L += 1;
    if (h->cfg.auto_merge == DL_MERGE_SEPARATE && h->L == h->cfg.C) {
        e = launch_merge(h, h->base, h->L, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch");
        h->L = 0;
    }
    return ok();
}

dl_status dl_merge(dl_handle *h, void *stream) {
    if (!h) return fail(DL_EINVAL, "handle is NULL");
    if (h->L == 0) return ok();
    cudaError_t e = launch_merge(h, h->base, h->L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch");
    h->L = 0;
    return ok();
}

dl_status dl_materialize(const dl_handle *h, float *S_out, void *stream) {
    if (!h) return fail(DL_EINVAL, "handle is NULL");
    if (h->NH == 0) return ok();
    if (!S_out || !aligned(S_out, 16)) return fail(DL_EINVAL, "S_out must be non-NULL and 16-byte aligned");
    const size_t bytes = (size_t)h->NH * h->cfg.dk * h->cfg.dv * 4;
    const char *a = reinterpret_cast<const char *>(S_out), *b = reinterpret_cast<const char *>(h->base);
    if (a < b + bytes && b < a + bytes) return fail(DL_EINVAL, "S_out overlaps the base state");
    cudaError_t e = launch_merge(h, S_out, h->L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "materialize kernel launch");
    return ok();
}

dl_status dl_eager_step(const dl_config *cfg, float *S, const void *q, const void *k,
                        const void *v, const float *beta, const float *g, const float *bonus,
                        void *out, void *stream) {
    dl_status s = check_config(cfg, false);
    if (s != DL_OK) return s;
    const int NH = cfg->B * cfg->H;
    if (NH == 0) return ok();
    if (!S || !aligned(S, 16)) return fail(DL_EINVAL, "S must be non-NULL and 16-byte aligned");
    s = check_step_ptrs(cfg, q, k, v, beta, g, out);
    if (s != DL_OK) return s;
    if (cfg->op == DL_RWKV6 && (!bonus || !aligned(bonus, 16)))
        return fail(DL_EINVAL, "RWKV6 needs a 16-byte aligned bonus [H, d_k]");
    dl::EagerParams p;
    p.S = S;
    p.q = q;
    p.k = k;
    p.v = v;
    p.beta = beta;
    p.g = g;
    p.bonus = cfg->op == DL_RWKV6 ? bonus : nullptr;
    p.out = out;
    p.NH = NH;
    p.H = cfg->H;
    p.scale = cfg->scale;
    p.in_bf16 = cfg->in_dtype == DL_BF16;
    p.out_bf16 = cfg->out_dtype == DL_BF16;
    cudaError_t e = dl::get_eager(cfg->op, cfg->dk, cfg->dv)(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "eager kernel launch");
    return ok();
}

int dl_log_len(const dl_handle *h) { return h ? h->L : -1; }

void dl_destroy(dl_handle *h) { delete h; }

dl_status dl_cycle_create(dl_handle *const *layers, int n_layers, const dl_step_io *io,
                          dl_cycle **out) {
    if (!out) return fail(DL_EINVAL, "out cycle pointer is NULL");
    *out = nullptr;
    if (!layers || n_layers < 1 || !io) return fail(DL_EINVAL, "need n_layers >= 1 layers and io");
    const int C = layers[0] ? layers[0]->cfg.C : 0;
    for (int l = 0; l < n_layers; ++l) {
        const dl_handle *h = layers[l];
        if (!h) return fail(DL_EINVAL, "layer %d is NULL", l);
        if (h->cfg.C != C) return fail(DL_EINVAL, "layers must share one log capacity C");
        if (h->cfg.auto_merge == DL_MERGE_OFF) return fail(DL_EINVAL, "layer %d has auto_merge = 0", l);
        if (h->L != 0) return fail(DL_ESTATE, "layer %d has L = %d, a cycle starts at L = 0", l, h->L);
        for (int t = 0; t < C; ++t) {
            const dl_step_io &x = io[(size_t)t * n_layers + l];
            if (h->NH > 0) {
                dl_status s = check_step_ptrs(&h->cfg, x.q, x.k, x.v, x.beta, x.g, x.out);
                if (s != DL_OK) return s;
            }
        }
    }
    dl_cycle *cy = new (std::nothrow) dl_cycle;
    if (!cy) return fail(DL_ENOMEM, "host allocation of the cycle failed");
    cy->graph = nullptr;
    cy->exec = nullptr;
    cy->kernels = 0;
    try {
        cy->layers.assign(layers, layers + n_layers);
    } catch (...) {
        delete cy;
        return fail(DL_ENOMEM, "host allocation of the cycle failed");
    }
    // with two or more layers on disjoint bases, consecutive kernels of the
    // token-major cycle belong to different layers: each may start streaming
    // its base during the previous kernel's tail
    const bool overlap = n_layers >= 2 && disjoint_bases(layers, n_layers);
    cudaStream_t st = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
        delete cy;
        return cuda_fail(e, "capture stream creation");
    }
    e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
    cudaError_t le = cudaSuccess;
    if (e == cudaSuccess) {
        // token-major: every layer's step for token t; the token that
        // completes a layer's log is its merge-token (DL_MERGE_FOLD) or its
        // append followed by its merge (DL_MERGE_SEPARATE)
        for (int t = 0; t < C && le == cudaSuccess; ++t) {
            for (int l = 0; l < n_layers && le == cudaSuccess; ++l) {
                const dl_handle *h = layers[l];
                const bool last = t == C - 1;
                const bool fold = last && h->cfg.auto_merge == DL_MERGE_FOLD;
                le = launch_append(h, io[(size_t)t * n_layers + l], t, fold, st, overlap);
                if (h->NH > 0) cy->kernels += 1;
                if (le == cudaSuccess && last && h->cfg.auto_merge == DL_MERGE_SEPARATE) {
                    le = launch_merge(h, h->base, C, st);
                    if (h->NH > 0) cy->kernels += 1;
                }
            }
        }
        cudaGraph_t g = nullptr;
        e = cudaStreamEndCapture(st, &g);
        cy->graph = g;
    }
    if (e == cudaSuccess && le != cudaSuccess) e = le;
    if (e == cudaSuccess) e = cudaGraphInstantiate(&cy->exec, cy->graph, 0);
    cudaStreamDestroy(st);
    if (e != cudaSuccess) {
        if (cy->graph) cudaGraphDestroy(cy->graph);
        delete cy;
        return cuda_fail(e, "merge-cycle graph capture");
    }
    *out = cy;
    return ok();
}

dl_status dl_cycle_launch(dl_cycle *cy, void *stream) {
    if (!cy) return fail(DL_EINVAL, "cycle is NULL");
    for (size_t l = 0; l < cy->layers.size(); ++l)
        if (cy->layers[l]->L != 0)
            return fail(DL_ESTATE, "layer %zu has L = %d, a cycle starts at L = 0", l, cy->layers[l]->L);
    cudaError_t e = cudaGraphLaunch(cy->exec, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "merge-cycle graph launch");
    return ok();
}

int dl_cycle_kernels(const dl_cycle *cy) { return cy ? cy->kernels : -1; }

void dl_cycle_destroy(dl_cycle *cy) {
    if (!cy) return;
    if (cy->exec) cudaGraphExecDestroy(cy->exec);
    if (cy->graph) cudaGraphDestroy(cy->graph);
    delete cy;
}

const char *dl_strerror(dl_status s) {
    switch (s) {
        case DL_OK: return "ok";
        case DL_EINVAL: return "invalid argument";
        case DL_ESTATE: return "call not allowed in the current log state";
        case DL_ECUDA: return "CUDA error";
        case DL_ENOMEM: return "out of host memory";
    }
    return "unknown status";
}

const char *dl_last_error(void) { return g_err; }

}  // extern "C"
