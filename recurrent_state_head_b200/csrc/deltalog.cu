// deltalog.cu -- host side of libdeltalog.so: argument checks, the decode
// handle with its log-length schedule (append while L < C, merge when the
// log is full), and the graph-captured merge cycle.
//
// Method: "DeltaLog: Deferred Materialization of Recurrent States for Linear
// Attention Decoding" (arXiv 2608.15533): append / merge phases (gist.science
// technical summary, "Meccanismo Core: Base + Log"; signal-papers page,
// Fig. 4 caption) and CUDA-Graph replay of one merge cycle (Fig. 9 caption).
#include <atomic>
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

namespace {

// Slot ids travel to the kernels as 16-bit list entries.
constexpr int kMaxSlotId = 65535;

// Log lengths of a handle's slots: one shared length while every slot has
// it (the common case), else one length per slot.
struct Lens {
    bool shared = true;
    int L = 0;                          // the shared length
    std::vector<unsigned char> per;     // per-slot lengths when !shared

    int of(int b) const { return shared ? L : per[(size_t)b]; }
    // Expand to per-slot form (B slots).
    void split(int B) {
        if (!shared) return;
        per.assign((size_t)B, (unsigned char)L);
        shared = false;
    }
    // Back to the shared form when every slot has the same length.
    void join() {
        if (shared || per.empty()) return;
        for (unsigned char x : per)
            if (x != per[0]) return;
        L = per[0];
        shared = true;
        per.clear();
    }
    bool operator==(const Lens &o) const {
        if (shared && o.shared) return L == o.L;
        const size_t n = shared ? o.per.size() : per.size();
        for (size_t b = 0; b < n; ++b)
            if (of((int)b) != o.of((int)b)) return false;
        return true;
    }
};

}  // namespace

struct dl_handle {
    dl_config cfg;
    float *base;
    char *log;
    Layout lay;
    const float *bonus;
    Lens lens;
    int NH;
};

struct dl_cycle {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    std::vector<dl_handle *> layers;
    std::vector<Lens> start;            // the layers' lengths the cycle starts (and ends) at
    int kernels;
};

namespace {

// Failure injection for host tests of the length bookkeeping
// (dl_debug_fake_launches): -1 issues every launch; n >= 0 issues none,
// reports the next n as launched and every later one as failed.
std::atomic<long long> g_fake_ok{-1};

template <typename Launch>
cudaError_t issue(Launch &&launch) {
    long long left = g_fake_ok.load(std::memory_order_relaxed);
    while (left >= 0) {
        if (left == 0) return cudaErrorLaunchFailure;
        if (g_fake_ok.compare_exchange_weak(left, left - 1, std::memory_order_relaxed))
            return cudaSuccess;
    }
    return launch();
}

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
    p.H = h->cfg.H;
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
    return issue([&] { return dl::get_append(h->cfg.op, h->cfg.dk, h->cfg.dv)(p, fold, s); });
}

// Do the layers' base states occupy pairwise disjoint memory?  (Layers
// without heads occupy none.)
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
    return issue([&] { return dl::get_merge(h->cfg.op, h->cfg.dk, h->cfg.dv)(merge_params(h, dst, L), s); });
}

// Slot-list launches of at most MAXSEL slots each: `ids` are the slots,
// `lens` their lengths.  merge == false: the append kernel, whose first
// `nfold` entries take the merge-token; merge == true: the merge kernel into
// dst.  *done (if given) receives how many leading entries of `ids` were
// launched, all of them on success.
cudaError_t launch_slots(const dl_handle *h, bool merge, const std::vector<int> &ids,
                         const std::vector<int> &lens, int nfold, const dl_step_io *io, float *dst,
                         cudaStream_t s, bool early, int *kernels, size_t *done = nullptr) {
    if (done) *done = 0;
    if (h->NH == 0) {
        if (done) *done = ids.size();
        return cudaSuccess;
    }
    for (size_t at = 0; at < ids.size(); at += dl::MAXSEL) {
        const size_t n = ids.size() - at < (size_t)dl::MAXSEL ? ids.size() - at : (size_t)dl::MAXSEL;
        dl::SlotList sl;
        sl.n = (int)n;
        const int fold_left = nfold - (int)at;
        sl.nfold = fold_left <= 0 ? 0 : (fold_left < (int)n ? fold_left : (int)n);
        int Lmax = 0;
        for (size_t i = 0; i < n; ++i) {
            sl.id[i] = (unsigned short)ids[at + i];
            sl.L[i] = (unsigned char)lens[at + i];
            if (lens[at + i] > Lmax) Lmax = lens[at + i];
        }
        cudaError_t e;
        if (merge) {
            e = issue([&] {
                return dl::get_merge_slots(h->cfg.op, h->cfg.dk, h->cfg.dv)(merge_params(h, dst, Lmax), sl, s);
            });
        } else {
            dl::AppendParams p = append_params(h, *io, Lmax);
            p.early = early ? 1 : 0;
            e = issue([&] { return dl::get_append_slots(h->cfg.op, h->cfg.dk, h->cfg.dv)(p, sl, s); });
        }
        if (e != cudaSuccess) return e;
        if (kernels) *kernels += 1;
        if (done) *done = at + n;
    }
    return cudaSuccess;
}

// One decode token for the active slots (active == nullptr: all of them),
// launched on `st`, with the lengths in `ln`.  Returns DL_OK, DL_ESTATE
// (nothing launched, nothing moved) or DL_ECUDA.  Every length in `ln` is
// kept true to what was launched: a slot whose kernel launched has taken
// the step (L + 1, or 0 after its merge-token; with DL_MERGE_SEPARATE a
// slot whose log filled stays at C until its merge launches), a slot whose
// kernel did not launch keeps its length.
dl_status decode_step(const dl_handle *h, Lens &ln, const unsigned char *active, const dl_step_io &io,
                      cudaStream_t st, bool early, int *kernels) {
    const int B = h->cfg.B, C = h->cfg.C, mode = h->cfg.auto_merge;
    const char *full_why = mode == DL_MERGE_OFF ? "auto_merge is off: merge first"
                                                : "a merge failed to launch: call dl_merge";
    bool all = true;
    if (active)
        for (int b = 0; b < B && all; ++b) all = active[b] != 0;
    if (ln.shared && all) {
        if (ln.L >= C) return fail(DL_ESTATE, "log is full (L = C = %d); %s", C, full_why);
        if (mode == DL_MERGE_FOLD && ln.L == C - 1) {
            // the token that completes the log: one kernel reads the base once
            // and writes the merged logical state back
            cudaError_t e = launch_append(h, io, ln.L, true, st, early);
            if (e != cudaSuccess) return cuda_fail(e, "merge-token kernel launch");
            if (kernels && h->NH > 0) *kernels += 1;
            ln.L = 0;
            return ok();
        }
        cudaError_t e = launch_append(h, io, ln.L, false, st, early);
        if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
        if (kernels && h->NH > 0) *kernels += 1;
        ln.L += 1;
        if (mode == DL_MERGE_SEPARATE && ln.L == C) {
            e = launch_merge(h, h->base, ln.L, st);
            if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch (the log stays full)");
            if (kernels && h->NH > 0) *kernels += 1;
            ln.L = 0;
        }
        return ok();
    }
    // slots at different lengths, or some idle: one append launch over the
    // active slots, merge-token slots (DL_MERGE_FOLD, log one short of full)
    // first; with DL_MERGE_SEPARATE the slots that fill their log are then
    // merged by the merge kernel
    if (B > kMaxSlotId + 1)
        return fail(DL_EINVAL, "per-slot lengths support at most %d slots (B = %d)", kMaxSlotId + 1, B);
    std::vector<int> ids, lens, idm, lm;
    int nfold = 0;
    for (int pass = 0; pass < 2; ++pass)
        for (int b = 0; b < B; ++b) {
            if (active && !active[b]) continue;
            const int L = ln.of(b);
            if (L >= C) return fail(DL_ESTATE, "slot %d: log is full (L = C = %d); %s", b, C, full_why);
            const bool fold = mode == DL_MERGE_FOLD && L == C - 1;
            if (fold != (pass == 0)) continue;
            ids.push_back(b);
            lens.push_back(L);
            nfold += fold ? 1 : 0;
            if (mode == DL_MERGE_SEPARATE && L + 1 == C) {
                idm.push_back(b);
                lm.push_back(C);
            }
        }
    if (ids.empty()) return ok();
    size_t done = 0, merged = 0;
    cudaError_t e = launch_slots(h, false, ids, lens, nfold, &io, nullptr, st, early, kernels, &done);
    if (e == cudaSuccess) e = launch_slots(h, true, idm, lm, 0, nullptr, h->base, st, false, kernels, &merged);
    ln.split(B);
    for (size_t i = 0; i < done; ++i) {
        const size_t b = (size_t)ids[i];
        const int L = ln.per[b] + 1;
        ln.per[b] = (unsigned char)((mode == DL_MERGE_FOLD && L == C) ? 0 : L);
    }
    for (size_t i = 0; i < merged; ++i) ln.per[(size_t)idm[i]] = 0;
    ln.join();
    if (e != cudaSuccess) return cuda_fail(e, "per-slot kernel launch");
    return ok();
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
    h->NH = NH;
    *out = h;
    return ok();
}

dl_status dl_decode_step_masked(dl_handle *h, const unsigned char *active, const void *q,
                                const void *k, const void *v, const float *beta,
                                const float *g, void *out, void *stream) {
    if (!h) return fail(DL_EINVAL, "handle is NULL");
    if (h->NH > 0) {
        dl_status s = check_step_ptrs(&h->cfg, q, k, v, beta, g, out);
        if (s != DL_OK) return s;
    }
    const dl_step_io io = {q, k, v, beta, g, out};
    return decode_step(h, h->lens, active, io, static_cast<cudaStream_t>(stream), false, nullptr);
}

dl_status dl_decode_step(dl_handle *h, const void *q, const void *k, const void *v,
                         const float *beta, const float *g, void *out, void *stream) {
    return dl_decode_step_masked(h, nullptr, q, k, v, beta, g, out, stream);
}

dl_status dl_merge(dl_handle *h, void *stream) {
    if (!h) return fail(DL_EINVAL, "handle is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (h->lens.shared) {
        if (h->lens.L == 0) return ok();
        cudaError_t e = launch_merge(h, h->base, h->lens.L, st);
        if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch");
        h->lens.L = 0;
        return ok();
    }
    std::vector<int> ids, lens;
    for (int b = 0; b < h->cfg.B; ++b)
        if (h->lens.of(b) > 0) {
            ids.push_back(b);
            lens.push_back(h->lens.of(b));
        }
    size_t done = 0;
    cudaError_t e = launch_slots(h, true, ids, lens, 0, nullptr, h->base, st, false, nullptr, &done);
    for (size_t i = 0; i < done; ++i) h->lens.per[(size_t)ids[i]] = 0;   // merged slots
    h->lens.join();
    if (e != cudaSuccess) return cuda_fail(e, "merge kernel launch");
    return ok();
}

dl_status dl_materialize(const dl_handle *h, float *S_out, void *stream) {
    if (!h) return fail(DL_EINVAL, "handle is NULL");
    if (h->NH == 0) return ok();
    if (!S_out || !aligned(S_out, 16)) return fail(DL_EINVAL, "S_out must be non-NULL and 16-byte aligned");
    const size_t bytes = (size_t)h->NH * h->cfg.dk * h->cfg.dv * 4;
    const char *a = reinterpret_cast<const char *>(S_out), *b = reinterpret_cast<const char *>(h->base);
    if (a < b + bytes && b < a + bytes) return fail(DL_EINVAL, "S_out overlaps the base state");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (h->lens.shared) {
        e = launch_merge(h, S_out, h->lens.L, st);
    } else {
        std::vector<int> ids, lens;
        for (int b = 0; b < h->cfg.B; ++b) {
            ids.push_back(b);
            lens.push_back(h->lens.of(b));
        }
        e = launch_slots(h, true, ids, lens, 0, nullptr, S_out, st, false, nullptr);
    }
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

int dl_log_len(const dl_handle *h) {
    if (!h) return -1;
    return h->lens.shared ? h->lens.L : -2;
}

dl_status dl_slot_reset(dl_handle *h, int slot) {
    if (!h) return fail(DL_EINVAL, "handle is NULL");
    if (slot < 0 || slot >= h->cfg.B) return fail(DL_EINVAL, "slot %d outside [0, %d)", slot, h->cfg.B);
    if (h->lens.of(slot) == 0) return ok();
    if (h->cfg.B > kMaxSlotId + 1)
        return fail(DL_EINVAL, "per-slot lengths support at most %d slots (B = %d)", kMaxSlotId + 1, h->cfg.B);
    h->lens.split(h->cfg.B);
    h->lens.per[(size_t)slot] = 0;
    h->lens.join();
    return ok();
}

int dl_slot_len(const dl_handle *h, int slot) {
    if (!h || slot < 0 || slot >= h->cfg.B) return -1;
    return h->lens.of(slot);
}

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
        for (int l = 0; l < n_layers; ++l) cy->start.push_back(layers[l]->lens);
    } catch (...) {
        delete cy;
        return fail(DL_ENOMEM, "host allocation of the cycle failed");
    }
    // with two or more layers that have heads, on disjoint bases,
    // consecutive kernels of the token-major cycle belong to different
    // layers (a layer's own consecutive kernels -- slot-list chunks, an
    // append and its merge -- touch disjoint heads, or the second one is an
    // ordinary launch): each may start streaming its base during the
    // previous kernel's tail.  A layer without heads launches nothing, so it
    // does not separate two steps of another layer.
    int with_heads = 0;
    for (int l = 0; l < n_layers; ++l) with_heads += layers[l]->NH > 0 ? 1 : 0;
    const bool overlap = with_heads >= 2 && disjoint_bases(layers, n_layers);
    cudaStream_t st = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
        delete cy;
        return cuda_fail(e, "capture stream creation");
    }
    e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
    dl_status ls = DL_OK;
    if (e == cudaSuccess) {
        // token-major: every layer's step for token t, on copies of the
        // layers' lengths (C steps bring every length back where it started);
        // the token that completes a log is its merge-token (DL_MERGE_FOLD)
        // or its append followed by its merge (DL_MERGE_SEPARATE)
        std::vector<Lens> lens(cy->start);
        for (int t = 0; t < C && ls == DL_OK; ++t)
            for (int l = 0; l < n_layers && ls == DL_OK; ++l)
                ls = decode_step(layers[l], lens[(size_t)l], nullptr, io[(size_t)t * n_layers + l], st,
                                 overlap, &cy->kernels);
        cudaGraph_t g = nullptr;
        e = cudaStreamEndCapture(st, &g);
        cy->graph = g;
    }
    if (e == cudaSuccess && ls != DL_OK) {
        if (cy->graph) cudaGraphDestroy(cy->graph);
        cudaStreamDestroy(st);
        delete cy;
        return ls;
    }
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
        if (!(cy->layers[l]->lens == cy->start[l]))
            return fail(DL_ESTATE, "layer %zu's log lengths are not those the cycle starts at", l);
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

void dl_debug_fake_launches(long long n_ok) { g_fake_ok.store(n_ok < 0 ? -1 : n_ok); }

}  // extern "C"
