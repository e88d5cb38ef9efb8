/*
 * deltalog.h -- C ABI of libdeltalog.so: DeltaLog recurrent-state decode for
 * linear-attention layers (Gated DeltaNet, KDA, RWKV6) on B200 (sm_100a).
 *
 * Method: "DeltaLog: Deferred Materialization of Recurrent States for Linear
 * Attention Decoding" (arXiv 2608.15533).  Each head keeps a dense fp32 base
 * state Sbar (d_k x d_v) plus a bounded log of at most C compact update
 * factors; most decode steps read the base once and append one factor to the
 * log, and a merge folds the log back into the base when it holds C entries
 * (signal-papers page, Fig. 4 caption; gist.science technical summary,
 * "Meccanismo Core: Base + Log" and "Implementazione del Kernel").
 *
 * Recurrences (per head; S is d_k x d_v, row i = key channel):
 *   GDN   a = exp(g) scalar;  S' = a S;     u = beta (v - S'^T k);  S = S' + k u^T;  o = scale S^T q
 *   KDA   a = exp(g) per key; S' = D(a) S;  same delta rule and readout
 *   RWKV6 w = exp(g) per key; o = scale (S^T r + (r . (bonus * k)) v);  S = D(w) S + k v^T
 * DeltaLog keeps, after t appends since the last merge,
 *   S_t = D(exp(Lambda_t)) Sbar + sum_{j<=t} D(exp(Lambda_t - Lambda_j)) k_j u_j^T
 * with Lambda_t the cumulative log-decay since the merge (inclusive of step t)
 * and u_j the value-side factor (the delta-rule u, or the raw v for RWKV6).
 *
 * Conventions for every call below
 *   - Device pointers are CUDA device (or managed) memory owned by the
 *     caller; the library never allocates, frees or keeps device memory, and
 *     every buffer must outlive the calls (and handles) that use it.
 *   - Tensors are dense, row-major, with no padding.  With NH = B * H heads,
 *     head n = b * H + h:
 *       base / S / S_out  float  [NH, d_k, d_v]          16-byte aligned
 *       q (r), k          in_dtype [NH, d_k]             16-byte aligned
 *       v                 in_dtype [NH, d_v]             16-byte aligned
 *       beta              float  [NH]   (GDN, KDA; ignored for RWKV6)  4-byte aligned
 *       g (log-decay)     float  [NH] (GDN, 4-byte aligned) or [NH, d_k]
 *                         (KDA, RWKV6, 16-byte aligned), g <= 0
 *       bonus             float  [H, d_k]  (RWKV6 only, 16-byte aligned;
 *                         ignored otherwise)
 *       out               out_dtype [NH, d_v]            element aligned
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on that stream: no host synchronisation, no
 *     device allocation; the kernel launches can be captured in a CUDA graph.
 *   - Arguments are checked on the host before anything is launched; on an
 *     error nothing is launched and the handle is left as it was (except
 *     where stated).  dl_last_error() gives a message for the calling thread.
 *   - Supported shapes: d_k, d_v in {64, 128}; 1 <= C <= 16; B >= 0, H >= 1.
 *     B = 0 (no heads) is accepted: nothing is launched, the log-length
 *     schedule still advances.
 */
#ifndef DELTALOG_H
#define DELTALOG_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DL_OK = 0,
    DL_EINVAL = 1,   /* bad configuration, shape, pointer or alignment      */
    DL_ESTATE = 2,   /* call not allowed in the current log state            */
    DL_ECUDA = 3,    /* a CUDA runtime call or kernel launch failed          */
    DL_ENOMEM = 4    /* host allocation failed                               */
} dl_status;

typedef enum { DL_GDN = 0, DL_KDA = 1, DL_RWKV6 = 2 } dl_op;
typedef enum { DL_F32 = 0, DL_BF16 = 1 } dl_dtype;

/* When the log is folded into the base (dl_config.auto_merge).  Both
 * automatic modes give the same outputs, states and log-length schedule:
 * L after a step is (steps since the last merge) mod C. */
typedef enum {
    DL_MERGE_OFF = 0,      /* never: a step with L = C fails (DL_ESTATE)      */
    DL_MERGE_FOLD = 1,     /* the C-th token is a merge-token: one kernel
                              reads the base once, replays the C-1 logged
                              factors and writes the merged state, this
                              token's update included (default)              */
    DL_MERGE_SEPARATE = 2  /* the C-th token appends, then the merge kernel
                              folds the full log into the base                */
} dl_merge_mode;

typedef struct {
    int op;          /* dl_op                                                  */
    int B, H;        /* batch slots and heads per slot                         */
    int dk, dv;      /* key and value width of one head's state                */
    int C;           /* log capacity = merge interval                          */
    int in_dtype;    /* dl_dtype of q (r), k, v and of the logged k (and v)   */
    int out_dtype;   /* dl_dtype of out                                        */
    float scale;     /* output scale (d_k^-1/2 for GDN/KDA is usual)           */
    int auto_merge;  /* dl_merge_mode                                          */
} dl_config;

typedef struct dl_handle dl_handle;   /* opaque; host memory only */

/* Size in bytes of the log workspace for `cfg` (0 if cfg is invalid).
 * Layout, each region 256-byte aligned, in this order:
 *   K      in_dtype [NH, C, d_k]   logged keys (bit-exact copies of k)
 *   U      [NH, C, d_v]            value factors: float (GDN, KDA), or
 *                                  in_dtype copies of v (RWKV6)
 *   Lambda float [NH, C, m]        cumulative log-decay since the last merge,
 *                                  m = 1 (GDN) or d_k (KDA, RWKV6)
 * The log is the paper's bounded log of compact update factors
 * (gist.science technical summary, "Meccanismo Core: Base + Log"). */
size_t dl_log_bytes(const dl_config *cfg);

/* Byte offsets of the K, U and Lambda regions inside the log workspace. */
dl_status dl_log_layout(const dl_config *cfg, size_t *off_K, size_t *off_U,
                        size_t *off_Lam);

/* Create a decode handle over a caller-owned base state (device, fp32
 * [NH, d_k, d_v], 16-byte aligned, holds S at the last merge) and log
 * workspace (device, dl_log_bytes(cfg) bytes, 16-byte aligned).  `bonus` is
 * the RWKV6 bonus [H, d_k] (device, float, 16-byte aligned; ignored for the
 * other operators).  The pair (base, log) is the paper's representation of
 * the recurrent state: a dense base holding the history up to the last merge
 * and a bounded buffer of compact update factors with their log-decay
 * metadata (gist.science technical summary, "Meccanismo Core: Base + Log";
 * signal-papers page, Fig. 4 caption).  The log starts empty (L = 0), as
 * right after a merge; its contents are never read before written.  Any
 * dense state can serve as the base, e.g. one a prefill produced.
 * Host-side only: nothing is launched or allocated on the device; the handle
 * (host memory) belongs to the caller until dl_destroy.
 * Errors: DL_EINVAL (config, NULL or misaligned pointer), DL_ENOMEM. */
dl_status dl_create(const dl_config *cfg, float *base, void *log_ws,
                    const float *bonus, dl_handle **out);

/* One decode token for all NH heads: the append + read-out step (paper:
 * "Fase di Append", kernel stages ReplayPrep and AppendDecode, gist.science
 * technical summary).  Reads the base once, replays the L logged factors,
 * writes `out` (out_dtype [NH, d_v]) and appends (k, u, Lambda) at slot L;
 * the base is not written.  Then L = L + 1.  The token that brings L to C
 * merges: with DL_MERGE_FOLD it is the merge-token (the merged state,
 * this token included, is written over the base by the same kernel), with
 * DL_MERGE_SEPARATE the merge kernel runs after its append; either way L
 * returns to 0.
 * Errors: DL_EINVAL (NULL / misaligned pointer; nothing launched),
 * DL_ESTATE (L = C: the log is full with DL_MERGE_OFF, or a separate merge
 * failed to launch earlier; nothing launched -- call dl_merge), DL_ECUDA (a
 * launch failed: L is unchanged if the append or merge-token kernel did not
 * launch; L = C if the append launched but the separate merge did not). */
dl_status dl_decode_step(dl_handle *h, const void *q, const void *k, const void *v,
                         const float *beta, const float *g, void *out, void *stream);

/* Merge phase (paper: "Fase di Merge", gist.science technical summary;
 * signal-papers page, Fig. 4 caption): Sbar <- D(exp(Lambda_L)) Sbar +
 * sum_j D(exp(Lambda_L - Lambda_j)) k_j u_j^T in place, then L = 0 (every
 * slot at its own length L_b; slots at 0 are left as they are).
 * A no-op when L = 0.  Errors: DL_ECUDA (the slots whose merge launched are
 * at 0, the others keep their lengths). */
dl_status dl_merge(dl_handle *h, void *stream);

/* Write the logical state (base + replayed log) to S_out (device fp32
 * [NH, d_k, d_v], 16-byte aligned, must not overlap the base); base and log
 * are left untouched.  With L = 0 this copies the base.  This is the
 * merge's materialisation of the accumulated logical state (gist.science
 * technical summary, "Fase di Merge") written out of place -- the state
 * whose error the paper reports (signal-papers page, Fig. 12(b),
 * materialized recurrent-state relative error); use it for checks and
 * checkpoints.  Errors: DL_EINVAL, DL_ECUDA. */
dl_status dl_materialize(const dl_handle *h, float *S_out, void *stream);

/* Eager dense step (the in-house dense baseline; paper: eager decoding that
 * materialises and writes back the full state every token, signal-papers
 * page Fig. 3/4 captions): reads and rewrites S (device fp32
 * [NH, d_k, d_v]) and writes out.  cfg->C and cfg->auto_merge are ignored.
 * Errors: DL_EINVAL, DL_ECUDA. */
dl_status dl_eager_step(const dl_config *cfg, float *S, const void *q, const void *k,
                        const void *v, const float *beta, const float *g,
                        const float *bonus, void *out, void *stream);

/* The log length L (0 <= L <= C) every slot has, -2 when the slots'
 * lengths differ (see dl_slot_len), or -1 for a NULL handle.  L is the
 * count in the paper's schedule (signal-papers page, Fig. 4 caption: append
 * while L < C, materialise into the base when L = C); with an automatic
 * merge mode it is (tokens since the last merge) mod C between calls. */
int dl_log_len(const dl_handle *h);

/* --------------------------------------------- per-slot log lengths ---- */
/* Continuous batching: every slot b (batch row, heads b*H .. b*H + H-1)
 * keeps its own log length L_b, so sequences can join, leave and idle
 * independently and each slot merges when its own log is full.  The log of
 * a (slot, head) pair is the paper's per-slot-head unit (gist.science
 * technical summary, "Implementazione del Kernel": ReplayPrep coefficients
 * are computed once per slot-head).  All slots start at L_b = 0; while every
 * slot has the same length and every slot decodes, nothing differs from
 * the shared-length calls above.  dl_merge folds every slot's log (each at
 * its own length); dl_materialize writes every slot's logical state. */

/* One decode token for the slots with active[b] != 0 (`active`: host array
 * of B bytes, read during the call; NULL = every slot).  Each active slot
 * takes the step dl_decode_step describes at its own length L_b; idle
 * slots' base, log and output rows are not touched and L_b does not move.
 * A step launches at most one append kernel (the slots below their last
 * entry), one merge-token kernel (DL_MERGE_FOLD: the slots at L_b = C-1)
 * and one merge kernel (DL_MERGE_SEPARATE: the slots that reach C), each
 * over just its slots (split into launches of at most 512 slots).
 * Errors: as dl_decode_step; DL_ESTATE if an active slot's log is full
 * (nothing launched, no length moves); DL_EINVAL if the step needs per-slot
 * lengths and B > 65536 (slot lists carry 16-bit ids).  After DL_ECUDA each
 * slot's length tells what happened to it: a slot whose kernel launched has
 * taken the step (L_b + 1, or 0 after its merge-token; with
 * DL_MERGE_SEPARATE L_b = C until its merge launched), the others kept
 * their lengths.  Retrying the step for every slot would apply the token
 * twice to the slots that took it: compare dl_slot_len before retrying. */
dl_status dl_decode_step_masked(dl_handle *h, const unsigned char *active, const void *q,
                                const void *k, const void *v, const float *beta,
                                const float *g, void *out, void *stream);

/* Slot `slot` begins a new sequence: L_slot = 0, so its logged entries are
 * dropped.  The slot's base rows ([H, d_k, d_v] at head slot*H) are the
 * caller's to fill with the sequence's starting state (zeros, or the state
 * a prefill produced) before the next call that reads them.  Host-side
 * only: nothing is launched.  Errors: DL_EINVAL (NULL handle, bad slot, or
 * B > 65536 while the slot's log is not empty). */
dl_status dl_slot_reset(dl_handle *h, int slot);

/* Log length of one slot, or -1 for a NULL handle or a slot out of range. */
int dl_slot_len(const dl_handle *h, int slot);

/* Release the handle (host memory only).  NULL is accepted.  The base and
 * log workspace -- the state of "Meccanismo Core: Base + Log" (gist.science
 * technical summary) -- stay the caller's and are not touched; work already
 * queued on a stream keeps using them.  The pages define no release call;
 * this ends the host-side bookkeeping of that state. */
void dl_destroy(dl_handle *h);

/* ------------------------------------------------------- merge cycle ---- */
/* One merge cycle of several layers as a single CUDA graph (paper: the
 * split-replay ablation replays its kernels from a CUDA graph and amortises
 * latencies over one merge cycle, signal-papers page Fig. 9 caption).  The graph holds, token
 * by token, every layer's step; the C-th token of a layer is its
 * merge-token (DL_MERGE_FOLD: n_layers * C kernels) or its append followed
 * by its merge (DL_MERGE_SEPARATE: n_layers * (C + 1) kernels).
 *
 * `io` is [C][n_layers] (token-major): the device pointers of each
 * (token, layer) step, laid out as for dl_decode_step.  All layers must have
 * the same C and an automatic merge mode.  The cycle decodes C tokens for
 * every slot starting from the log lengths the layers have at creation
 * (usually L = 0; with per-slot lengths, every step holds one launch per
 * kind of step its slots take), after which every length is back where it
 * started: a launch requires the layers to be in that state.  The graph
 * captures the pointers: new inputs are written into the same buffers
 * between launches. */
typedef struct {
    const void *q, *k, *v;
    const float *beta, *g;
    void *out;
} dl_step_io;

typedef struct dl_cycle dl_cycle;

/* Errors: DL_EINVAL (mixed C, DL_MERGE_OFF, bad pointer), DL_ECUDA, DL_ENOMEM. */
dl_status dl_cycle_create(dl_handle *const *layers, int n_layers, const dl_step_io *io,
                          dl_cycle **out);
/* Launch one cycle on `stream`.  DL_ESTATE if any layer's log lengths are
 * not those the cycle was created at. */
dl_status dl_cycle_launch(dl_cycle *cy, void *stream);
/* Kernels in one launch of the cycle. */
int dl_cycle_kernels(const dl_cycle *cy);
void dl_cycle_destroy(dl_cycle *cy);

/* ------------------------------------------------------------ errors ---- */
/* Name of a status code.  The pages describe no API, so no passage defines
 * the codes themselves; DL_ESTATE is the one state their schedule forbids
 * (a step when the log already holds C entries, signal-papers page, Fig. 4
 * caption).  Never NULL. */
const char *dl_strerror(dl_status s);
/* Detail of the last error on the calling thread ("" if none). */
const char *dl_last_error(void);

/* ---------------------------------------------------------- testing ---- */
/* Failure injection for tests of the log-length bookkeeping on machines
 * with or without a GPU (no passage of the paper corresponds: this checks
 * the error semantics above).  n_ok >= 0: from now on no kernel is issued
 * at all -- the next n_ok launches are reported as launched (nothing is
 * computed, no memory is touched) and every later one as failed
 * (DL_ECUDA).  n_ok < 0 (the initial state): launches are issued normally.
 * Process-wide; not for use outside tests. */
void dl_debug_fake_launches(long long n_ok);

#ifdef __cplusplus
}
#endif
#endif /* DELTALOG_H */
