/*
 * moe_decode.h -- C ABI of libmoe_decode.so: the decode-time Mixture-of-
 * Experts layer with batch-aware expert re-routing, for one NVIDIA B200
 * (sm_100a).
 *
 * The layer (one call per MoE layer per decode step):
 *   1. router: logits = x Wg^T + bias, softmax, top-k
 *      ("Router Caching and Optimization", section "Analyzing Router
 *      Inference Cost", steps 1-3);
 *   2. batch-aware re-selection, which shrinks the set of experts the batch
 *      activates: OEA piggybacking ("Opportunistic Expert Activation:
 *      Batch-Aware Expert Routing for Faster Decode Without Retraining",
 *      abstract), XShare greedy selection under an expert budget, flat or
 *      per request first ("XShare: Collaborative in-Batch Expert Sharing for
 *      Faster MoE Inference", abstract), or Lynx affinity binning ("Lynx:
 *      Enabling Efficient MoE Inference through Dynamic Batch-Aware Expert
 *      Selection", section 2.2);
 *   3. the SwiGLU FFN of every activated expert over its tokens, combined
 *      with the renormalised gate weights; each activated expert's weights
 *      are read from HBM once per call ("Lynx: Enabling Efficient MoE
 *      Inference through Dynamic Batch-Aware Expert Selection", section 1:
 *      decode latency follows the number of distinct activated experts).
 *
 * Conventions for every entry point
 *  - Pointers named "device" are CUDA device pointers of the current
 *    device; the caller allocates and frees every buffer.  The library never
 *    allocates or frees device memory and keeps no device state between
 *    calls other than what lives in the caller's workspace (and, for
 *    moe_expert_ffn_noalloc, its static scratch array).
 *  - All layouts are dense row-major (C order).  bf16 values are passed as
 *    their uint16_t bit patterns.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and runs asynchronously; no entry point synchronises except
 *    moe_check_error.
 *  - Arguments are validated on the host before anything is enqueued.  On
 *    any error nothing is launched and the status says why.
 *  - Device buffers must be 16-byte aligned, the workspace 256-byte aligned
 *    (MOE_ERR_MISALIGNED otherwise).  The workspace must be zero-filled
 *    once before its first use (e.g. cudaMemset); the library keeps it
 *    consistent afterwards (each call leaves its counters at zero).  After
 *    a CUDA error, or a device error reported by moe_check_error, zero it
 *    again before reusing it.  Calls that share one workspace must not
 *    overlap in time on the device (same stream, or ordered by events).
 *  - Limits: 1 <= B <= 256, 1 <= k <= 16, k <= E <= 256, d % 64 == 0,
 *    64 <= d <= 16384, d_ff % 64 == 0, 64 <= d_ff <= 8192.  moe_route reads
 *    B, d, E, k of the dims (d_ff is ignored); moe_reselect reads B, E, k.
 *  - Inputs must be finite; NaN or Inf inputs give unspecified results.
 *  - Nothing is thrown across the ABI.
 */
#ifndef MOE_DECODE_H
#define MOE_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad dimension or rule parameter */
    MOE_ERR_MISALIGNED = 2,   /* a buffer is not 16-byte aligned */
    MOE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than moe_workspace_bytes() */
    MOE_ERR_UNSUPPORTED = 4,  /* valid but outside the implemented limits, or no sm_100 device */
    MOE_ERR_CUDA = 5,         /* a CUDA runtime/driver call or a launch failed */
    MOE_ERR_INTERNAL = 6      /* a kernel recorded an internal error (see moe_check_error) */
} moe_status_t;

/* Re-selection rules. */
typedef enum {
    MOE_RESELECT_NONE = 0,    /* standard top-k routing */
    MOE_RESELECT_OEA = 1,     /* keep top-k0, fill from the batch union of kept sets */
    MOE_RESELECT_XSHARE = 2,  /* budgeted greedy batch selection, then top-k within it */
    MOE_RESELECT_AFFINITY = 3, /* Lynx affinity binning: confidence bins, critical set, remap */
    MOE_RESELECT_XSHARE_HIER = 4 /* XShare per request, then under the batch budget */
} moe_reselect_mode_t;

/* Layer dimensions: B tokens, hidden size d, E experts, top-k k,
 * expert intermediate size d_ff. */
typedef struct {
    int32_t B, d, E, k, d_ff;
} moe_dims_t;

/* Re-selection rule: mode (moe_reselect_mode_t); k0 (OEA: 1 <= k0 <= k);
 * budget (both XShare rules: k <= budget <= E); group (hierarchical XShare:
 * tokens per request, 1 <= group <= 256).  Unused fields are ignored.
 *
 * MOE_RESELECT_AFFINITY ("Lynx: Enabling Efficient MoE Inference through
 * Dynamic Batch-Aware Expert Selection", sections 2.1-2.2; the page gives
 * no formulas, this is the library's reading): a token's confidence c is
 * the gap between the probabilities of its two top-ranked experts; bins
 * have width k/E and there are min(32, ceil(E/k)) of them (bin = the
 * largest j with j*k <= c*E in fp32); each expert scores the sum of 2^bin
 * over the tokens whose top-k holds it; the critical set is the shortest
 * prefix of the score order (descending, ties to the lower index), at
 * least k long, that holds every token's top-ranked expert; every token
 * keeps exactly k experts, its first k inside the critical set.
 *
 * MOE_RESELECT_XSHARE_HIER ("XShare: Collaborative in-Batch Expert Sharing
 * for Faster MoE Inference", abstract: hierarchical, correlation-aware
 * selection for speculative decoding; the page gives no formulas, this is
 * the library's reading): a request is a run of `group` consecutive tokens
 * (a request's token and its drafts; the last run may be shorter).  Each
 * request picks the k experts with the largest request score (its tokens'
 * top-k gate probabilities summed, tokens ascending, fp32); an expert's
 * batch score sums the request scores of the requests that picked it
 * (requests ascending); the min(budget, |picked|) picked experts with the
 * largest batch scores (ties to the lower index) form the batch set, and
 * each token takes its k highest-ranked experts inside it.  group = 1 is
 * MOE_RESELECT_XSHARE. */
typedef struct {
    int32_t mode, k0, budget, group;
} moe_reselect_t;

/* Per-expert token lists (all device pointers, int32 / fp32):
 *   n_active[1]   number of activated experts;
 *   active[E]     activated expert ids, ascending; -1 past n_active;
 *   offsets[E+1]  offsets[i] = first entry of active[i]; offsets[n_active]
 *                 and every later entry = total (token, expert) pairs;
 *   tok[B*k]      token of each entry; entries of one expert in ascending
 *                 token order; -1 past the total;
 *   w[B*k]        renormalised gate weight of each entry; 0 past the total. */
typedef struct {
    int32_t *n_active;
    int32_t *active;
    int32_t *offsets;
    int32_t *tok;
    float *w;
} moe_lists_t;

/* Bytes of device workspace every entry point below may use for `dims`
 * (one size serves all of them).  Returns 0 if dims are invalid. */
size_t moe_workspace_bytes(moe_dims_t dims);

/* Router ("Router Caching and Optimization", "Analyzing Router Inference
 * Cost", steps 1-3, computed in one pass per token as its "Kernel Fusion"
 * section suggests).
 *   x[B][d] fp32, Wg[E][d] fp32, bias[E] fp32 (device; bias may be NULL);
 *   outputs (device): logits[B][E], probs[B][E] fp32, topk_idx[B][k] int32,
 *   topk_w[B][k] fp32.
 * logits[b][e] = dot(x[b], Wg[e]) + bias[e] in fp32 with a fixed summation
 * order; probs = softmax(logits) with the library's own exp; topk_idx = the
 * k largest logits, descending, equal logits to the lower expert index;
 * topk_w = probs of those experts renormalised to sum 1.  Bit-reproducible
 * (identical results for identical inputs on every call). */
moe_status_t moe_route(const float *x, const float *Wg, const float *bias,
                       moe_dims_t dims, float *logits, float *probs,
                       int32_t *topk_idx, float *topk_w, void *stream);

/* Batch-aware re-selection + per-expert token lists.
 * The rules follow "Opportunistic Expert Activation: Batch-Aware Expert
 * Routing for Faster Decode Without Retraining" (abstract: a token keeps
 * its most important experts and reuses experts the batch already loads),
 * "XShare: Collaborative in-Batch Expert Sharing for Faster MoE Inference"
 * (abstract: batch selection as a modular objective solved greedily, and
 * its hierarchical form for speculative decoding) and "Lynx: Enabling
 * Efficient MoE Inference through Dynamic Batch-Aware Expert Selection"
 * (sections 2.1-2.2: confidence bins, critical experts, remapping); the
 * pages give no formulas, so the precise rules below are this library's
 * reading.  The lists are the expert-major dispatch the Lynx page's
 * remapper hands to the experts (section 2.3).
 *   logits[B][E], probs[B][E] fp32 (device; as produced by moe_route);
 *   outputs (device): sel_idx[B][k] int32 (chosen experts in rank order,
 *   -1 in unused slots), sel_w[B][k] fp32 (gate weights renormalised over
 *   the chosen set, 0 in unused slots), and `lists`.
 * Rules (rank order = logit descending, ties to the lower index):
 *   NONE   : the token's top-k.
 *   OEA    : the token keeps its first k0 experts; the union of all kept
 *            sets is formed; each token then fills up to k slots with the
 *            highest-ranked experts of that union it does not yet hold
 *            (fewer when the union is short).  Activated set = the union.
 *   XSHARE : score s_e = sum over tokens whose top-k holds e of p[b][e]
 *            (fp32, tokens ascending); the min(budget, |union of top-k|)
 *            experts of that union with the largest scores (ties to the
 *            lower index) form the batch set -- the greedy, exact for this
 *            modular objective; each token takes its k highest-ranked
 *            experts inside the set.
 *   AFFINITY, XSHARE_HIER : as described at moe_reselect_t.
 * Results are bit-exact and deterministic.  Needs no workspace. */
moe_status_t moe_reselect(const float *logits, const float *probs,
                          moe_dims_t dims, moe_reselect_t rule,
                          int32_t *sel_idx, float *sel_w, moe_lists_t lists,
                          void *stream);

/* Grouped SwiGLU expert FFN with the weighted combine: every activated
 * expert's weights are streamed from HBM once per call, which is what decode
 * latency follows ("Lynx: Enabling Efficient MoE Inference through Dynamic
 * Batch-Aware Expert Selection", section 1; "Opportunistic Expert
 * Activation: Batch-Aware Expert Routing for Faster Decode Without
 * Retraining", abstract: decode is memory-bound and its MoE latency grows
 * with the number of activated experts).  SwiGLU is the expert type of the
 * Qwen3 MoE models the OEA page evaluates; the pages do not restate it.
 *   x[B][d] fp32; Wgate[E][d_ff][d], Wup[E][d_ff][d], Wdown[E][d][d_ff]
 *   bf16 bits (device; nn.Linear out x in layout); lists as written by
 *   moe_reselect (device, read only);
 *   y[B][d] fp32 (device, overwritten):
 *   y[t] = sum over (t, e, w) entries of w * Wdown[e] (silu(Wgate[e] x_t)
 *          * (Wup[e] x_t)).
 * Only the experts in `lists` are read, each once per call.  x and the
 * SwiGLU activations are rounded to bf16 for the tensor cores; sums are
 * fp32; the combine uses fp32 atomics (summation order not fixed).
 * ws: device workspace of at least moe_workspace_bytes(dims) bytes. */
moe_status_t moe_expert_ffn(const float *x, const uint16_t *Wgate,
                            const uint16_t *Wup, const uint16_t *Wdown,
                            moe_dims_t dims, moe_lists_t lists, float *y,
                            void *ws, size_t ws_bytes, void *stream);

/* The whole layer: moe_route -> moe_reselect -> moe_expert_ffn, chained on
 * the device with no host round trip (the activated-expert count never
 * leaves the GPU): the re-routing step sits between the router and the
 * experts and intercepts the router's output ("Lynx: Enabling Efficient MoE
 * Inference through Dynamic Batch-Aware Expert Selection", section 2.2).
 * Up to 64 tokens the call is one persistent kernel (router, a grid-wide
 * barrier, selection and expert stream); above, four kernels chained with
 * programmatic dependent launch.  Arguments as above; y[B][d] is
 * overwritten.
 * sel_idx[B][k], sel_w[B][k] and n_active[1] are optional device outputs
 * (NULL = not returned).  ws: device workspace of at least
 * moe_workspace_bytes(dims) bytes. */
moe_status_t moe_layer_decode(const float *x, const float *Wg, const float *bias,
                              const uint16_t *Wgate, const uint16_t *Wup,
                              const uint16_t *Wdown, moe_dims_t dims,
                              moe_reselect_t rule, float *y, int32_t *sel_idx,
                              float *sel_w, int32_t *n_active, void *ws,
                              size_t ws_bytes, void *stream);

/* One MoE layer's weights for moe_decode_stack (device pointers, layouts as
 * for moe_layer_decode; bias may be NULL). */
typedef struct {
    const float *Wg;
    const float *bias;
    const uint16_t *Wgate;
    const uint16_t *Wup;
    const uint16_t *Wdown;
} moe_layer_weights_t;

/* Phase of a stack call.  Re-selection pays only in decode, where the layer
 * is bound by memory bandwidth; prefill is compute-bound and sensitive to
 * which experts a token gets, so a phase-aware caller bypasses re-routing
 * there ("Lynx: Enabling Efficient MoE Inference through Dynamic
 * Batch-Aware Expert Selection", section 2.1 "Phase Sensitivity" and
 * section 2.2 "Phase-Aware Optimizer"). */
typedef enum {
    MOE_PHASE_DECODE = 0,   /* apply the given re-selection rule */
    MOE_PHASE_PREFILL = 1   /* prefill or chunked prefill: standard top-k (MOE_RESELECT_NONE) */
} moe_phase_t;

#define MOE_STACK_MAX_LAYERS 1024

/* n_layers MoE layers back to back on a residual stream:
 *   xs[l + 1] = xs[l] + layer_l(xs[l]),   l = 0 .. n_layers - 1,
 * each layer_l as moe_layer_decode with layers[l]'s weights and the same
 * dims and rule (the attention blocks between MoE layers are not part of
 * this library).  Consecutive layers are chained on the device with no host
 * round trip: layer l + 1 is launched with programmatic dependent launch,
 * so its CTAs start, and stage layer l + 1's router weights, while layer
 * l's last CTAs still stream experts; its router reads xs[l + 1] once layer
 * l has completed ("Router Caching and Optimization", "Scheduling Router
 * Computation": router computation for a layer partially overlapped with
 * the previous layer's).
 *   layers: HOST array of n_layers weight sets (1 <= n_layers <=
 *   MOE_STACK_MAX_LAYERS); phase: moe_phase_t (PREFILL replaces `rule` by
 *   standard top-k);
 *   xs[n_layers + 1][B][d] fp32 (device): xs[0] is the input, read only;
 *   xs[1 .. n_layers] are written;
 *   sel_idx[n_layers][B][k] int32, n_active[n_layers] int32: optional
 *   device outputs per layer (NULL = not returned);
 *   ws: one workspace of moe_workspace_bytes(dims) bytes, reused by every
 *   layer.
 * Validation covers every layer before anything is enqueued. */
moe_status_t moe_decode_stack(const moe_layer_weights_t *layers, int32_t n_layers, moe_dims_t dims,
                              moe_reselect_t rule, int32_t phase, float *xs, int32_t *sel_idx,
                              int32_t *n_active, void *ws, size_t ws_bytes, void *stream);

/* ---- Per-token channel top-k inside the activated experts ----------------
 * "Channel Selection for Mixture-of-Experts Decoding Needs No Calibration
 * Data", methodology: a channel selector is a score plus a keep rule; the
 * top-k keep rule takes each token's c highest-scoring channels of an
 * expert; channel f of expert e is gate row f, up row f and down column f,
 * and only the kept channels' weights are read (counted in 32-byte
 * sectors).  The scores come from the caller (any selector).  The down
 * projection is read from a channel-major copy, so that a channel's down
 * weights are one contiguous 2*d-byte row like its gate and up rows. */
#define MOE_CHANNELS_B_MAX 8

/* WdownT[E][d_ff][d] = Wdown[E][d][d_ff] transposed per expert (bf16 bits,
 * device; done once when the weights are loaded).  d, d_ff as for the
 * layer (multiples of 64).  Enqueued on `stream`. */
moe_status_t moe_down_channel_major(const uint16_t *Wdown, moe_dims_t dims, uint16_t *WdownT, void *stream);

/* Device workspace bytes of moe_expert_ffn_channels for dims (0 if the
 * dims are outside its limits: B <= MOE_CHANNELS_B_MAX, 2 * B * d * 4 +
 * 2 * 3 * d * 2 <= 200 KB of shared memory, plus the layer's limits). */
size_t moe_channels_workspace_bytes(moe_dims_t dims);

/* y[b] = sum over slots s with e = sel_idx[b][s] >= 0 of sel_w[b][s] *
 *        sum over the kept channels f of Wdown[e][:, f] silu(g_f) u_f,
 * g_f = Wgate[e][f] . x[b], u_f = Wup[e][f] . x[b], where (b, s) keeps the
 * c channels with the largest score[b][s][f] (equal scores to the lower
 * channel index).
 *   x[B][d] fp32; Wgate, Wup [E][d_ff][d] bf16; WdownT [E][d_ff][d] bf16
 *   (moe_down_channel_major); sel_idx[B][k] int32 (-1 = empty slot) and
 *   sel_w[B][k] fp32, e.g. from moe_reselect; score[B][k][d_ff] fp32;
 *   1 <= c <= d_ff; y[B][d] fp32 (overwritten); keep[B][k][d_ff / 32]
 *   uint32 (optional output, bit f of word f / 32 = channel f kept; NULL =
 *   not returned); ws of moe_channels_workspace_bytes(dims) bytes, 256-byte
 *   aligned, zero-filled once before its first use (its first word is the
 *   error word moe_check_error reads and clears).  Weights are read in fp32 FMAs (no
 *   tensor cores: a handful of tokens share a channel); summation order
 *   within a dot product is fixed per launch shape. */
moe_status_t moe_expert_ffn_channels(const float *x, const uint16_t *Wgate, const uint16_t *Wup,
                                     const uint16_t *WdownT, moe_dims_t dims, const int32_t *sel_idx,
                                     const float *sel_w, const float *score, int32_t c, float *y,
                                     uint32_t *keep, void *ws, size_t ws_bytes, void *stream);

/* moe_expert_ffn for callers that cannot allocate device memory.
 * (The source pages have no counterpart to this entry point; it is a
 * deployment convenience of this library.)
 *
 * Some callers have no workspace to pass and may not call cudaMalloc:
 * plugins whose host framework hands them only inputs and outputs, code
 * running where all device memory was reserved up front by the host
 * application, and latency-critical paths that cannot afford the device
 * synchronisation cudaMalloc/cudaFree may cause.  This entry point takes the
 * same arguments as moe_expert_ffn minus the workspace, and allocates
 * nothing: its scratch (the expert kernel's counters, x in bf16 and the
 * SwiGLU activations) lives in a file-scope static device array of
 * MOE_NOALLOC_SCRATCH_BYTES (32 MiB), which every GPU that loads the library
 * holds until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 *  - Size limit: the scratch must fit in MOE_NOALLOC_SCRATCH_BYTES: when
 *    B <= 64, B*d*2 bytes of bf16 x, min(E, B*k)*B*d_ff*2 bytes of SwiGLU
 *    activations and min(E, B*k)*B*4 bytes of dense weights; above,
 *    B*k*d*2 bytes of per-pair x rows and B*k*d_ff*2 bytes of activations;
 *    plus about 7 KB of counters, each part rounded up to 256 bytes.  Larger
 *    dims return MOE_ERR_UNSUPPORTED before anything is enqueued.  The
 *    Qwen3-30B-A3B- and Qwen3-235B-A22B-shaped layers fit for every B <= 256.
 *  - Set-up: the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make
 *    that first call before any stream capture begins.
 *  - Sharing: all calls on a device use the same array, which keeps the
 *    last call's contents; each call clears the counters that must start at
 *    zero.  Calls that overlap in time on the GPU (for example on two
 *    streams with no ordering between them) race on the array and give
 *    wrong results: order them on one stream or with events.
 *  - A bounded wait that expires inside the kernels is recorded in the
 *    array but not reported; use moe_expert_ffn + moe_check_error to
 *    diagnose such a failure. */
#define MOE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
moe_status_t moe_expert_ffn_noalloc(const float *x, const uint16_t *Wgate,
                                    const uint16_t *Wup, const uint16_t *Wdown,
                                    moe_dims_t dims, moe_lists_t lists, float *y,
                                    void *stream);

/* Limit of every bounded wait inside the library's kernels, for kernels
 * launched after this call (process-wide; 0 restores the default of 1 s).
 * A kernel waits on other CTAs (the fused layer kernel's grid barrier and
 * its flags), on its own copies and on the previous kernel's results; when
 * a wait runs past the limit the CTA records an error code in the
 * workspace (reported by moe_check_error as MOE_ERR_INTERNAL), lets the
 * copies already in flight into its shared memory land (up to a further
 * 1 s), and ends its share of the call, so that the device stays usable.
 * A limit shorter than the work it waits for makes calls fail on purpose
 * (a diagnostic of the error path); the default never expires in normal
 * operation. */
void moe_set_wait_limit_ns(uint64_t ns);

/* Synchronises `stream`, then reads and clears the error word that kernels
 * of earlier calls using this workspace may have set (a bounded wait that
 * ran out, or inconsistent token lists); works for the layer workspace and
 * for the channel path's workspace alike (both start with the word).  Returns MOE_OK, MOE_ERR_INTERNAL or MOE_ERR_CUDA. */
moe_status_t moe_check_error(void *ws, size_t ws_bytes, void *stream);

/* Static description of a status code (never NULL). */
const char *moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DECODE_H */
