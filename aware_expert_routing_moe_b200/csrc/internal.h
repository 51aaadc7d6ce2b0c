// Internal declarations shared by the translation units of libmoe_decode.so.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "moe_decode.h"

namespace moe {

constexpr int B_MAX = 256;
constexpr int E_MAX = 256;
constexpr int K_MAX = 16;
constexpr int D_MIN = 64, D_MAX = 16384;
constexpr int F_MIN = 64, F_MAX = 8192;

// Counters the kernels share inside one workspace.  They are zero between
// calls: the last CTA of the expert stream puts them back.
// One published copy of the activated set, alone in a 128-byte line.
struct PubLine {
    int32_t pub;                // 1 once `mask` holds the activated set
    int32_t pad0[3];
    uint32_t mask[E_MAX / 32];  // the activated set, one bit per expert
    int32_t pad1[20];
};
static_assert(sizeof(PubLine) == 128, "PubLine must fill one 128-byte line");
constexpr int MAX_DEVICES = 64;  // per-device host caches (attributes, SM counts)
constexpr int PUB_COPIES = 8;  // expert-kernel CTA c polls copy c % PUB_COPIES

struct Counters {
    int32_t error;     // first error code a kernel recorded (0 = none)
    int32_t k3_exit;   // expert-kernel CTAs finished
    int32_t arrive;    // fused layer kernel: CTAs past the router (grid barrier)
    int32_t lists_ready;  // fused layer kernel: the selection CTA has written the lists
    int32_t pad0[28];
    PubLine pubs[PUB_COPIES];   // fused layer kernel, batch-wide rules: the activated set
    int32_t gu_done[E_MAX];     // finished gate/up units per active-expert slot
};
static_assert(sizeof(Counters) % 16 == 0, "Counters must keep 16-byte alignment");

// Device error codes written into Counters::error.
enum DeviceError : int32_t {
    DEV_OK = 0,
    DEV_TIMEOUT_FULL = 1,   // a consumer waited too long for a pipeline stage
    DEV_TIMEOUT_EMPTY = 2,  // the producer waited too long for a free stage
    DEV_TIMEOUT_DEP = 3,    // a down-projection unit waited too long for gate/up
    DEV_BAD_LISTS = 4,      // lists inconsistent with dims
};

// Byte offsets of the workspace segments (each 256-byte aligned).
struct WsLayout {
    size_t counters, logits, probs, sel_idx, sel_w;
    size_t n_active, active, offsets, tok, w;
    size_t xb, xd, h, wd;
    size_t total;
};

// Activated-expert slots a call can have: min(E, B*k).
inline int active_slots(const moe_dims_t &d) { return d.E < d.B * d.k ? d.E : d.B * d.k; }
// Batches up to this many tokens run the dense mode: every unit takes the
// whole batch (the tokens that did not choose the expert weigh 0).
constexpr int DENSE_B_MAX = 64;
// Bytes of the expert kernel's H scratch: token-indexed [slot][B][d_ff]
// in dense mode (B <= 64), else pair-indexed [B*k][d_ff]; bf16.
inline size_t h_scratch_bytes(const moe_dims_t &d) {
    const size_t F = d.d_ff;
    return d.B <= DENSE_B_MAX ? static_cast<size_t>(active_slots(d)) * d.B * F * 2
                              : static_cast<size_t>(d.B) * d.k * F * 2;
}
// Bytes of the dispatched x rows [B*k][d] bf16 (B > 64 only).
inline size_t xd_bytes(const moe_dims_t &d) {
    return d.B <= DENSE_B_MAX ? 0 : static_cast<size_t>(d.B) * d.k * d.d * 2;
}
// Bytes of the dense weight matrix [slot][B] fp32 (B <= 64 only).
inline size_t wd_bytes(const moe_dims_t &d) {
    return d.B <= DENSE_B_MAX ? static_cast<size_t>(active_slots(d)) * d.B * 4 : 0;
}

WsLayout ws_layout(const moe_dims_t &d);

// TMA descriptors of the router: x [B][d] and Wg [E][d] (fp32) seen as
// columns of 128-byte lines, 128-byte swizzle, boxes of whole rows (at most
// 256 lines).
struct RouterMaps {
    CUtensorMap x, wg;
};
bool encode_router_maps(RouterMaps *m, const moe_dims_t &d, const float *x, const float *Wg);
// Lines per router box for `d` (the box of encode_router_maps).
int router_box_lines(int d);

// Launchers (enqueue only; arguments already validated).
cudaError_t launch_router_logits(const RouterMaps &maps, const float *bias, const moe_dims_t &d, float *logits,
                                 cudaStream_t s);
cudaError_t launch_route_topk(const float *logits, const moe_dims_t &d, float *probs,
                              int32_t *topk_idx, float *topk_w, cudaStream_t s);
cudaError_t launch_reselect(const float *logits, const float *probs, const moe_dims_t &d,
                            const moe_reselect_t &r, int32_t *sel_idx, float *sel_w,
                            const moe_lists_t &l, cudaStream_t s);
// Layer path above 64 tokens, first kernel: router GEMV; also sets y = 0
// (y = x with residual).  chained: launched with programmatic dependent
// launch after the previous layer of a stack.
cudaError_t launch_layer_route(const RouterMaps &maps, const float *x, const float *bias, const moe_dims_t &d,
                               float *logits, float *y, Counters *ctr, bool residual, bool chained, cudaStream_t s);
// Layer path above 64 tokens, second kernel (chained with programmatic
// dependent launch): softmax, selection, lists.
cudaError_t launch_layer_select(const float *logits, float *probs, const moe_dims_t &d, const moe_reselect_t &rule,
                                int32_t *sel_idx, float *sel_w, const moe_lists_t &l, int32_t *n_active_copy,
                                cudaStream_t s);
// Input preparation of the expert kernel (all pointers may be null, each
// step is skipped then): x -> bf16 (xb, dense mode), each pair's x row ->
// xd (larger batches), y = 0, gate/up counts cleared and, for B <= 64, the
// dense weights built from the lists.  chained: launched with programmatic
// dependent launch after the kernel that writes the lists.
cudaError_t launch_ffn_prep(const float *x, const moe_dims_t &d, uint16_t *xb, uint16_t *xd, float *y,
                            Counters *ctr, const moe_lists_t &l, float *wd, bool chained, cudaStream_t s);

// TMA descriptors of the expert kernel: the three weight tensors, the H
// scratch and the bf16 x rows (xb for B <= 64, the dispatched pair rows xd
// above) as (64-column chunk, row, chunk index) boxes.  gu: Wgate and Wup
// as one 4-D tensor whose matrix dimension steps from the lower of the two
// buffers to the higher, so that one box holds a whole gate/up stage in
// the tensor-core stage's layout; gu_mode 0: not used (the warp-MMA
// path) or not encodable (the buffers coincide, or their distance is no
// valid TMA stride), the stage takes per-matrix boxes; 1: Wgate is the
// lower buffer; 2: Wup is (gate and up halves swapped in shared memory).
struct ExpertMaps {
    CUtensorMap gate, up, down, h, x, gu;
    int gu_mode;
};
// The expert kernel alone (moe_expert_ffn): lists from the previous kernel
// (chained with programmatic dependent launch) or the caller; wd: dense
// weights (B <= 64).
cudaError_t launch_expert_ffn(const ExpertMaps &maps, const uint16_t *xb, const moe_dims_t &d,
                              const moe_lists_t &l, float *y, uint16_t *h, const float *wd, Counters *ctr, int wm,
                              cudaStream_t s);
// The whole layer in one cooperative persistent kernel (B <= 64): router,
// grid barrier, selection (last CTA), expert stream (the other CTAs).  xb:
// x in bf16 (written), h: the SwiGLU scratch, wd: the dense weights.
// wm: the warp-MMA expert stream (expert_ffn_warp_mma); residual: y = x +
// the experts' output; chained: launched with programmatic dependent launch
// after the previous layer of a stack.
cudaError_t launch_layer_fused(const ExpertMaps &maps, const RouterMaps &rmaps, const moe_dims_t &d,
                               const moe_reselect_t &rule, const float *x, const float *bias, float *logits,
                               float *probs, uint16_t *xb, float *y, uint16_t *h, float *wd, int32_t *sel_idx,
                               float *sel_w, const moe_lists_t &lists, int32_t *n_active_copy, Counters *ctr,
                               int wm, bool residual, bool chained, cudaStream_t s);
// Per-token channel top-k (channels.cu): workspace bytes, ring stages of the
// stream kernel for d (0: the dims do not fit its shared memory), the
// channel-major copy of Wdown, and the three kernels of one call.
size_t channels_workspace_bytes(const moe_dims_t &d);
int channels_stages(const moe_dims_t &d);
cudaError_t launch_down_transpose(const uint16_t *Wdown, const moe_dims_t &d, uint16_t *WdownT, cudaStream_t s);
cudaError_t launch_channels(const float *x, const uint16_t *Wgate, const uint16_t *Wup, const uint16_t *WdownT,
                            const moe_dims_t &d, const int32_t *sel_idx, const float *sel_w, const float *score,
                            int c, float *y, uint32_t *keep_out, void *ws, cudaStream_t s);
// Limit of every bounded wait inside the kernels launched from now on
// (nanoseconds; moe_set_wait_limit_ns).
unsigned long long wait_limit_ns();
int expert_ffn_h_rows(int B);         // rows of one H box
int expert_ffn_dense_batch(int B);    // 1 if gate/up stages load all B token rows at once
// 1 if the expert stream of a call runs on warp-level MMAs (16-row gate/up
// units): at most 8 tokens and at most 32 activated experts (max_active:
// the most the call's rule can activate)
int expert_ffn_warp_mma(const moe_dims_t &d, int max_active);
int expert_ffn_gu_rows(int wm);       // rows of Wgate / Wup per gate-up unit
int expert_ffn_d_rows();              // rows of Wdown per down unit
int expert_ffn_gu_chunks(int d, int wm);  // 64-column chunks of d per gate-up stage
int expert_ffn_gu_box_chunks(int d, int wm);  // chunks per gate (or up) copy: 1, or a stage's on the warp-MMA path
int expert_ffn_d_chunks(int d_ff);    // 64-column chunks of d_ff per down stage

// Builds the expert kernel's TMA descriptors (weights, H scratch at `h`,
// bf16 x at `x`: xb [B][d] for B <= 64, xd [B*k][d] above); wm: the
// gate/up boxes of the warp-MMA path.
bool encode_expert_maps(ExpertMaps *m, const moe_dims_t &d, const uint16_t *Wgate, const uint16_t *Wup,
                        const uint16_t *Wdown, const uint16_t *h, const uint16_t *x, int wm);

}  // namespace moe
