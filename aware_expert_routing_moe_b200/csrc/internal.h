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

// Counters the kernels share inside one workspace.
struct Counters {
    int32_t ticket;        // next work unit of the expert kernel
    int32_t error;         // first error code a kernel recorded (0 = none)
    int32_t pad[30];
    int32_t gu_done[E_MAX];  // finished gate/up units per active-expert slot
};

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
    size_t xb, h;
    size_t total;
};

WsLayout ws_layout(const moe_dims_t &d);

// Launchers (enqueue only; arguments already validated).
cudaError_t launch_router_logits(const float *x, const float *Wg, const float *bias,
                                 const moe_dims_t &d, float *logits, uint16_t *xb,
                                 float *y_zero, cudaStream_t s);
cudaError_t launch_route_topk(const float *logits, const moe_dims_t &d, float *probs,
                              int32_t *topk_idx, float *topk_w, cudaStream_t s);
cudaError_t launch_reselect(const float *logits, float *probs, bool fuse_softmax,
                            const moe_dims_t &d, const moe_reselect_t &r,
                            int32_t *sel_idx, float *sel_w, const moe_lists_t &l,
                            int32_t *n_active_copy, Counters *ctr, bool pdl, cudaStream_t s);
cudaError_t launch_ffn_prep(const float *x, const moe_dims_t &d, uint16_t *xb, float *y,
                            Counters *ctr, cudaStream_t s);

// TMA descriptors of the expert kernel: the three weight tensors and the H
// scratch as (64-column chunk, row, chunk index) boxes, and x in bf16 as
// single rows for gather-by-four loads.
struct ExpertMaps {
    CUtensorMap gate, up, down, h, x;
};
cudaError_t launch_expert_ffn(const ExpertMaps &maps, const uint16_t *xb,
                              const moe_dims_t &d, const moe_lists_t &l, float *y,
                              uint16_t *h, Counters *ctr, bool pdl, cudaStream_t s);
int expert_ffn_h_rows();              // rows of one H box (tokens per tile)
int expert_ffn_dense_batch(int B);    // 1 if gate/up stages load all B token rows at once
int expert_ffn_gather_cols(int d);    // columns of one x row box in gather mode
int expert_ffn_gu_rows();             // rows of Wgate / Wup per gate-up unit
int expert_ffn_d_rows();              // rows of Wdown per down unit
int expert_ffn_gu_chunks(int d);      // 64-column chunks of d per gate-up stage
int expert_ffn_d_chunks(int d_ff);    // 64-column chunks of d_ff per down stage

// Builds the expert kernel's TMA descriptors (weights, H scratch at `h`,
// bf16 x at `xb`).
bool encode_expert_maps(ExpertMaps *m, const moe_dims_t &d, const uint16_t *Wgate, const uint16_t *Wup,
                        const uint16_t *Wdown, const uint16_t *h, const uint16_t *xb);

}  // namespace moe
