// Router and batch-aware re-selection kernels (sm_100a).
//
//  route_gemv_kernel    : logits = x Wg^T + bias in a fixed fp32 order
//      ("Router Caching and Optimization", "Analyzing Router Inference Cost",
//      step 1).  In the layer path for batches above 64 tokens it also
//      zeroes y.  (Batches up to 64 tokens run the whole layer in the fused
//      kernel of expert.cu, which uses the same dot products.)
//  route_topk_kernel    : warp per token: softmax (step 2) + top-k (step 3)
//      with a warp-shuffle reduction and register-resident keys.
//  reselect_kernel      : one CTA for the whole batch: (softmax +) top-k,
//      OEA / XShare / hierarchical XShare / affinity-binning re-selection
//      ("Lynx: Enabling Efficient MoE Inference through Dynamic Batch-Aware
//      Expert Selection", section 2.2), renormalised weights, per-expert
//      token lists and, for small batches, the dense weight matrix.
//
// Every floating-point step that decides an index is written with explicit
// round-to-nearest intrinsics (__fmaf_rn, __fadd_rn, __fsub_rn, __fdiv_rn)
// so that no contraction or reassociation can change a result:
//  - dot products: lane l accumulates elements j = 256 c + 8 l + t (c, t
//    ascending) with fma from +0, then a butterfly over lanes xor 16..1;
//  - softmax: m = max, q = exp(l - m) with the library's own exp, Z = lane
//    sums over e = l + 32 i (i ascending) then the butterfly, p = q / Z;
//  - rank order: logit descending, equal logits to the lower expert index.
#include <climits>
#include <cmath>

#include <cuda_bf16.h>

#include "internal.h"
#include "route_dev.cuh"

namespace moe {
namespace {

// ------------------------------------------------------------ route only --
template <int NI>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int B, int E,
                                                         int k, float *__restrict__ probs,
                                                         int32_t *__restrict__ topk_idx,
                                                         float *__restrict__ topk_w) {
    __shared__ int s_sel[8][K_MAX];
    __shared__ float s_w[8][K_MAX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * 8 + warp;
    if (b >= B) return;
    float l[NI], p[NI];
    load_row<NI>(logits + static_cast<size_t>(b) * E, E, lane, l);
    token_softmax<NI>(l, E, lane, p);
#pragma unroll
    for (int i = 0; i < NI; ++i)
        if (lane + 32 * i < E) probs[static_cast<size_t>(b) * E + lane + 32 * i] = p[i];
    unsigned long long key[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) key[i] = rank_key(l[i], lane + 32 * i);
    unsigned cand = valid_bits<NI>(E, lane);
    warp_select<NI>(key, cand, p, k, lane, s_sel[warp], s_w[warp]);
    renormalise_slots(s_sel[warp], s_w[warp], k, lane);
    if (lane < k) {
        topk_idx[static_cast<size_t>(b) * k + lane] = s_sel[warp][lane];
        topk_w[static_cast<size_t>(b) * k + lane] = s_w[warp][lane];
    }
}

// moe_reselect: the selection alone (one block of 1024 threads).
template <int NI>
__global__ void __launch_bounds__(1024, 1) reselect_kernel(ReselectArgs a) {
    // chained after the router (layer path): its logits are complete once
    // this wait returns
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    reselect_body<NI>(a, smem_raw);
}

// ------------------------------------------------------------ router GEMV --
// logits = x Wg^T (+ bias).  Block (bx, by) computes experts
// bx*epb .. bx*epb+epb-1 (one warp each) for tokens by*tpb .. by*tpb+tpb-1.
// One thread first loads those Wg rows and token rows into shared memory
// with TMA: each row is a column of 128-byte lines (32 floats) stored with
// the 128-byte swizzle, so lane l's two 16-byte loads of its group of eight
// columns 256 c + 8 l .. + 7 hit eight different bank quads in each
// quarter-warp phase.  Each lane runs the fixed-order fma chains of the
// block's tokens over its columns, chunk by chunk, the tokens' chains
// interleaved.
//
// Layer path for batches above 64 tokens (y != null): while the loads are
// in flight the blocks zero y, into which the expert kernel adds.
struct GemvArgs {
    const float *bias;
    int B, d, E;
    unsigned long long wait_ns;  // limit of the wait for the staged rows
    int epb, tpb;     // experts (= warps) and tokens per block; tpb <= 4
    int row_bytes;    // shared-memory stride of one staged row (multiple of 1024)
    int box_lines;    // 128-byte lines per TMA box
    int boxes;        // boxes per row
    float *logits;
    const float *x;   // layer path: the tokens (y has their shape)
    float *y;         // layer path: zeroed, or set to x when residual (else null)
    Counters *ctr;    // layer path: error word (else null)
    int residual;     // layer path: y = x (the experts add on top of the layer's input)
    int chained;      // launched with programmatic dependent launch after the previous layer
};

template <int NI>
__global__ void __launch_bounds__(32 * GEMV_EPB_MAX) route_gemv_kernel(const __grid_constant__ RouterMaps maps,
                                                                       const GemvArgs g) {
    extern __shared__ unsigned char gemv_smem[];
    __shared__ __align__(8) unsigned long long s_bar;
    __shared__ int s_fail;
    // the next kernel (the selection) may become resident while this runs
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // a layer of a stack reads the previous layer's output and workspace
    if (g.chained) asm volatile("griddepcontrol.wait;" ::: "memory");
    unsigned char *rows = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(gemv_smem) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = blockIdx.x * g.epb, b0 = blockIdx.y * g.tpb;
    const int nb = min(g.tpb, g.B - b0), ne = min(g.epb, g.E - e0);
    unsigned char *wrows = rows;                                 // [epb][row_bytes]
    unsigned char *xrows = rows + g.epb * g.row_bytes;           // [tpb][row_bytes]
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&s_bar)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_fail = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned bytes = static_cast<unsigned>((ne + nb) * g.boxes * g.box_lines * 128);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(&s_bar)), "r"(bytes)
                     : "memory");
        const int lines = g.d >> 5;  // 128-byte lines per row
        for (int r = 0; r < ne; ++r)
            for (int bx = 0; bx < g.boxes; ++bx)
                tma_rows(wrows + r * g.row_bytes + bx * g.box_lines * 128, &maps.wg,
                         (e0 + r) * lines + bx * g.box_lines, &s_bar);
        for (int r = 0; r < nb; ++r)
            for (int bx = 0; bx < g.boxes; ++bx)
                tma_rows(xrows + r * g.row_bytes + bx * g.box_lines * 128, &maps.x,
                         (b0 + r) * lines + bx * g.box_lines, &s_bar);
    }
    if (g.y != nullptr) layer_prep(g.x, g.B, g.d, nullptr, g.y, g.residual != 0);  // overlaps the loads
    if (!bar_try_wait0(&s_bar)) {
        // bounded: past the limit the block records the error and skips its
        // dot products, but still lets the copies land (up to a further
        // limit) before it exits
        const unsigned long long t0 = now_ns();
        bool late = false;
        while (!bar_try_wait0(&s_bar)) {
            const unsigned long long dt = now_ns() - t0;
            if (!late && dt > g.wait_ns) {
                late = true;
                s_fail = 1;
                if (g.ctr != nullptr) atomicCAS(&g.ctr->error, 0, DEV_TIMEOUT_FULL);
            }
            if (dt > g.wait_ns + GEMV_WAIT_LIMIT_NS) break;
        }
    }
    __syncthreads();

    if (warp < ne && !s_fail) {
        const int e = e0 + warp;
        float acc[GEMV_TPB_MAX];
#pragma unroll
        for (int t = 0; t < GEMV_TPB_MAX; ++t) acc[t] = 0.0f;
        if ((g.d & 255) == 0) gemv_rows<true>(wrows + warp * g.row_bytes, xrows, g.row_bytes, g.d, nb, lane, acc);
        else gemv_rows<false>(wrows + warp * g.row_bytes, xrows, g.row_bytes, g.d, nb, lane, acc);
        float mine = 0.0f;
#pragma unroll
        for (int t = 0; t < GEMV_TPB_MAX; ++t) {
            const float v = warp_butterfly_sum(acc[t]);
            if (lane == t) mine = v;
        }
        if (lane < nb) {
            const float v = g.bias ? __fadd_rn(mine, __ldg(g.bias + e)) : mine;
            g.logits[static_cast<size_t>(b0 + lane) * g.E + e] = v;
        }
    }
}

struct GemvShape {
    int epb, tpb, row_bytes, box_lines, boxes;
    size_t smem;
};

// Rows are staged in boxes of at most 256 lines (32 KB); a staged row takes
// a multiple of 1024 bytes so that every row starts a swizzle period.
// Tokens per block up to 4; experts per block up to 4, fewer when that
// leaves fewer than 120 blocks (small batches); both cut back while the
// staged rows exceed 160 KB.
GemvShape gemv_shape(const moe_dims_t &d) {
    GemvShape g;
    const int lines = d.d / 32;
    g.box_lines = router_box_lines(d.d);
    g.boxes = (lines + g.box_lines - 1) / g.box_lines;
    g.row_bytes = (g.boxes * g.box_lines * 128 + 1023) / 1024 * 1024;
    g.tpb = d.B < GEMV_TPB_MAX ? d.B : GEMV_TPB_MAX;
    g.epb = GEMV_EPB_MAX;
    while (g.epb > 1 && ((d.E + g.epb - 1) / g.epb) * ((d.B + g.tpb - 1) / g.tpb) < 120) --g.epb;
    while (static_cast<size_t>(g.tpb + g.epb) * g.row_bytes > GEMV_SMEM_MAX) {
        if (g.tpb >= g.epb && g.tpb > 1) --g.tpb;
        else if (g.epb > 1) --g.epb;
        else break;
    }
    g.smem = static_cast<size_t>(g.tpb + g.epb) * g.row_bytes + 1024;  // + alignment slack
    return g;
}

template <int NI>
cudaError_t launch_gemv_ni(const RouterMaps &maps, const GemvArgs &g, const GemvShape &sh, cudaStream_t s,
                           bool chained) {
    // the attributes belong to the function on each device: set them once per device
    static bool configured[MAX_DEVICES] = {};
    int dev = 0;
    cudaError_t derr = cudaGetDevice(&dev);
    if (derr != cudaSuccess) return derr;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaError_t err = cudaFuncSetAttribute(route_gemv_kernel<NI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(GEMV_SMEM_MAX + 1024));
        if (err != cudaSuccess) return err;
        // same shared-memory carve-out as the expert kernel: an SM switching
        // between the two needs no reconfiguration
        err = cudaFuncSetAttribute(route_gemv_kernel<NI>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (err != cudaSuccess) return err;
        configured[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((g.E + sh.epb - 1) / sh.epb, (g.B + sh.tpb - 1) / sh.tpb);
    cfg.blockDim = dim3(32 * sh.epb);
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = chained ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, route_gemv_kernel<NI>, maps, g);
}

cudaError_t launch_gemv(const RouterMaps &maps, const GemvArgs &g, const GemvShape &sh, cudaStream_t s,
                        bool chained = false) {
    switch (ni_for(g.E)) {
        case 1: return launch_gemv_ni<1>(maps, g, sh, s, chained);
        case 2: return launch_gemv_ni<2>(maps, g, sh, s, chained);
        case 4: return launch_gemv_ni<4>(maps, g, sh, s, chained);
        default: return launch_gemv_ni<8>(maps, g, sh, s, chained);
    }
}

GemvArgs make_gemv_args(const float *bias, const moe_dims_t &d, const GemvShape &sh, float *logits) {
    GemvArgs g;
    g.bias = bias;
    g.B = d.B;
    g.d = d.d;
    g.E = d.E;
    g.wait_ns = wait_limit_ns();
    g.epb = sh.epb;
    g.tpb = sh.tpb;
    g.row_bytes = sh.row_bytes;
    g.box_lines = sh.box_lines;
    g.boxes = sh.boxes;
    g.logits = logits;
    g.x = nullptr;
    g.y = nullptr;
    g.ctr = nullptr;
    g.residual = 0;
    g.chained = 0;
    return g;
}

}  // namespace

int router_box_lines(int d) { return d / 32 <= 256 ? d / 32 : 256; }

cudaError_t launch_router_logits(const RouterMaps &maps, const float *bias, const moe_dims_t &d, float *logits,
                                 cudaStream_t s) {
    const GemvShape sh = gemv_shape(d);
    return launch_gemv(maps, make_gemv_args(bias, d, sh, logits), sh, s);
}

cudaError_t launch_route_topk(const float *logits, const moe_dims_t &d, float *probs,
                              int32_t *topk_idx, float *topk_w, cudaStream_t s) {
    dim3 grid((d.B + 7) / 8);
    switch (ni_for(d.E)) {
        case 1: route_topk_kernel<1><<<grid, 256, 0, s>>>(logits, d.B, d.E, d.k, probs, topk_idx, topk_w); break;
        case 2: route_topk_kernel<2><<<grid, 256, 0, s>>>(logits, d.B, d.E, d.k, probs, topk_idx, topk_w); break;
        case 4: route_topk_kernel<4><<<grid, 256, 0, s>>>(logits, d.B, d.E, d.k, probs, topk_idx, topk_w); break;
        default: route_topk_kernel<8><<<grid, 256, 0, s>>>(logits, d.B, d.E, d.k, probs, topk_idx, topk_w); break;
    }
    return cudaGetLastError();
}

template <int NI>
static cudaError_t launch_reselect_ni(const ReselectArgs &a, size_t smem, bool chained, cudaStream_t s) {
    // the attributes belong to the function on each device: set them once per device
    static bool configured[MAX_DEVICES] = {};
    int dev = 0;
    cudaError_t derr = cudaGetDevice(&dev);
    if (derr != cudaSuccess) return derr;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaError_t err =
            cudaFuncSetAttribute(reselect_kernel<NI>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(reselect_kernel<NI>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (err != cudaSuccess) return err;
        configured[dev] = true;
    }
    if (!chained) {
        reselect_kernel<NI><<<1, 1024, smem, s>>>(a);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1024);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, reselect_kernel<NI>, a);
}

static cudaError_t launch_reselect_args(const ReselectArgs &a, size_t smem, bool chained, cudaStream_t s) {
    switch (ni_for(a.E)) {
        case 1: return launch_reselect_ni<1>(a, smem, chained, s);
        case 2: return launch_reselect_ni<2>(a, smem, chained, s);
        case 4: return launch_reselect_ni<4>(a, smem, chained, s);
        default: return launch_reselect_ni<8>(a, smem, chained, s);
    }
}

cudaError_t launch_reselect(const float *logits, const float *probs, const moe_dims_t &d,
                            const moe_reselect_t &r, int32_t *sel_idx, float *sel_w, const moe_lists_t &l,
                            cudaStream_t s) {
    ReselectArgs a = make_reselect_args(logits, const_cast<float *>(probs), false, d, r, sel_idx, sel_w, l,
                                        nullptr);
    const size_t smem = reselect_smem(d, r, &a.cache_rows);
    return launch_reselect_args(a, smem, false, s);
}

cudaError_t launch_layer_route(const RouterMaps &maps, const float *x, const float *bias, const moe_dims_t &d,
                               float *logits, float *y, Counters *ctr, bool residual, bool chained, cudaStream_t s) {
    const GemvShape sh = gemv_shape(d);
    GemvArgs g = make_gemv_args(bias, d, sh, logits);
    g.x = x;
    g.y = y;
    g.ctr = ctr;
    g.residual = residual ? 1 : 0;
    g.chained = chained ? 1 : 0;
    return launch_gemv(maps, g, sh, s, chained);
}

cudaError_t launch_layer_select(const float *logits, float *probs, const moe_dims_t &d, const moe_reselect_t &rule,
                                int32_t *sel_idx, float *sel_w, const moe_lists_t &l, int32_t *n_active_copy,
                                cudaStream_t s) {
    ReselectArgs a = make_reselect_args(logits, probs, true, d, rule, sel_idx, sel_w, l, n_active_copy);
    const size_t smem = reselect_smem(d, rule, &a.cache_rows);
    return launch_reselect_args(a, smem, true, s);
}

}  // namespace moe
