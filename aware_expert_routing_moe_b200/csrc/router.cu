// Router and batch-aware re-selection kernels (sm_100a).
//
//  router_logits_kernel : logits = x Wg^T + bias in a fixed fp32 order
//      ("Router Caching and Optimization", "Analyzing Router Inference Cost",
//      step 1).  Optionally also writes x as bf16 for the expert kernel and
//      zeroes y (the layer path).
//  route_topk_kernel    : warp per token: softmax (step 2) + top-k (step 3)
//      with a warp-shuffle reduction and register-resident keys.
//  reselect_kernel      : one CTA for the whole batch: (softmax +) top-k,
//      OEA / XShare re-selection, renormalised weights, per-expert token
//      lists, and the reset of the expert kernel's counters.
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

namespace moe {
namespace {

constexpr unsigned FULL = 0xffffffffu;

// exp(x) for x in [-87, 0]: Cody-Waite reduction x = n ln2 + r with
// n = rint(x log2 e), ln2 split into a 15-significant-bit head and a float
// tail; exp(r) by its Taylor series to degree 7 (Horner, fma); 2^n applied
// to the exponent field.  +0 below -87.
__device__ __forceinline__ float exp_own(float x) {
    if (!(x >= -87.0f)) return 0.0f;
    const float kLog2e = 1.44269504088896341f;
    const float kLn2Hi = 0.693145751953125f;
    const float kLn2Lo = 1.42860682030941723212e-6f;
    const float n = rintf(__fmul_rn(x, kLog2e));
    float r = __fmaf_rn(-n, kLn2Hi, x);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = 1.0f / 5040.0f;
    p = __fmaf_rn(p, r, 1.0f / 720.0f);
    p = __fmaf_rn(p, r, 1.0f / 120.0f);
    p = __fmaf_rn(p, r, 1.0f / 24.0f);
    p = __fmaf_rn(p, r, 1.0f / 6.0f);
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    return __int_as_float(__float_as_int(p) + (static_cast<int>(n) << 23));
}

__device__ __forceinline__ float warp_butterfly_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(FULL, v, o));
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
    return v;
}

// Rank key: a larger key ranks earlier (larger logit, then lower index).
// Key 0 never occurs for a real expert and marks "no candidate".
__device__ __forceinline__ unsigned long long rank_key(float v, int idx) {
    v = (v == 0.0f) ? 0.0f : v;  // -0 and +0 compare equal
    const unsigned u = __float_as_uint(v);
    const unsigned ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<unsigned long long>(ord) << 32) | static_cast<unsigned>(~static_cast<unsigned>(idx));
}

// One round of warp arg-max over the lane's candidate bits; the winner is
// removed from the candidates.  Returns the expert index or -1.
template <int NI>
__device__ __forceinline__ int warp_take_best(const unsigned long long (&key)[NI], unsigned &cand,
                                              int lane) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int i = 0; i < NI; ++i)
        if ((cand >> i) & 1u) best = key[i] > best ? key[i] : best;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(FULL, best, o);
        best = other > best ? other : best;
    }
    if (best == 0ull) return -1;
    const int idx = static_cast<int>(~static_cast<unsigned>(best & 0xffffffffull));
    if ((idx & 31) == lane) cand &= ~(1u << (idx >> 5));
    return idx;
}

// Value held by the owner lane of expert e, broadcast to the warp.
template <int NI>
__device__ __forceinline__ float warp_fetch(const float (&v)[NI], int e) {
    float mine = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i)
        if (i == (e >> 5)) mine = v[i];
    return __shfl_sync(FULL, mine, e & 31);
}

template <int NI>
__device__ __forceinline__ void load_row(const float *row, int E, int lane, float (&l)[NI]) {
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        const int e = lane + 32 * i;
        l[i] = e < E ? row[e] : -INFINITY;
    }
}

template <int NI>
__device__ __forceinline__ unsigned valid_bits(int E, int lane) {
    unsigned m = 0;
#pragma unroll
    for (int i = 0; i < NI; ++i)
        if (lane + 32 * i < E) m |= 1u << i;
    return m;
}

// Softmax of one token's logits held lane-distributed (e = lane + 32 i).
template <int NI>
__device__ __forceinline__ void token_softmax(const float (&l)[NI], int E, int lane, float (&p)[NI]) {
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NI; ++i)
        if (lane + 32 * i < E) m = fmaxf(m, l[i]);
    m = warp_max(m);
    float q[NI];
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        if (lane + 32 * i < E) {
            q[i] = exp_own(__fsub_rn(l[i], m));
            acc = __fadd_rn(acc, q[i]);
        } else {
            q[i] = 0.0f;
        }
    }
    const float Z = warp_butterfly_sum(acc);
#pragma unroll
    for (int i = 0; i < NI; ++i) p[i] = (lane + 32 * i < E) ? __fdiv_rn(q[i], Z) : 0.0f;
}

// Top-r of the candidate experts by rank key, r rounds of warp arg-max.
// Lane 0 writes the winners to out[0..) and their probabilities to pout[0..)
// (when pout != nullptr).  Stops early when no candidate is left; returns the
// number found.
template <int NI>
__device__ int warp_select(const unsigned long long (&key)[NI], unsigned &cand, const float (&p)[NI], int r,
                           int lane, int *out, float *pout) {
    int n = 0;
#pragma unroll 1
    for (int j = 0; j < r; ++j) {
        const int e = warp_take_best<NI>(key, cand, lane);
        if (e < 0) break;
        const float pe = warp_fetch<NI>(p, e);
        if (lane == 0) {
            out[j] = e;
            if (pout) pout[j] = pe;
        }
        ++n;
    }
    __syncwarp();
    return n;
}

// Gate weights renormalised over the chosen slots: sel[0..k) and their
// probabilities pv[0..k) in shared memory (sel < 0 = empty slot); pv is
// overwritten with the weights.  The sum runs in slot order from +0 (lane 0),
// then lane j divides slot j.
__device__ void renormalise_slots(const int *sel, float *pv, int k, int lane) {
    float s = 0.0f;
    if (lane == 0) {
#pragma unroll 1
        for (int j = 0; j < k; ++j)
            if (sel[j] >= 0) s = __fadd_rn(s, pv[j]);
    }
    s = __shfl_sync(FULL, s, 0);
    __syncwarp();
    if (lane < k) pv[lane] = sel[lane] >= 0 ? __fdiv_rn(pv[lane], s) : 0.0f;
    __syncwarp();
}

// ------------------------------------------------------------------ K1 --
// Block (bx, by) computes experts 8 bx .. 8 bx + 7 (one per warp) for the
// tokens tb * by .. tb * by + tb - 1.  The block stages those token rows in
// shared memory; each warp holds up to R_CH 256-column chunks of its Wg row
// in registers (all loads issued before any use) and runs the fixed-order
// fma chains against the shared rows.
constexpr int R_TB = 4;  // tokens per block (at most)
constexpr int R_CH = 8;  // 256-column chunks of a Wg row held at once

__global__ void __launch_bounds__(256) router_logits_kernel(
    const float *__restrict__ x, const float *__restrict__ Wg, const float *__restrict__ bias,
    int B, int d, int E, int tb, float *__restrict__ logits, uint16_t *__restrict__ xb,
    float *__restrict__ y_zero) {
    extern __shared__ float4 xs4[];  // [tb][d / 4]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + warp;
    const int b0 = blockIdx.y * tb;
    const int nb = min(tb, B - b0);
    const int nch = (d + 255) / 256;
    const float *wrow = Wg + static_cast<size_t>(min(e, E - 1)) * d;
    // first R_CH chunks of this warp's Wg row: issued before anything waits
    float4 w[R_CH][2];
#pragma unroll
    for (int cc = 0; cc < R_CH; ++cc) {
        const int j0 = 256 * cc + 8 * lane;
        if (cc < nch && j0 < d) {
            w[cc][0] = __ldg(reinterpret_cast<const float4 *>(wrow + j0));
            w[cc][1] = __ldg(reinterpret_cast<const float4 *>(wrow + j0 + 4));
        }
    }
    {
        // stage the token rows: eight loads in flight per thread, then stores
        const float4 *src = reinterpret_cast<const float4 *>(x) + static_cast<size_t>(b0) * (d / 4);
        const int total4 = nb * (d / 4);
#pragma unroll 1
        for (int base = 0; base < total4; base += 8 * 256) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * 256 + static_cast<int>(threadIdx.x);
                if (i < total4) v[u] = __ldg(src + i);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = base + u * 256 + static_cast<int>(threadIdx.x);
                if (i < total4) xs4[i] = v[u];
            }
        }
    }
    __syncthreads();
    if (e < E) {
        float acc[R_TB];
#pragma unroll
        for (int t = 0; t < R_TB; ++t) acc[t] = 0.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < nch; c0 += R_CH) {
            if (c0 > 0) {
#pragma unroll
                for (int cc = 0; cc < R_CH; ++cc) {
                    const int j0 = 256 * (c0 + cc) + 8 * lane;
                    if (c0 + cc < nch && j0 < d) {
                        w[cc][0] = __ldg(reinterpret_cast<const float4 *>(wrow + j0));
                        w[cc][1] = __ldg(reinterpret_cast<const float4 *>(wrow + j0 + 4));
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < R_TB; ++t) {
                if (t >= nb) break;
                float a = acc[t];
#pragma unroll
                for (int cc = 0; cc < R_CH; ++cc) {
                    const int j0 = 256 * (c0 + cc) + 8 * lane;
                    if (c0 + cc < nch && j0 < d) {
                        const float4 x0 = xs4[(t * d + j0) / 4];
                        const float4 x1 = xs4[(t * d + j0) / 4 + 1];
                        a = __fmaf_rn(x0.x, w[cc][0].x, a);
                        a = __fmaf_rn(x0.y, w[cc][0].y, a);
                        a = __fmaf_rn(x0.z, w[cc][0].z, a);
                        a = __fmaf_rn(x0.w, w[cc][0].w, a);
                        a = __fmaf_rn(x1.x, w[cc][1].x, a);
                        a = __fmaf_rn(x1.y, w[cc][1].y, a);
                        a = __fmaf_rn(x1.z, w[cc][1].z, a);
                        a = __fmaf_rn(x1.w, w[cc][1].w, a);
                    }
                }
                acc[t] = a;
            }
        }
        float mine = 0.0f;
#pragma unroll
        for (int t = 0; t < R_TB; ++t) {
            const float v = warp_butterfly_sum(acc[t]);
            if (lane == t) mine = v;
        }
        if (lane < nb) {
            const float v = bias ? __fadd_rn(mine, __ldg(bias + e)) : mine;
            logits[static_cast<size_t>(b0 + lane) * E + e] = v;
        }
    }
    if (xb != nullptr) {
        // layer path: x -> bf16 copy for the expert kernel, y = 0
        const int n4 = B * d / 4;
        const int nthreads = gridDim.x * gridDim.y * blockDim.x;
        for (int i = (blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
             i += nthreads) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(x) + i);
            const unsigned lo = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x))) |
                                (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
            const unsigned hi = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.z))) |
                                (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.w))) << 16);
            reinterpret_cast<uint2 *>(xb)[i] = make_uint2(lo, hi);
            if (y_zero) reinterpret_cast<float4 *>(y_zero)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // let the dependent (re-selection) kernel become resident; it waits for
    // this grid's completion before reading the logits
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

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

// -------------------------------------------------------------- reselect --
struct ReselectArgs {
    const float *logits;
    float *probs;  // read, or written when fuse_softmax
    int fuse_softmax;
    int cache_rows;  // logits / probabilities kept in shared memory
    int B, E, k, mode, k0, budget;
    int32_t *sel_idx;
    float *sel_w;
    moe_lists_t lists;
    int32_t *n_active_copy;
    Counters *ctr;
};

// Inclusive scan over threads 0..255 (value 0 for t >= n); every thread of
// the block must call it.  Returns the inclusive prefix, sets *total.
__device__ int block_scan256(int v, int *wsum, int *total) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += u;
    }
    if (warp < 8 && lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (t == 0) {
        int run = 0;
        for (int i = 0; i < 8; ++i) {
            const int s = wsum[i];
            wsum[i] = run;
            run += s;
        }
        wsum[8] = run;
    }
    __syncthreads();
    const int res = (warp < 8) ? incl + wsum[warp] : 0;
    *total = wsum[8];
    __syncthreads();
    return res;
}

// Order-preserving unsigned image of a logit (larger logit -> larger value,
// -0 and +0 equal); never 0 for a finite or infinite float.
__device__ __forceinline__ unsigned ord_of(float v) {
    v = (v == 0.0f) ? 0.0f : v;
    const unsigned u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float float_of_ord(unsigned o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// One round of warp arg-max over candidate bits with two hardware warp
// reductions: the largest logit image, then, among lanes holding it, the
// lowest expert index.  The winner leaves the candidates.  -1 if none.
template <int NI>
__device__ __forceinline__ int warp_argmax(const unsigned (&ord)[NI], unsigned &cand, int lane) {
    unsigned bo = 0u, bl = 0u;  // this lane's best: logit image, ~index
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        if ((cand >> i) & 1u) {
            const unsigned lo = ~static_cast<unsigned>(lane + 32 * i);
            if (ord[i] > bo || (ord[i] == bo && lo > bl)) {
                bo = ord[i];
                bl = lo;
            }
        }
    }
    const unsigned H = __reduce_max_sync(FULL, bo);
    if (H == 0u) return -1;
    const unsigned Lw = __reduce_max_sync(FULL, bo == H ? bl : 0u);
    const int idx = static_cast<int>(~Lw);
    if ((idx & 31) == lane) cand &= ~(1u << (idx >> 5));
    return idx;
}

// Softmax of one token (row lane-distributed: e = lane + 32 i), max by
// warp reduction of logit images, sum in the canonical lane/butterfly order.
template <int NI>
__device__ __forceinline__ void token_softmax_r(const float (&l)[NI], const unsigned (&ord)[NI], int E, int lane,
                                                float (&p)[NI]) {
    unsigned om = 0u;
#pragma unroll
    for (int i = 0; i < NI; ++i)
        if (lane + 32 * i < E) om = ord[i] > om ? ord[i] : om;
    const float m = float_of_ord(__reduce_max_sync(FULL, om));
    float q[NI];
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        if (lane + 32 * i < E) {
            q[i] = exp_own(__fsub_rn(l[i], m));
            acc = __fadd_rn(acc, q[i]);
        } else {
            q[i] = 0.0f;
        }
    }
    const float Z = warp_butterfly_sum(acc);
#pragma unroll
    for (int i = 0; i < NI; ++i) p[i] = (lane + 32 * i < E) ? __fdiv_rn(q[i], Z) : 0.0f;
}

// Records slot j of one token: every lane adds the winner's probability to
// the running sum (slot order, from +0); lane j keeps it for its weight.
__device__ __forceinline__ void take_slot(int j, float pe, int lane, float &sum, float &myp) {
    sum = __fadd_rn(sum, pe);
    if (lane == j) myp = pe;
}

template <int NI>
__global__ void __launch_bounds__(1024, 1) reselect_kernel(ReselectArgs a) {
    // wait until the router's logits are complete and visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the expert kernel may become resident now; it waits for this grid
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int B = a.B, E = a.E, k = a.k;
    const int BW = (B + 31) >> 5;
    int *T = reinterpret_cast<int *>(smem_raw);                    // [B][k] first ranks
    unsigned *ASSIGN = reinterpret_cast<unsigned *>(T + B * k);     // [E][BW] final assignment
    unsigned *TMEMB = ASSIGN + E * BW;                                // [E][BW] top-k membership
    float *PC = reinterpret_cast<float *>(TMEMB + E * BW);           // [B][E] probability cache
    float *LC = PC + (a.cache_rows ? B * E : 0);                      // [B][E] logit cache
    __shared__ float s_score[E_MAX];
    __shared__ int s_off[E_MAX];
    __shared__ unsigned ukept[E_MAX / 32], ubase[E_MAX / 32], sbits[E_MAX / 32];
    __shared__ int wsum[9];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < 2 * E * BW; i += blockDim.x) ASSIGN[i] = 0u;  // and TMEMB
    if (tid < E_MAX / 32) ukept[tid] = ubase[tid] = sbits[tid] = 0u;
    __syncthreads();

    const int mode = a.mode;
    float *prob_rows = a.cache_rows ? PC : a.probs;
    const float *logit_rows = a.cache_rows ? LC : a.logits;

    // ---- phase 1: softmax (layer path) and each token's first ranks
    const int r1 = (mode == MOE_RESELECT_OEA) ? a.k0 : k;
#pragma unroll 1
    for (int b = warp; b < B; b += 32) {
        float l[NI], p[NI];
        unsigned ord[NI];
        load_row<NI>(a.logits + static_cast<size_t>(b) * E, E, lane, l);
#pragma unroll
        for (int i = 0; i < NI; ++i) ord[i] = ord_of(l[i]);
        if (a.fuse_softmax) {
            token_softmax_r<NI>(l, ord, E, lane, p);
        } else {
            load_row<NI>(a.probs + static_cast<size_t>(b) * E, E, lane, p);
        }
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int e = lane + 32 * i;
            if (e < E) {
                if (a.cache_rows) {
                    LC[b * E + e] = l[i];
                    PC[b * E + e] = p[i];
                } else if (a.fuse_softmax) {
                    a.probs[static_cast<size_t>(b) * E + e] = p[i];
                }
            }
        }
        unsigned cand = valid_bits<NI>(E, lane);
        float sum = 0.0f, myp = 0.0f;
        int mye = -1;
#pragma unroll 1
        for (int j = 0; j < r1; ++j) {
            const int e = warp_argmax<NI>(ord, cand, lane);
            if (lane == j) mye = e;
            if (mode == MOE_RESELECT_NONE) take_slot(j, warp_fetch<NI>(p, e), lane, sum, myp);
        }
        if (lane < r1) {
            T[b * k + lane] = mye;
            if (mode == MOE_RESELECT_OEA) atomicOr(&ukept[mye >> 5], 1u << (mye & 31));
            if (mode == MOE_RESELECT_XSHARE) {
                atomicOr(&ubase[mye >> 5], 1u << (mye & 31));
                atomicOr(&TMEMB[mye * BW + (b >> 5)], 1u << (b & 31));
            }
        }
        if (mode == MOE_RESELECT_NONE && lane < k) {
            a.sel_idx[static_cast<size_t>(b) * k + lane] = mye;
            a.sel_w[static_cast<size_t>(b) * k + lane] = __fdiv_rn(myp, sum);
            atomicOr(&ASSIGN[mye * BW + (b >> 5)], 1u << (b & 31));
        }
    }
    __syncthreads();

    // ---- XShare: batch scores, budget, greedy set (= top-M' by score)
    if (mode == MOE_RESELECT_XSHARE) {
        if (tid < E) {
            float sc = 0.0f;
#pragma unroll 1
            for (int b = 0; b < B; ++b)
                if ((TMEMB[tid * BW + (b >> 5)] >> (b & 31)) & 1u)
                    sc = __fadd_rn(sc, prob_rows[static_cast<size_t>(b) * E + tid]);
            s_score[tid] = sc;
        }
        __syncthreads();
        if (tid < E && ((ubase[tid >> 5] >> (tid & 31)) & 1u)) {
            int nb = 0;
            for (int i = 0; i < E_MAX / 32; ++i) nb += __popc(ubase[i]);
            const int Mp = a.budget < nb ? a.budget : nb;
            const float se = s_score[tid];
            int rank = 0;
#pragma unroll 1
            for (int e2 = 0; e2 < E; ++e2) {
                if (!((ubase[e2 >> 5] >> (e2 & 31)) & 1u)) continue;
                const float s2 = s_score[e2];
                rank += (s2 > se || (s2 == se && e2 < tid)) ? 1 : 0;
            }
            if (rank < Mp) atomicOr(&sbits[tid >> 5], 1u << (tid & 31));
        }
        __syncthreads();
    }

    // ---- phase 2: OEA fills / XShare top-k within the batch set; weights
    if (mode != MOE_RESELECT_NONE) {
#pragma unroll 1
        for (int b = warp; b < B; b += 32) {
            float l[NI], p[NI];
            unsigned ord[NI];
            load_row<NI>(logit_rows + static_cast<size_t>(b) * E, E, lane, l);
            load_row<NI>(prob_rows + static_cast<size_t>(b) * E, E, lane, p);
#pragma unroll
            for (int i = 0; i < NI; ++i) ord[i] = ord_of(l[i]);
            unsigned cand = 0;
            const unsigned *bits = (mode == MOE_RESELECT_OEA) ? ukept : sbits;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int e = lane + 32 * i;
                if (e < E && ((bits[e >> 5] >> (e & 31)) & 1u)) cand |= 1u << i;
            }
            float sum = 0.0f, myp = 0.0f;
            int mye = -1;
            const int kk = (mode == MOE_RESELECT_OEA) ? a.k0 : 0;
#pragma unroll 1
            for (int j = 0; j < kk; ++j) {  // kept experts first, in rank order
                const int e = T[b * k + j];
                if ((e & 31) == lane) cand &= ~(1u << (e >> 5));
                if (lane == j) mye = e;
                take_slot(j, warp_fetch<NI>(p, e), lane, sum, myp);
            }
#pragma unroll 1
            for (int j = kk; j < k; ++j) {
                const int e = warp_argmax<NI>(ord, cand, lane);
                if (e < 0) break;
                if (lane == j) mye = e;
                take_slot(j, warp_fetch<NI>(p, e), lane, sum, myp);
            }
            if (lane < k) {
                a.sel_idx[static_cast<size_t>(b) * k + lane] = mye;
                a.sel_w[static_cast<size_t>(b) * k + lane] = mye >= 0 ? __fdiv_rn(myp, sum) : 0.0f;
                if (mye >= 0) atomicOr(&ASSIGN[mye * BW + (b >> 5)], 1u << (b & 31));
            }
        }
    }
    __syncthreads();

    // ---- phase 3: counts, active list, offsets (one scan of flag and count)
    int cnt = 0;
    if (tid < E)
        for (int wd = 0; wd < BW; ++wd) cnt += __popc(ASSIGN[tid * BW + wd]);
    const int flag = (tid < E && cnt > 0) ? 1 : 0;
    int tot = 0;
    const int incl = block_scan256((flag << 16) | cnt, wsum, &tot);
    const int n_active = tot >> 16, total = tot & 0xffff;
    if (tid < E) {
        const int off = (incl & 0xffff) - cnt;
        s_off[tid] = off;
        if (flag) {
            a.lists.active[(incl >> 16) - 1] = tid;
            a.lists.offsets[(incl >> 16) - 1] = off;
        }
    }
    if (tid >= n_active && tid < E) a.lists.active[tid] = -1;
    if (tid >= n_active && tid <= E) a.lists.offsets[tid] = total;
    if (tid == 0) {
        *a.lists.n_active = n_active;
        if (a.n_active_copy) *a.n_active_copy = n_active;
    }
    __syncthreads();

    // ---- phase 4: compaction (expert ascending, token ascending)
    for (int i = tid; i < B * k; i += blockDim.x) {
        const int b = i / k;
        const int e = a.sel_idx[i];
        if (e < 0) continue;
        int before = 0;
        for (int wd = 0; wd < (b >> 5); ++wd) before += __popc(ASSIGN[e * BW + wd]);
        before += __popc(ASSIGN[e * BW + (b >> 5)] & ((1u << (b & 31)) - 1u));
        const int pos = s_off[e] + before;
        a.lists.tok[pos] = b;
        a.lists.w[pos] = a.sel_w[i];
    }
    for (int i = total + tid; i < B * k; i += blockDim.x) {
        a.lists.tok[i] = -1;
        a.lists.w[i] = 0.0f;
    }
    // ---- reset the expert kernel's counters (layer path)
    if (a.ctr) {
        if (tid == 0) a.ctr->ticket = 0;
        for (int i = tid; i < E_MAX; i += blockDim.x) a.ctr->gu_done[i] = 0;
    }
}

int ni_for(int E) { return E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8; }

}  // namespace

cudaError_t launch_router_logits(const float *x, const float *Wg, const float *bias,
                                 const moe_dims_t &d, float *logits, uint16_t *xb,
                                 float *y_zero, cudaStream_t s) {
    static bool configured = false;  // one GPU per process
    if (!configured) {
        const cudaError_t err = cudaFuncSetAttribute(router_logits_kernel,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, 192 * 1024);
        if (err != cudaSuccess) return err;
        configured = true;
    }
    // tokens per block: up to R_TB, and at most 160 KB of staged rows
    int tb = R_TB;
    while (tb > 1 && static_cast<size_t>(tb) * d.d * 4 > 160u * 1024u) --tb;
    dim3 grid((d.E + 7) / 8, (d.B + tb - 1) / tb);
    const size_t smem = static_cast<size_t>(tb) * d.d * 4;
    router_logits_kernel<<<grid, 256, smem, s>>>(x, Wg, bias, d.B, d.d, d.E, tb, logits, xb, y_zero);
    return cudaGetLastError();
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
static cudaError_t launch_reselect_ni(const ReselectArgs &a, size_t smem, bool pdl, cudaStream_t s) {
    static bool configured = false;  // the attribute is per function; set it once
    cudaError_t err = cudaSuccess;
    if (!configured) {
        err = cudaFuncSetAttribute(reselect_kernel<NI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   96 * 1024);
        if (err != cudaSuccess) return err;
        configured = true;
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
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, reselect_kernel<NI>, a);
}

cudaError_t launch_reselect(const float *logits, float *probs, bool fuse_softmax,
                            const moe_dims_t &d, const moe_reselect_t &r,
                            int32_t *sel_idx, float *sel_w, const moe_lists_t &l,
                            int32_t *n_active_copy, Counters *ctr, bool pdl, cudaStream_t s) {
    ReselectArgs a;
    a.logits = logits;
    a.probs = probs;
    a.fuse_softmax = fuse_softmax ? 1 : 0;
    a.B = d.B;
    a.E = d.E;
    a.k = d.k;
    a.mode = r.mode;
    a.k0 = r.k0;
    a.budget = r.budget;
    a.sel_idx = sel_idx;
    a.sel_w = sel_w;
    a.lists = l;
    a.n_active_copy = n_active_copy;
    a.ctr = ctr;
    const int BW = (d.B + 31) / 32;
    const size_t base = static_cast<size_t>(d.B) * d.k * 4 + static_cast<size_t>(d.E) * BW * 8;
    const size_t rows = static_cast<size_t>(d.B) * d.E * 8;
    a.cache_rows = (base + rows <= 96u * 1024u) ? 1 : 0;
    const size_t smem = base + (a.cache_rows ? rows : 0);
    switch (ni_for(d.E)) {
        case 1: return launch_reselect_ni<1>(a, smem, pdl, s);
        case 2: return launch_reselect_ni<2>(a, smem, pdl, s);
        case 4: return launch_reselect_ni<4>(a, smem, pdl, s);
        default: return launch_reselect_ni<8>(a, smem, pdl, s);
    }
}

}  // namespace moe
