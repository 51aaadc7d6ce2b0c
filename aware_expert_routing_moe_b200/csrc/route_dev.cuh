// Device code shared by the router kernels and the fused layer kernel:
// the fixed-order fp32 arithmetic of the router (dot products, the
// library's own exp, softmax, rank order), warp-level ranking, and the
// one-block batch selection (re-selection rules, weights, token lists).
// Included by router.cu and expert.cu; everything here has internal
// linkage.
#pragma once

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
    // global rows written by other blocks or kernels: read through L2
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        const int e = lane + 32 * i;
        l[i] = e < E ? __ldcg(row + e) : -INFINITY;
    }
}

// A row in shared or global memory (generic load).
template <int NI>
__device__ __forceinline__ void load_row_any(const float *row, int E, int lane, float (&l)[NI]) {
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

// -------------------------------------------------------------- reselect --
struct ReselectArgs {
    const float *logits;
    float *probs;  // read, or written when fuse_softmax
    int fuse_softmax;
    int cache_rows;  // logits / probabilities kept in shared memory
    int B, E, k, mode, k0, budget;
    int group;  // hierarchical XShare: tokens per request
    int32_t *sel_idx;
    float *sel_w;
    moe_lists_t lists;
    int32_t *n_active_copy;
    Counters *ctr;  // fused layer kernel: the counters of the call (else null)
    // dense weights [active slot][B] (0 where a token does not use the
    // expert), written when non-null
    float *wd;
    // fused layer kernel: publish the activated set in ctr->pubs as soon as
    // it is fixed (the batch-wide rules; the other CTAs stream from it)
    int publish_set;
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

// Sort keys of a batch-wide score order (score descending, ties to the
// lower expert index), unique per expert; 0 marks a non-member.  Affinity
// scores are exact integers below 2^44; XShare scores are non-negative
// floats, whose bit patterns order like their values.
__device__ __forceinline__ unsigned long long key_int_score(unsigned long long sc, int e) {
    return (sc << 8) | static_cast<unsigned long long>(255 - e);
}
__device__ __forceinline__ unsigned long long key_float_score(float sc, int e) {
    return (static_cast<unsigned long long>(__float_as_uint(sc)) << 32) | static_cast<unsigned>(~static_cast<unsigned>(e));
}
// Position of expert e in the score order of the members (keys > 0),
// computed by one warp: the number of members with a larger key.
__device__ __forceinline__ int warp_rank(const unsigned long long *key, int E, int e, int lane) {
    const unsigned long long ke = key[e];
    unsigned c = 0u;
    for (int e2 = lane; e2 < E; e2 += 32) c += key[e2] > ke ? 1u : 0u;
    return static_cast<int>(__reduce_add_sync(FULL, c));
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

// ---------------------------------------------------- warp top-R set --
// The R largest of a token's rank keys (logit image, then lower index),
// R a power of two: every lane ends with the same list, descending.  Each
// lane first sorts its own keys; then, at each of five butterfly levels, a
// lane merges its list with its partner's: the elementwise maximum of the
// list and the reversed partner list holds the R largest of the two (a
// bitonic sequence), which a bitonic merge sorts.  Five shuffle levels
// instead of R dependent rounds of warp arg-max.  Key 0 = no expert.
__device__ __forceinline__ unsigned long long topr_key(unsigned ord, int e) {
    return (static_cast<unsigned long long>(ord) << 32) | static_cast<unsigned>(~static_cast<unsigned>(e));
}
__device__ __forceinline__ int topr_expert(unsigned long long key) {
    return key == 0ull ? -1 : static_cast<int>(~static_cast<unsigned>(key & 0xffffffffull));
}
template <int R>
__device__ __forceinline__ void bitonic_sort_desc(unsigned long long (&v)[R]) {
    // v is bitonic: sort it descending
#pragma unroll
    for (int half = R / 2; half >= 1; half >>= 1)
#pragma unroll
        for (int i = 0; i < R; ++i)
            if ((i & half) == 0) {
                const unsigned long long a = v[i], b = v[i + half];
                v[i] = a > b ? a : b;
                v[i + half] = a > b ? b : a;
            }
}
// top = the R largest of top and other (both descending), descending.
template <int R>
__device__ __forceinline__ void merge_top(unsigned long long (&top)[R], const unsigned long long (&other)[R]) {
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const unsigned long long b = other[R - 1 - i];
        top[i] = top[i] > b ? top[i] : b;
    }
    bitonic_sort_desc<R>(top);
}
// v (any order) sorted descending: runs of doubling length, each made
// bitonic by reversing its second half, then merged.
template <int R>
__device__ __forceinline__ void sort_desc(unsigned long long (&v)[R]) {
#pragma unroll
    for (int len = 2; len <= R; len <<= 1) {
#pragma unroll
        for (int base = 0; base < R; base += len)
#pragma unroll
            for (int i = 0; i < len / 4; ++i) {
                const unsigned long long t = v[base + len / 2 + i];
                v[base + len / 2 + i] = v[base + len - 1 - i];
                v[base + len - 1 - i] = t;
            }
#pragma unroll
        for (int half = len / 2; half >= 1; half >>= 1)
#pragma unroll
            for (int i = 0; i < R; ++i)
                if ((i & half) == 0) {
                    const unsigned long long a = v[i], b = v[i + half];
                    v[i] = a > b ? a : b;
                    v[i + half] = a > b ? b : a;
                }
    }
}
template <int NI, int R>
__device__ __forceinline__ void warp_top_r(const unsigned (&ord)[NI], int E, int lane, unsigned long long (&top)[R]) {
    // this lane's keys (e = lane + 32 i), R at a time
#pragma unroll
    for (int c = 0; c < (NI + R - 1) / R; ++c) {
        unsigned long long cur[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int ii = c * R + i;
            const int e = lane + 32 * ii;
            cur[i] = (ii < NI && e < E) ? topr_key(ord[ii < NI ? ii : 0], e) : 0ull;
        }
        sort_desc<R>(cur);
        if (c == 0) {
#pragma unroll
            for (int i = 0; i < R; ++i) top[i] = cur[i];
        } else {
            merge_top<R>(top, cur);
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        unsigned long long other[R];
#pragma unroll
        for (int i = 0; i < R; ++i) other[i] = __shfl_xor_sync(FULL, top[i], o);
        merge_top<R>(top, other);
    }
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

// Dense weights of token b: wd[i][b] for every active slot i (0 unless the
// token chose active[i]).  Lane j < k holds the token's slot j.
__device__ void write_dense_weights(float *wd, int B, int b, int n_active, const int *s_rank, int mye, float myw,
                                    int k, int lane) {
    for (int i = lane; i < n_active; i += 32) wd[static_cast<size_t>(i) * B + b] = 0.0f;
    __syncwarp();
    if (lane < k && mye >= 0) wd[static_cast<size_t>(s_rank[mye]) * B + b] = myw;
}

// The batch-level selection, run by one block (any multiple of 32 threads,
// at least 256): phase 1 per token (softmax in the layer path, first ranks),
// the batch set of a batch-wide rule, phase 2 per token (OEA fills / top-k
// within the batch set, weights), then the per-expert lists.  Every thread
// of the block must call it.
template <int NI>
__device__ void reselect_body(const ReselectArgs &a, unsigned char *smem_raw) {
    const int B = a.B, E = a.E, k = a.k;
    const int BW = (B + 31) >> 5;
    const int nwarps = blockDim.x >> 5;
    int *T = reinterpret_cast<int *>(smem_raw);                    // [B][k] first ranks
    unsigned *ASSIGN = reinterpret_cast<unsigned *>(T + B * k);     // [E][BW] final assignment
    unsigned *TMEMB = ASSIGN + E * BW;                                // [E][BW] top-k membership
    float *PC = reinterpret_cast<float *>(TMEMB + E * BW);           // [B][E] probability cache
    float *LC = PC + (a.cache_rows ? B * E : 0);                      // [B][E] logit cache
    // hierarchical XShare: bit r of word RPICK[e * BW + r / 32] = request r
    // picked expert e (present only in that mode)
    unsigned *RPICK = reinterpret_cast<unsigned *>(LC + (a.cache_rows ? B * E : 0));
    __shared__ float s_score[E_MAX];
    __shared__ int s_off[E_MAX];
    __shared__ int s_rank[E_MAX];  // expert -> active slot (dense weights)
    __shared__ unsigned ukept[E_MAX / 32], ubase[E_MAX / 32], sbits[E_MAX / 32], r0bits[E_MAX / 32];
    __shared__ unsigned long long s_aff[E_MAX];  // affinity scores (exact integers)
    __shared__ int s_pos[E_MAX];                 // position in the affinity score order
    __shared__ int s_M;
    __shared__ int wsum[9];
    __shared__ int s_nact;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < 2 * E * BW; i += blockDim.x) ASSIGN[i] = 0u;  // and TMEMB
    if (tid < E_MAX / 32) ukept[tid] = ubase[tid] = sbits[tid] = r0bits[tid] = 0u;
    for (int i = tid; i < E_MAX; i += blockDim.x) s_aff[i] = 0ull;
    if (tid == 0) s_M = k;
    __syncthreads();

    const int mode = a.mode;
    float *prob_rows = a.cache_rows ? PC : a.probs;
    const float *logit_rows = a.cache_rows ? LC : a.logits;
    const bool dense_w = a.wd != nullptr;

    // ---- phase 1: softmax (layer path) and each token's first ranks
    const int r1 = (mode == MOE_RESELECT_OEA) ? a.k0 : k;
#pragma unroll 1
    for (int b = warp; b < B; b += nwarps) {
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
        if (mode == MOE_RESELECT_AFFINITY) {
            // confidence = gap of the two top probabilities, in bins of
            // width k/E (min(32, ceil(E/k)) of them); each of the token's
            // top-k experts scores 2^bin
            const int r0 = __shfl_sync(FULL, mye, 0);
            const int r1e = k >= 2 ? __shfl_sync(FULL, mye, 1) : warp_argmax<NI>(ord, cand, lane);
            const float p0 = warp_fetch<NI>(p, r0);
            const float c = r1e >= 0 ? __fsub_rn(p0, warp_fetch<NI>(p, r1e)) : p0;
            const float cE = __fmul_rn(c, static_cast<float>(E));
            const int nb = min(32, (E + k - 1) / k);
            int bin = 0;
            for (int j = nb - 1; j > 0; --j)
                if (static_cast<float>(j * k) <= cE) {
                    bin = j;
                    break;
                }
            if (lane < k) atomicAdd(&s_aff[mye], 1ull << bin);
            if (lane == 0) atomicOr(&r0bits[r0 >> 5], 1u << (r0 & 31));
        }
        if (lane < r1) {
            T[b * k + lane] = mye;
            if (mode == MOE_RESELECT_OEA) atomicOr(&ukept[mye >> 5], 1u << (mye & 31));
            if (mode != MOE_RESELECT_OEA) atomicOr(&ubase[mye >> 5], 1u << (mye & 31));
            if (mode == MOE_RESELECT_XSHARE || mode == MOE_RESELECT_XSHARE_HIER)
                atomicOr(&TMEMB[mye * BW + (b >> 5)], 1u << (b & 31));
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
        // rank the batch union by score (one warp per expert)
        for (int e = tid; e < E; e += blockDim.x)
            s_aff[e] = ((ubase[e >> 5] >> (e & 31)) & 1u) ? key_float_score(s_score[e], e) : 0ull;
        __syncthreads();
        int nbase = 0;
        for (int i = 0; i < E_MAX / 32; ++i) nbase += __popc(ubase[i]);
        const int Mp = a.budget < nbase ? a.budget : nbase;
#pragma unroll 1
        for (int e = warp; e < E; e += nwarps) {
            if (s_aff[e] == 0ull) continue;
            const int rank = warp_rank(s_aff, E, e, lane);
            if (lane == 0 && rank < Mp) atomicOr(&sbits[e >> 5], 1u << (e & 31));
        }
        __syncthreads();
    }

    // ---- hierarchical XShare.  Request level (one warp per request, a run
    // of `group` tokens): the request score of expert e sums the
    // probabilities of the request's tokens whose top-k holds e (tokens
    // ascending); the request picks its k best experts (score > 0; ties to
    // the lower index).  Batch level: the batch score sums the request
    // scores of the requests that picked e (requests ascending), and the
    // batch set is the first min(budget, |picked|) picked experts by it.
    if (mode == MOE_RESELECT_XSHARE_HIER) {
        const int G = a.group;
        const int nreq = (B + G - 1) / G;
        for (int i = tid; i < E * BW; i += blockDim.x) RPICK[i] = 0u;
        __syncthreads();
#pragma unroll 1
        for (int r = warp; r < nreq; r += nwarps) {
            const int bb = r * G, be = min(B, bb + G);
            unsigned o[NI];
            unsigned cand = 0u;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int e = lane + 32 * i;
                float sc = 0.0f;
                if (e < E)
                    for (int b = bb; b < be; ++b)
                        if ((TMEMB[e * BW + (b >> 5)] >> (b & 31)) & 1u)
                            sc = __fadd_rn(sc, prob_rows[static_cast<size_t>(b) * E + e]);
                o[i] = ord_of(sc);
                if (sc > 0.0f) cand |= 1u << i;
            }
#pragma unroll 1
            for (int j = 0; j < k; ++j) {
                const int e = warp_argmax<NI>(o, cand, lane);
                if (e < 0) break;
                if ((e & 31) == lane) atomicOr(&RPICK[e * BW + (r >> 5)], 1u << (r & 31));
            }
        }
        __syncthreads();
        bool picked = false;
        if (tid < E) {
            float sc = 0.0f;
#pragma unroll 1
            for (int r = 0; r < nreq; ++r) {
                if (!((RPICK[tid * BW + (r >> 5)] >> (r & 31)) & 1u)) continue;
                picked = true;
                float sr = 0.0f;
                const int bb = r * G, be = min(B, bb + G);
                for (int b = bb; b < be; ++b)
                    if ((TMEMB[tid * BW + (b >> 5)] >> (b & 31)) & 1u)
                        sr = __fadd_rn(sr, prob_rows[static_cast<size_t>(b) * E + tid]);
                sc = __fadd_rn(sc, sr);
            }
            s_aff[tid] = picked ? key_float_score(sc, tid) : 0ull;
        }
        const int npicked = __syncthreads_count(picked ? 1 : 0);
        const int Mp = a.budget < npicked ? a.budget : npicked;
#pragma unroll 1
        for (int e = warp; e < E; e += nwarps) {
            if (s_aff[e] == 0ull) continue;
            const int rank = warp_rank(s_aff, E, e, lane);
            if (lane == 0 && rank < Mp) atomicOr(&sbits[e >> 5], 1u << (e & 31));
        }
        __syncthreads();
    }

    // ---- affinity binning: the critical set = the shortest prefix of the
    // score order (score descending, ties to the lower index), at least k
    // long, that holds every token's rank-0 expert
    if (mode == MOE_RESELECT_AFFINITY) {
        for (int e = tid; e < E; e += blockDim.x)
            s_aff[e] = ((ubase[e >> 5] >> (e & 31)) & 1u) ? key_int_score(s_aff[e], e) : 0ull;
        __syncthreads();
#pragma unroll 1
        for (int e = warp; e < E; e += nwarps) {
            if (s_aff[e] == 0ull) continue;
            const int pos = warp_rank(s_aff, E, e, lane);
            if (lane == 0) {
                s_pos[e] = pos;
                if ((r0bits[e >> 5] >> (e & 31)) & 1u) atomicMax(&s_M, pos + 1);
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += blockDim.x)
            if (s_aff[e] != 0ull && s_pos[e] < s_M) atomicOr(&sbits[e >> 5], 1u << (e & 31));
        __syncthreads();
    }

    // ---- the activated set is now fixed: OEA = union of kept sets, XShare
    // and hierarchical XShare = the batch set, affinity binning = the
    // critical set, NONE = union of top-k sets.  Map experts to active slots
    // for the dense weights.
    const unsigned *abits = (mode == MOE_RESELECT_OEA) ? ukept : (mode == MOE_RESELECT_NONE ? ubase : sbits);
    if (a.publish_set && a.ctr != nullptr) {
        // every copy's mask, then (release) its count
        for (int i = tid; i < PUB_COPIES * (E_MAX / 32); i += blockDim.x) {
            const unsigned m = abits[i % (E_MAX / 32)];
            if (m != 0u) atomicOr(&a.ctr->pubs[i / (E_MAX / 32)].mask[i % (E_MAX / 32)], m);
        }
        __syncthreads();
        if (tid < PUB_COPIES) {
            __threadfence();
            asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(&a.ctr->pubs[tid].pub), "r"(1) : "memory");
        }
    }
    if (dense_w) {
        if (warp == 0) {
            const unsigned word = lane < E_MAX / 32 ? abits[lane] : 0u;
            int incl = __popc(word);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(FULL, incl, o);
                if (lane >= o) incl += u;
            }
            int pos = incl - __popc(word);
            for (int bit = 0; bit < 32; ++bit) {
                const int e = 32 * lane + bit;
                if (e >= E) break;
                s_rank[e] = ((word >> bit) & 1u) ? pos++ : -1;
            }
            const int na = __shfl_sync(FULL, incl, 31);
            if (lane == 0) s_nact = na;
        }
        __syncthreads();
    }

    // ---- phase 2: OEA fills / XShare top-k within the batch set; weights
    if (mode != MOE_RESELECT_NONE) {
#pragma unroll 1
        for (int b = warp; b < B; b += nwarps) {
            float l[NI], p[NI];
            unsigned ord[NI];
            load_row_any<NI>(logit_rows + static_cast<size_t>(b) * E, E, lane, l);
            load_row_any<NI>(prob_rows + static_cast<size_t>(b) * E, E, lane, p);
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
            const float myw = mye >= 0 ? __fdiv_rn(myp, sum) : 0.0f;
            if (lane < k) {
                a.sel_idx[static_cast<size_t>(b) * k + lane] = mye;
                a.sel_w[static_cast<size_t>(b) * k + lane] = myw;
                if (mye >= 0) atomicOr(&ASSIGN[mye * BW + (b >> 5)], 1u << (b & 31));
            }
            if (dense_w) write_dense_weights(a.wd, B, b, s_nact, s_rank, mye, myw, k, lane);
        }
    } else if (dense_w) {
#pragma unroll 1
        for (int b = warp; b < B; b += nwarps) {
            const int mye = lane < k ? a.sel_idx[static_cast<size_t>(b) * k + lane] : -1;
            const float myw = lane < k ? a.sel_w[static_cast<size_t>(b) * k + lane] : 0.0f;
            write_dense_weights(a.wd, B, b, s_nact, s_rank, mye, myw, k, lane);
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
}

constexpr int GEMV_TPB_MAX = 4;
constexpr int GEMV_EPB_MAX = 4;
constexpr size_t GEMV_SMEM_MAX = 160u * 1024u;
// drain limit: how long a block that gave up on its staged rows still lets
// them land before it exits
constexpr unsigned long long GEMV_WAIT_LIMIT_NS = 1000000000ull;  // 1 s

__device__ __forceinline__ unsigned smem_addr(const void *p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool bar_try_wait0(unsigned long long *bar) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar))
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void tma_rows(void *dst, const CUtensorMap *map, int line, unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(0), "r"(line), "r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ float comp(const float4 &v, int u) {
    return u == 0 ? v.x : u == 1 ? v.y : u == 2 ? v.z : v.w;
}

// Layer path: x -> bf16 copy for the expert kernel (when xb is non-null),
// y = 0, or y = x for a residual layer whose experts add on top of its
// input (grid-stride over the blocks of the launch).
__device__ void layer_prep(const float *__restrict__ x, int B, int d, uint16_t *__restrict__ xb,
                           float *__restrict__ y, bool residual) {
    const int n4 = B * d / 4;
    const int nblocks = gridDim.x * gridDim.y;
    const int nthreads = nblocks * blockDim.x;
    for (int i = (blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += nthreads) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(x) + i);
        const unsigned lo = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x))) |
                            (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
        const unsigned hi = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.z))) |
                            (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.w))) << 16);
        if (xb) reinterpret_cast<uint2 *>(xb)[i] = make_uint2(lo, hi);
        reinterpret_cast<float4 *>(y)[i] = residual ? v : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// Dot products of one Wg row (wrow) with nb <= 4 token rows (xrows, stride
// row_bytes), all in staged, swizzled shared memory.  One 256-column chunk
// per iteration (a short loop body: this code runs once per call, so its
// instruction fetch is on the critical path).  FULL: every chunk is
// complete (d % 256 == 0).
template <bool FULL>
__device__ __forceinline__ void gemv_rows(const unsigned char *wrow, const unsigned char *xrows, int row_bytes,
                                          int d, int nb, int lane, float (&acc)[GEMV_TPB_MAX]) {
    // byte offsets of this lane's two halves within a 1024-byte chunk: line
    // lane / 4, 16-byte units 2 (lane % 4) and 2 (lane % 4) + 1, swizzled
    const int line = lane >> 2;
    const int o0 = line * 128 + (((2 * (lane & 3)) ^ line) << 4);
    const int o1 = line * 128 + (((2 * (lane & 3) + 1) ^ line) << 4);
    const int nch = (d + 255) >> 8;
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
        if (!FULL && 256 * c + 8 * lane >= d) continue;
        const float4 w0 = *reinterpret_cast<const float4 *>(wrow + c * 1024 + o0);
        const float4 w1 = *reinterpret_cast<const float4 *>(wrow + c * 1024 + o1);
        float4 xa[GEMV_TPB_MAX], xc[GEMV_TPB_MAX];
#pragma unroll
        for (int t = 0; t < GEMV_TPB_MAX; ++t) {
            if (t < nb) {
                xa[t] = *reinterpret_cast<const float4 *>(xrows + t * row_bytes + c * 1024 + o0);
                xc[t] = *reinterpret_cast<const float4 *>(xrows + t * row_bytes + c * 1024 + o1);
            } else {
                xa[t] = xc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int t = 0; t < GEMV_TPB_MAX; ++t) acc[t] = __fmaf_rn(comp(xa[t], u), comp(w0, u), acc[t]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int t = 0; t < GEMV_TPB_MAX; ++t) acc[t] = __fmaf_rn(comp(xc[t], u), comp(w1, u), acc[t]);
    }
}

// ------------------------------------------------------- host helpers --
// Logits a lane holds for E experts (e = lane + 32 i, i < NI): 1, 2, 4 or 8.
inline int ni_for(int E) { return E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8; }

// Dynamic shared memory of the selection for d and r; sets *cache_rows when
// the B x E logits and probabilities fit beside the rest (96 KB).
inline size_t reselect_smem(const moe_dims_t &d, const moe_reselect_t &r, int *cache_rows) {
    const int BW = (d.B + 31) / 32;
    const size_t picks = r.mode == MOE_RESELECT_XSHARE_HIER ? static_cast<size_t>(d.E) * BW * 4 : 0;
    const size_t base = static_cast<size_t>(d.B) * d.k * 4 + static_cast<size_t>(d.E) * BW * 8 + picks;
    const size_t rows = static_cast<size_t>(d.B) * d.E * 8;
    *cache_rows = (base + rows <= 96u * 1024u) ? 1 : 0;
    return base + (*cache_rows ? rows : 0);
}

// Selection arguments (no workspace counters, no dense weights, no
// publication; callers set those).
inline ReselectArgs make_reselect_args(const float *logits, float *probs, bool fuse_softmax, const moe_dims_t &d,
                                       const moe_reselect_t &r, int32_t *sel_idx, float *sel_w,
                                       const moe_lists_t &l, int32_t *n_active_copy) {
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
    a.group = r.mode == MOE_RESELECT_XSHARE_HIER ? r.group : 1;
    a.sel_idx = sel_idx;
    a.sel_w = sel_w;
    a.lists = l;
    a.n_active_copy = n_active_copy;
    a.ctr = nullptr;
    a.wd = nullptr;
    a.cache_rows = 0;
    a.publish_set = 0;
    return a;
}

}  // namespace
}  // namespace moe
