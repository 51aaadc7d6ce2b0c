// Per-token channel top-k inside the activated experts (sm_100a).
//
// "Channel Selection for Mixture-of-Experts Decoding Needs No Calibration
// Data", methodology: a channel selector is a score plus a keep rule; the
// top-k keep rule takes each token's c highest-scoring channels of an
// expert, and the reads it saves are counted in 32-byte sectors.  Channel f
// of expert e is gate row f, up row f and down column f; the scores come
// from the caller (any selector).
//
// Decode with a handful of tokens is GEMV-shaped (at most a few tokens share
// a channel), so these kernels use no tensor cores.  Three kernels:
//   channel_select_kernel : one warp per (token, slot) pair: radix select of
//       the c-th largest score image, then the keep mask (equal scores to the
//       lower channel index); also zeroes y;
//   channel_items_kernel  : one CTA: the activated experts (ascending), each
//       expert's pairs, the union of its pairs' kept channels, and the work
//       list of (expert slot, channel) items;
//   channel_stream_kernel : persistent CTAs stream each item's gate row, up
//       row and down row from the channel-major down copy -- three
//       contiguous 2 d-byte rows, one bulk copy each -- through a
//       shared-memory ring, compute h = silu(g) u for the pairs that keep the
//       channel and accumulate w h down_f into a per-CTA y in shared memory,
//       which is added to y once at the end.
// Every wait is bounded; on expiry a CTA records an error code and drains
// its copies before it exits.
#include <cstdint>
#include <cstring>

#include "internal.h"

namespace moe {
namespace {

constexpr int CH_WARPS = 8;
constexpr int CH_THREADS = CH_WARPS * 32;
constexpr int CH_STAGES_MAX = 4;
constexpr unsigned long long CH_DRAIN_NS = 1000000000ull;  // 1 s

// Workspace of the channel path (byte offsets, 256-byte aligned).
struct ChLayout {
    size_t ctr, keep, slot_e, slot_np, slot_pairs, items, total;
};
struct ChCounters {
    int32_t error;
    int32_t n_slots;
    int32_t n_items;
    int32_t pad[61];
};

size_t al256(size_t v) { return (v + 255) / 256 * 256; }

ChLayout ch_layout(const moe_dims_t &d) {
    ChLayout L;
    size_t o = 0;
    const size_t pairs = static_cast<size_t>(d.B) * d.k, words = static_cast<size_t>(d.d_ff) / 32;
    const size_t slots = static_cast<size_t>(d.E < d.B * d.k ? d.E : d.B * d.k);
    L.ctr = o;        o += al256(sizeof(ChCounters));
    L.keep = o;       o += al256(pairs * words * 4);
    L.slot_e = o;     o += al256(slots * 4);
    L.slot_np = o;    o += al256(slots * 4);
    L.slot_pairs = o; o += al256(slots * MOE_CHANNELS_B_MAX * 4);
    L.items = o;      o += al256(slots * static_cast<size_t>(d.d_ff) * 4);
    L.total = o;
    return L;
}

__device__ __forceinline__ unsigned long long ch_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ uint32_t ch_smem(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// Order-preserving unsigned image of a score (larger score -> larger
// image; -0 and +0 equal).
__device__ __forceinline__ unsigned score_ord(float v) {
    v = (v == 0.0f) ? 0.0f : v;
    const unsigned u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------- selection --
struct SelectArgs {
    const int32_t *sel_idx;
    const float *score;  // [B][k][F]
    int B, k, F, c, d;
    uint32_t *keep;      // [B][k][F/32] bit masks
    float *y;            // zeroed
};

// One warp per (token, slot) pair.  The c-th largest image T is found by a
// radix select (four passes of 8 bits, a 256-bin histogram per warp); the
// pair keeps every channel with image > T and, of those with image == T,
// the (c - #greater) with the lowest indices.
__global__ void __launch_bounds__(CH_THREADS) channel_select_kernel(SelectArgs a) {
    __shared__ unsigned hist[CH_WARPS][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the union kernel may launch now; it waits for this grid before reading
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // y = 0 (the stream kernel adds into it)
    const int n4 = a.B * a.d / 4;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x)
        reinterpret_cast<float4 *>(a.y)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int p = blockIdx.x * CH_WARPS + warp;
    if (p >= a.B * a.k) return;
    const int words = a.F / 32;
    uint32_t *km = a.keep + static_cast<size_t>(p) * words;
    if (a.sel_idx[p] < 0) {
        for (int w = lane; w < words; w += 32) km[w] = 0u;
        return;
    }
    const float *sc = a.score + static_cast<size_t>(p) * a.F;
    unsigned prefix = 0u, pmask = 0u;
    int need = a.c;  // channels still to place at or below the current prefix
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) hist[warp][i] = 0u;
        __syncwarp();
        for (int f = lane; f < a.F; f += 32) {
            const unsigned o = score_ord(__ldg(sc + f));
            if ((o & pmask) == prefix) atomicAdd(&hist[warp][(o >> shift) & 255u], 1u);
        }
        __syncwarp();
        // the bin holding the need-th largest image: scan from the top
        int chosen = 0, above = 0;
        if (lane == 0) {
            int run = 0;
            for (int bin = 255; bin >= 0; --bin) {
                const int h = static_cast<int>(hist[warp][bin]);
                if (run + h >= need) {
                    chosen = bin;
                    above = run;
                    break;
                }
                run += h;
            }
        }
        chosen = __shfl_sync(0xffffffffu, chosen, 0);
        above = __shfl_sync(0xffffffffu, above, 0);
        need -= above;
        prefix |= static_cast<unsigned>(chosen) << shift;
        pmask |= 255u << shift;
        __syncwarp();
    }
    // prefix = T; `need` channels with image == T are kept, lowest index first
    int taken = 0;
    for (int base = 0; base < a.F; base += 32) {
        const int f = base + lane;
        const unsigned o = score_ord(__ldg(sc + f));
        const unsigned eq = __ballot_sync(0xffffffffu, o == prefix);
        const int rank = __popc(eq & ((1u << lane) - 1u));
        const bool kept = o > prefix || (o == prefix && taken + rank < need);
        const unsigned m = __ballot_sync(0xffffffffu, kept);
        if (lane == 0) km[base / 32] = m;
        taken += __popc(eq);
    }
}

// ----------------------------------------------------------------- items --
struct ItemsArgs {
    const int32_t *sel_idx;
    int B, k, E, F;
    const uint32_t *keep;
    ChCounters *ctr;
    int32_t *slot_e, *slot_np, *slot_pairs;  // slot_pairs[slot][MOE_CHANNELS_B_MAX]
    int32_t *items;                          // (slot << 16) | channel
};

// One CTA of CH_THREADS threads.
__global__ void __launch_bounds__(CH_THREADS) channel_items_kernel(ItemsArgs a) {
    __shared__ unsigned s_emask[E_MAX / 32];
    __shared__ int s_nslots;
    __shared__ int s_part[CH_THREADS];
    const int t = threadIdx.x;
    const int pairs = a.B * a.k, words = a.F / 32;
    if (t < E_MAX / 32) s_emask[t] = 0u;
    // launched early (programmatic dependent launch): the keep masks are
    // complete once the selection grid has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();
    for (int p = t; p < pairs; p += blockDim.x) {
        const int e = a.sel_idx[p];
        if (e >= 0 && e < a.E) atomicOr(&s_emask[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (t < 32) {
        // activated experts in ascending order
        const unsigned wv = t < E_MAX / 32 ? s_emask[t] : 0u;
        int incl = __popc(wv);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (t >= o) incl += v;
        }
        int pos = incl - __popc(wv);
        for (int bit = 0; bit < 32; ++bit) {
            const int e = 32 * t + bit;
            if (e >= E_MAX) break;
            if ((wv >> bit) & 1u) a.slot_e[pos++] = e;
        }
        if (t == 31) s_nslots = incl;
    }
    __syncthreads();
    const int ns = s_nslots;
    // each slot's pairs, in pair order (token ascending)
    for (int i = t; i < ns; i += blockDim.x) {
        const int e = a.slot_e[i];
        int n = 0;
        for (int p = 0; p < pairs; ++p)
            if (a.sel_idx[p] == e && n < MOE_CHANNELS_B_MAX) a.slot_pairs[i * MOE_CHANNELS_B_MAX + n++] = p;
        a.slot_np[i] = n;
    }
    __syncthreads();
    // union of the kept channels per slot, then the items in (slot,
    // channel) order: thread t takes a contiguous run of the ns * words
    // union words, counts, and a block scan places its items
    const int total_w = ns * words;
    const int per = (total_w + blockDim.x - 1) / blockDim.x;
    const int w0 = t * per, w1 = min(total_w, w0 + per);
    int cnt = 0;
    for (int q = w0; q < w1; ++q) {
        const int i = q / words, w = q - i * words;
        unsigned u = 0u;
        for (int j = 0; j < a.slot_np[i]; ++j) u |= a.keep[static_cast<size_t>(a.slot_pairs[i * MOE_CHANNELS_B_MAX + j]) * words + w];
        cnt += __popc(u);
    }
    s_part[t] = cnt;
    __syncthreads();
    if (t == 0) {
        int run = 0;
        for (int i = 0; i < static_cast<int>(blockDim.x); ++i) {
            const int v = s_part[i];
            s_part[i] = run;
            run += v;
        }
        a.ctr->n_items = run;
        a.ctr->n_slots = ns;
    }
    __syncthreads();
    int pos = s_part[t];
    for (int q = w0; q < w1; ++q) {
        const int i = q / words, w = q - i * words;
        unsigned u = 0u;
        for (int j = 0; j < a.slot_np[i]; ++j) u |= a.keep[static_cast<size_t>(a.slot_pairs[i * MOE_CHANNELS_B_MAX + j]) * words + w];
        while (u != 0u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1u;
            a.items[pos++] = (i << 16) | (32 * w + bit);
        }
    }
}

// ---------------------------------------------------------------- stream --
struct StreamArgs {
    const float *x;          // [B][d]
    const uint16_t *Wgate, *Wup, *WdownT;  // [E][F][d] each (down channel-major)
    const int32_t *sel_idx;
    const float *sel_w;
    int B, k, F, d, stages;
    unsigned long long wait_ns;
    const uint32_t *keep;
    const ChCounters *ctr_ro;
    ChCounters *ctr;
    const int32_t *slot_e, *slot_np, *slot_pairs, *items;
    float *y;
};

__device__ __forceinline__ void ch_bulk(void *dst, const void *src, unsigned bytes, unsigned long long *bar,
                                        unsigned long long policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(ch_smem(dst)), "l"(src), "r"(bytes), "r"(ch_smem(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ bool ch_try_wait(unsigned long long *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(ch_smem(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Shared memory: x [B][d] fp32, the CTA's y [B][d] fp32, then the ring of
// stages, each gate row | up row | down row (2 d bytes each).
__global__ void __launch_bounds__(CH_THREADS, 1) channel_stream_kernel(StreamArgs a) {
    extern __shared__ __align__(128) unsigned char ch_raw[];
    __shared__ __align__(8) unsigned long long full[CH_STAGES_MAX];
    __shared__ float red[2][CH_WARPS][MOE_CHANNELS_B_MAX];
    __shared__ float s_h[MOE_CHANNELS_B_MAX];
    __shared__ int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = a.B, d = a.d;
    float *xs = reinterpret_cast<float *>(ch_raw);
    float *ys = xs + B * d;
    unsigned char *ring = reinterpret_cast<unsigned char *>(ys + B * d);
    const unsigned row_bytes = static_cast<unsigned>(d) * 2u;
    const unsigned stage_bytes = 3u * row_bytes;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(ch_smem(&full[s])) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
    }
    for (int i = threadIdx.x; i < B * d; i += blockDim.x) {
        xs[i] = __ldg(a.x + i);
        ys[i] = 0.0f;
    }
    // everything above overlaps the union kernel (programmatic dependent
    // launch); the items, the slots and y = 0 are complete once it (and the
    // selection before it) has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();
    const int n_items = a.ctr_ro->n_items;
    unsigned long long policy;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    auto issue = [&](int j, int slot) {
        const int it = a.items[j];
        const int si = it >> 16, f = it & 0xffff;
        const size_t row = static_cast<size_t>(a.slot_e[si]) * a.F + f;
        unsigned char *dst = ring + static_cast<size_t>(slot) * stage_bytes;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(ch_smem(&full[slot])),
                     "r"(stage_bytes)
                     : "memory");
        ch_bulk(dst, a.Wgate + row * d, row_bytes, &full[slot], policy);
        ch_bulk(dst + row_bytes, a.Wup + row * d, row_bytes, &full[slot], policy);
        ch_bulk(dst + 2 * row_bytes, a.WdownT + row * d, row_bytes, &full[slot], policy);
    };
    // this CTA's items: blockIdx.x, + gridDim.x, ...; up to `stages` in flight
    int issued = 0, done = 0;
    const int first = blockIdx.x, step = gridDim.x;
    const int mine = first < n_items ? (n_items - first + step - 1) / step : 0;
    if (threadIdx.x == 0)
        for (; issued < mine && issued < a.stages; ++issued) issue(first + issued * step, issued);
    for (; done < mine; ++done) {
        const int slot = done % a.stages;
        const unsigned parity = (done / a.stages) & 1;
        if (threadIdx.x == 0 && !ch_try_wait(&full[slot], parity)) {
            const unsigned long long t0 = ch_now();
            while (!ch_try_wait(&full[slot], parity)) {
                if (ch_now() - t0 > a.wait_ns) {
                    atomicCAS(&a.ctr->error, 0, DEV_TIMEOUT_FULL);
                    s_abort = 1;
                    break;
                }
            }
        }
        __syncthreads();
        if (s_abort) break;
        const int it = a.items[first + done * step];
        const int si = it >> 16, f = it & 0xffff;
        const int np = a.slot_np[si];
        const int words = a.F / 32;
        const uint32_t *g2 = reinterpret_cast<const uint32_t *>(ring + static_cast<size_t>(slot) * stage_bytes);
        const uint32_t *u2 = g2 + d / 2;
        const uint32_t *d2 = u2 + d / 2;
        // pairs of this expert that keep channel f
        int pk[MOE_CHANNELS_B_MAX];
        int nk = 0;
        for (int j = 0; j < np; ++j) {
            const int p = a.slot_pairs[si * MOE_CHANNELS_B_MAX + j];
            if ((a.keep[static_cast<size_t>(p) * words + (f >> 5)] >> (f & 31)) & 1u) pk[nk++] = p;
        }
        // g and u of each such pair's token: each thread takes element pairs
        // i = 2 t, 2 t + 1 (+ 2 CH_THREADS ...), warp sums, then CTA sums
        for (int j = 0; j < nk; ++j) {
            const float2 *xt = reinterpret_cast<const float2 *>(xs + (pk[j] / a.k) * d);
            float gs = 0.0f, us = 0.0f;
            for (int q = threadIdx.x; q < d / 2; q += blockDim.x) {
                const uint32_t gv = g2[q], uv = u2[q];
                const float2 xv = xt[q];
                const float x0 = xv.x, x1 = xv.y;
                gs = fmaf(bf16_lo(gv), x0, gs);
                gs = fmaf(bf16_hi(gv), x1, gs);
                us = fmaf(bf16_lo(uv), x0, us);
                us = fmaf(bf16_hi(uv), x1, us);
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                gs += __shfl_xor_sync(0xffffffffu, gs, o);
                us += __shfl_xor_sync(0xffffffffu, us, o);
            }
            if (lane == 0) {
                red[0][warp][j] = gs;
                red[1][warp][j] = us;
            }
        }
        __syncthreads();
        if (threadIdx.x < nk) {
            float g = 0.0f, u = 0.0f;
            for (int w = 0; w < CH_WARPS; ++w) {
                g += red[0][w][threadIdx.x];
                u += red[1][w][threadIdx.x];
            }
            const int p = pk[threadIdx.x];
            s_h[threadIdx.x] = a.sel_w[p] * (g / (1.0f + __expf(-g)) * u);
        }
        __syncthreads();
        // y_t += w h down_f for the pairs' tokens
        for (int j = 0; j < nk; ++j) {
            float2 *yt = reinterpret_cast<float2 *>(ys + (pk[j] / a.k) * d);
            const float hw = s_h[j];
            for (int q = threadIdx.x; q < d / 2; q += blockDim.x) {
                const uint32_t dv = d2[q];
                float2 v = yt[q];
                v.x = fmaf(hw, bf16_lo(dv), v.x);
                v.y = fmaf(hw, bf16_hi(dv), v.y);
                yt[q] = v;
            }
        }
        __syncthreads();  // the stage is consumed
        if (threadIdx.x == 0 && issued < mine) {
            issue(first + issued * step, issued % a.stages);
            ++issued;
        }
    }
    if (s_abort && threadIdx.x == 0) {
        // let the copies in flight land before the shared memory goes away
        for (int q = done; q < issued; ++q) {
            const unsigned long long t0 = ch_now();
            while (!ch_try_wait(&full[q % a.stages], (q / a.stages) & 1))
                if (ch_now() - t0 > CH_DRAIN_NS) break;
        }
    }
    __syncthreads();
    // add this CTA's y (tokens it touched) into y
    if (mine > 0 && !s_abort)
        for (int i = threadIdx.x; i < B * d / 4; i += blockDim.x) {
            const float4 v = reinterpret_cast<const float4 *>(ys)[i];
            if (v.x != 0.0f || v.y != 0.0f || v.z != 0.0f || v.w != 0.0f) {
                float *dst = a.y + 4 * i;
                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v.x), "f"(v.y),
                             "f"(v.z), "f"(v.w)
                             : "memory");
            }
        }
}

// ------------------------------------------------------------- transpose --
// WdownT[e][f][i] = Wdown[e][i][f]: 32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256) down_transpose_kernel(const uint16_t *Wdown, int d, int F, uint16_t *WdownT) {
    __shared__ uint16_t tile[32][33];
    const int e = blockIdx.z;
    const int i0 = blockIdx.y * 32, f0 = blockIdx.x * 32;
    const uint16_t *src = Wdown + static_cast<size_t>(e) * d * F;
    uint16_t *dst = WdownT + static_cast<size_t>(e) * F * d;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int r = ty; r < 32; r += 8) tile[r][tx] = src[static_cast<size_t>(i0 + r) * F + f0 + tx];
    __syncthreads();
    for (int r = ty; r < 32; r += 8) dst[static_cast<size_t>(f0 + r) * d + i0 + tx] = tile[tx][r];
}

int g_ch_sms[MAX_DEVICES] = {0};

}  // namespace

size_t channels_workspace_bytes(const moe_dims_t &d) { return ch_layout(d).total; }

int channels_stages(const moe_dims_t &d) {
    const size_t fixed = 2ull * d.B * d.d * 4;
    const size_t stage = 3ull * d.d * 2;
    const size_t budget = 200u * 1024u;
    if (fixed + 2 * stage > budget) return 0;
    const size_t s = (budget - fixed) / stage;
    return static_cast<int>(s < CH_STAGES_MAX ? s : CH_STAGES_MAX);
}

cudaError_t launch_down_transpose(const uint16_t *Wdown, const moe_dims_t &d, uint16_t *WdownT, cudaStream_t s) {
    dim3 grid(d.d_ff / 32, d.d / 32, d.E);
    down_transpose_kernel<<<grid, 256, 0, s>>>(Wdown, d.d, d.d_ff, WdownT);
    return cudaGetLastError();
}

cudaError_t launch_channels(const float *x, const uint16_t *Wgate, const uint16_t *Wup, const uint16_t *WdownT,
                            const moe_dims_t &d, const int32_t *sel_idx, const float *sel_w, const float *score,
                            int c, float *y, uint32_t *keep_out, void *ws, cudaStream_t s) {
    const ChLayout L = ch_layout(d);
    unsigned char *w = static_cast<unsigned char *>(ws);
    ChCounters *ctr = reinterpret_cast<ChCounters *>(w + L.ctr);
    uint32_t *keep = keep_out ? keep_out : reinterpret_cast<uint32_t *>(w + L.keep);
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    if (g_ch_sms[dev] == 0) {
        int n = 0;
        err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        g_ch_sms[dev] = n;
    }
    SelectArgs sa;
    sa.sel_idx = sel_idx;
    sa.score = score;
    sa.B = d.B;
    sa.k = d.k;
    sa.F = d.d_ff;
    sa.c = c;
    sa.d = d.d;
    sa.keep = keep;
    sa.y = y;
    channel_select_kernel<<<(d.B * d.k + CH_WARPS - 1) / CH_WARPS, CH_THREADS, 0, s>>>(sa);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ItemsArgs ia;
    ia.sel_idx = sel_idx;
    ia.B = d.B;
    ia.k = d.k;
    ia.E = d.E;
    ia.F = d.d_ff;
    ia.keep = keep;
    ia.ctr = ctr;
    ia.slot_e = reinterpret_cast<int32_t *>(w + L.slot_e);
    ia.slot_np = reinterpret_cast<int32_t *>(w + L.slot_np);
    ia.slot_pairs = reinterpret_cast<int32_t *>(w + L.slot_pairs);
    ia.items = reinterpret_cast<int32_t *>(w + L.items);
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(CH_THREADS);
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, channel_items_kernel, ia);
    if (err != cudaSuccess) return err;
    StreamArgs ta;
    ta.x = x;
    ta.Wgate = Wgate;
    ta.Wup = Wup;
    ta.WdownT = WdownT;
    ta.sel_idx = sel_idx;
    ta.sel_w = sel_w;
    ta.B = d.B;
    ta.k = d.k;
    ta.F = d.d_ff;
    ta.d = d.d;
    ta.stages = channels_stages(d);
    ta.wait_ns = wait_limit_ns();
    ta.keep = keep;
    ta.ctr_ro = ctr;
    ta.ctr = ctr;
    ta.slot_e = ia.slot_e;
    ta.slot_np = ia.slot_np;
    ta.slot_pairs = ia.slot_pairs;
    ta.items = ia.items;
    ta.y = y;
    const size_t smem = 2ull * d.B * d.d * 4 + static_cast<size_t>(ta.stages) * 3 * d.d * 2;
    static bool configured[MAX_DEVICES] = {};
    if (!configured[dev]) {
        err = cudaFuncSetAttribute(channel_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (err != cudaSuccess) return err;
        configured[dev] = true;
    }
    cfg.gridDim = dim3(g_ch_sms[dev]);
    cfg.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&cfg, channel_stream_kernel, ta);
}

}  // namespace moe
