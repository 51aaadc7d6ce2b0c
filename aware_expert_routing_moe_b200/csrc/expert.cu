// Grouped SwiGLU expert kernel (sm_100a) and its input preparation.
//
// Streams only the activated experts' bf16 weights from HBM, each byte once
// per call: decode is bandwidth-bound and its latency follows the number of
// distinct activated experts ("Lynx: Enabling Efficient MoE Inference
// through Dynamic Batch-Aware Expert Selection", section 1; "Opportunistic
// Expert Activation: Batch-Aware Expert Routing for Faster Decode Without
// Retraining", abstract).
//
// Work units, handed out by an atomic ticket to persistent CTAs (one per SM):
//   GU unit (expert e, token tile, 16-row block of d_ff):
//       g = Wgate[e][rows] x_t, u = Wup[e][rows] x_t over all of d,
//       h = silu(g) * u -> H scratch (bf16, [pair][d_ff]);
//   D unit (expert e, token tile, 64-row block of d):
//       y[t][rows] += w_t * Wdown[e][rows] h_t over all of d_ff.
// All GU units come before all D units in ticket order; a D unit's producer
// waits (bounded) until its expert's GU units are counted done.
//
// Per CTA: one producer warp issues TMA tensor copies (128B-swizzled weight
// boxes, H boxes) and bulk copies (token rows of x) into a ring of stages,
// each guarded by a full/empty mbarrier pair; four consumer warps run
// mma.sync m16n8k16 bf16 tiles with the weights as the 16-row A operand and
// up to 32 tokens as the B operand (tokens padded to 8-column tiles), fp32
// accumulation.  Every wait is bounded by a time limit; on expiry the CTA
// records an error code in the workspace, drains its in-flight copies and
// returns.
#include <cuda_bf16.h>

#include "internal.h"

namespace moe {
namespace {

constexpr int NCW = 4;                    // consumer warps
constexpr int NTHREADS = (NCW + 1) * 32;  // + one producer warp
constexpr int TN = 32;                    // tokens per tile
constexpr int GU_ROWS = 16;               // rows of Wgate and of Wup per GU unit
constexpr int GU_KC = 256;                // d elements per GU stage
constexpr int D_ROWS = 64;                // rows of Wdown per D unit
constexpr int D_KC = 128;                 // d_ff elements per D stage
constexpr int STAGES = 6;
constexpr int W_BYTES = 16384;            // weight bytes per stage (both kinds)
constexpr int XROW_BYTES = GU_KC * 2 + 16;  // padded token row of x in a GU stage
constexpr int OP_BYTES = 17408;           // operand region: >= TN * XROW_BYTES, 1 KiB multiple
constexpr int SLOT_BYTES = W_BYTES + OP_BYTES;
constexpr int PART_FLOATS = NCW * 2 * 16 * TN;  // GU partial sums for the epilogue
constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * SLOT_BYTES + PART_FLOATS * 4 + 4096;
static_assert(TN * XROW_BYTES <= OP_BYTES, "x tile does not fit");
static_assert(2 * TN * 128 <= OP_BYTES, "H tile does not fit");
static_assert(SLOT_BYTES % 1024 == 0, "slots must keep 1 KiB alignment for 128B swizzle");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;  // 1 s

enum : int { UNIT_GU = 0, UNIT_D = 1, UNIT_END = 2 };

struct StageHdr {
    int type, e, i_act, p0, n, row0, s, ns;
};

struct SharedCtl {
    unsigned long long full[STAGES];
    unsigned long long empty[STAGES];
    StageHdr hdr[STAGES];
    volatile int abort_flag;
    volatile int consumed;
    int n_active, total_tiles;
    int tile_start[E_MAX + 1];
};

struct ExpertArgs {
    const uint16_t *xb;
    int B, d, E, k, F;
    const int32_t *n_active, *active, *offsets, *tok;
    const float *w;
    float *y;
    uint16_t *h;
    Counters *ctr;
};

// ---------------------------------------------------------------- PTX --
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(unsigned long long *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(unsigned long long *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, unsigned bytes,
                                          unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<unsigned long long>(map)) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory"); }

// address of (row r, 16-byte chunk c) in a 128B-swizzled box with 128-byte rows
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int c) {
    return base + r * 128 + ((c ^ (r & 7)) << 4);
}

__device__ void record_error(Counters *ctr, SharedCtl *ctl, int code) {
    atomicCAS(&ctr->error, 0, code);
    ctl->abort_flag = 1;
}

// Bounded wait on an mbarrier phase; false if the CTA aborted or the time
// limit expired (the latter records `code`).
__device__ bool wait_phase(unsigned long long *bar, unsigned parity, SharedCtl *ctl, Counters *ctr,
                           int code) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (ctl->abort_flag) return false;
        if (global_ns() - t0 > WAIT_LIMIT_NS) {
            record_error(ctr, ctl, code);
            return false;
        }
    }
}

// ------------------------------------------------------------ producer --
struct UnitInfo {
    int type, e, i_act, p0, n, row0, ns, need;
};

__device__ UnitInfo decode_unit(int u, const ExpertArgs &a, const SharedCtl *ctl) {
    UnitInfo ui;
    const int gu_per_tile = a.F / GU_ROWS;
    const int d_per_tile = a.d / D_ROWS;
    const int n_gu = ctl->total_tiles * gu_per_tile;
    int tile, blk;
    if (u < n_gu) {
        ui.type = UNIT_GU;
        tile = u / gu_per_tile;
        blk = u % gu_per_tile;
        ui.row0 = blk * GU_ROWS;
        ui.ns = (a.d + GU_KC - 1) / GU_KC;
    } else {
        ui.type = UNIT_D;
        const int v = u - n_gu;
        tile = v / d_per_tile;
        blk = v % d_per_tile;
        ui.row0 = blk * D_ROWS;
        ui.ns = (a.F + D_KC - 1) / D_KC;
    }
    // active expert owning this tile: largest i with tile_start[i] <= tile
    int lo = 0, hi = ctl->n_active - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ctl->tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int i = lo;
    const int tt = tile - ctl->tile_start[i];
    const int off0 = __ldg(a.offsets + i), off1 = __ldg(a.offsets + i + 1);
    ui.i_act = i;
    ui.e = __ldg(a.active + i);
    ui.p0 = off0 + tt * TN;
    ui.n = min(TN, off1 - ui.p0);
    ui.need = (ctl->tile_start[i + 1] - ctl->tile_start[i]) * gu_per_tile;
    return ui;
}

__device__ void producer(const ExpertArgs &a, const ExpertMaps &m, SharedCtl *ctl, unsigned char *slots) {
    const int lane = threadIdx.x & 31;
    const int n_units = ctl->total_tiles * (a.F / GU_ROWS + a.d / D_ROWS);
    int g = 0;  // stages issued
    bool ok = true;
    for (;;) {
        int u = 0;
        if (lane == 0) u = atomicAdd(&a.ctr->ticket, 1);
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= n_units) break;
        const UnitInfo ui = decode_unit(u, a, ctl);
        bool dep_ready = (ui.type == UNIT_GU);
        for (int s = 0; s < ui.ns && ok; ++s, ++g) {
            const int slot = g % STAGES;
            if (g >= STAGES) {
                if (!wait_phase(&ctl->empty[slot], ((g / STAGES) - 1) & 1, ctl, a.ctr, DEV_TIMEOUT_EMPTY)) {
                    ok = false;
                    break;
                }
            }
            unsigned char *wdst = slots + slot * SLOT_BYTES;
            unsigned char *odst = wdst + W_BYTES;
            int kvalid, nbox;
            unsigned bytes;
            if (ui.type == UNIT_GU) {
                const int k0 = s * GU_KC;
                kvalid = min(GU_KC, a.d - k0);
                nbox = kvalid / 64;
                bytes = 2u * nbox * (GU_ROWS * 128) + static_cast<unsigned>(ui.n) * kvalid * 2u;
            } else {
                const int k0 = s * D_KC;
                kvalid = min(D_KC, a.F - k0);
                nbox = kvalid / 64;
                bytes = nbox * (D_ROWS * 128u) + nbox * (TN * 128u);
            }
            if (lane == 0) {
                StageHdr &h = ctl->hdr[slot];
                h.type = ui.type;
                h.e = ui.e;
                h.i_act = ui.i_act;
                h.p0 = ui.p0;
                h.n = ui.n;
                h.row0 = ui.row0;
                h.s = s;
                h.ns = ui.ns;
                mbar_expect_tx(&ctl->full[slot], bytes);
            }
            __syncwarp();
            if (ui.type == UNIT_GU) {
                const int k0 = s * GU_KC;
                const int grow = ui.e * a.F + ui.row0;
                if (lane < nbox) {
                    tma_load_2d(wdst + lane * (GU_ROWS * 128), &m.gate, k0 + 64 * lane, grow, &ctl->full[slot]);
                    tma_load_2d(wdst + 8192 + lane * (GU_ROWS * 128), &m.up, k0 + 64 * lane, grow,
                                &ctl->full[slot]);
                }
                if (lane < ui.n) {
                    const int t = __ldg(a.tok + ui.p0 + lane);
                    bulk_load(odst + lane * XROW_BYTES, a.xb + static_cast<size_t>(t) * a.d + k0,
                              static_cast<unsigned>(kvalid) * 2u, &ctl->full[slot]);
                }
            } else {
                const int k0 = s * D_KC;
                if (lane < nbox)
                    tma_load_2d(wdst + lane * (D_ROWS * 128), &m.down, k0 + 64 * lane, ui.e * a.d + ui.row0,
                                &ctl->full[slot]);
                if (!dep_ready) {
                    // gate/up of this expert must be complete before its H is read
                    if (lane == 0) {
                        const unsigned long long t0 = global_ns();
                        while (ld_acquire(&a.ctr->gu_done[ui.i_act]) < ui.need) {
                            if (ctl->abort_flag) { ok = false; break; }
                            if (global_ns() - t0 > WAIT_LIMIT_NS) {
                                record_error(a.ctr, ctl, DEV_TIMEOUT_DEP);
                                ok = false;
                                break;
                            }
                            __nanosleep(128);
                        }
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    dep_ready = true;
                }
                if (ok && lane < nbox)
                    tma_load_2d(odst + lane * (TN * 128), &m.h, k0 + 64 * lane, ui.p0, &ctl->full[slot]);
                if (!ok) { ++g; break; }
            }
        }
        if (!ok) break;
    }
    if (ok) {
        // end marker for the consumers
        const int slot = g % STAGES;
        if (g >= STAGES && !wait_phase(&ctl->empty[slot], ((g / STAGES) - 1) & 1, ctl, a.ctr, DEV_TIMEOUT_EMPTY))
            ok = false;
        if (ok && lane == 0) {
            ctl->hdr[slot].type = UNIT_END;
            mbar_arrive(&ctl->full[slot]);
        }
    }
    if (!ok && lane == 0) {
        // drain copies still in flight before the CTA's shared memory goes away
        for (int q = ctl->consumed; q < g; ++q) {
            const unsigned long long t0 = global_ns();
            while (!mbar_try_wait(&ctl->full[q % STAGES], (q / STAGES) & 1)) {
                if (global_ns() - t0 > WAIT_LIMIT_NS) break;
            }
        }
    }
}

// ------------------------------------------------------------ consumers --
template <int NT>
__device__ __forceinline__ void gu_stage(uint32_t wbase, uint32_t xbase, int kvalid, int warp, int lane,
                                         float (&acc_g)[4][4], float (&acc_u)[4][4]) {
    const int nks = kvalid / 16;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int ks = warp + NCW * q;
        if (ks >= nks) break;
        const int box = ks >> 2;
        const int chunk = ((ks & 3) << 1) + (lane >> 4);
        const int r = lane & 15;
        uint32_t g0, g1, g2, g3, u0, u1, u2, u3;
        ldsm_x4(swz(wbase + box * (GU_ROWS * 128), r, chunk), g0, g1, g2, g3);
        ldsm_x4(swz(wbase + 8192 + box * (GU_ROWS * 128), r, chunk), u0, u1, u2, u3);
        const int xk = ks * 16 + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int np = 0; np < (NT + 1) / 2; ++np) {
            const int n = np * 16 + (lane & 7) + ((lane >> 4) << 3);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(xbase + n * XROW_BYTES + xk * 2, b0, b1, b2, b3);
            mma_bf16(acc_g[2 * np], g0, g1, g2, g3, b0, b1);
            mma_bf16(acc_u[2 * np], u0, u1, u2, u3, b0, b1);
            if (2 * np + 1 < NT) {
                mma_bf16(acc_g[2 * np + 1], g0, g1, g2, g3, b2, b3);
                mma_bf16(acc_u[2 * np + 1], u0, u1, u2, u3, b2, b3);
            }
        }
    }
}

template <int NT>
__device__ __forceinline__ void d_stage(uint32_t wbase, uint32_t hbase, int kvalid, int warp, int lane,
                                        float (&acc)[4][4]) {
    const int nks = kvalid / 16;
#pragma unroll
    for (int ks = 0; ks < D_KC / 16; ++ks) {
        if (ks >= nks) break;
        const int box = ks >> 2;
        const int r = warp * 16 + (lane & 15);
        const int chunk = ((ks & 3) << 1) + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4(swz(wbase + box * (D_ROWS * 128), r, chunk), a0, a1, a2, a3);
        const int hchunk = ((ks & 3) << 1) + ((lane >> 3) & 1);
#pragma unroll
        for (int np = 0; np < (NT + 1) / 2; ++np) {
            const int n = np * 16 + (lane & 7) + ((lane >> 4) << 3);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(swz(hbase + box * (TN * 128), n, hchunk), b0, b1, b2, b3);
            mma_bf16(acc[2 * np], a0, a1, a2, a3, b0, b1);
            if (2 * np + 1 < NT) mma_bf16(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
    }
}

template <int NT>
__device__ __forceinline__ void stage_dispatch(const StageHdr &h, uint32_t wbase, uint32_t obase, const ExpertArgs &a,
                                               int warp, int lane, float (&acc_g)[4][4], float (&acc_u)[4][4]) {
    if (h.type == UNIT_GU) {
        gu_stage<NT>(wbase, obase, min(GU_KC, a.d - h.s * GU_KC), warp, lane, acc_g, acc_u);
    } else {
        d_stage<NT>(wbase, obase, min(D_KC, a.F - h.s * D_KC), warp, lane, acc_g);
    }
}

__device__ void consumer(const ExpertArgs &a, SharedCtl *ctl, unsigned char *slots, float *part) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ct = threadIdx.x;  // 0 .. NCW*32-1
    float acc_g[4][4], acc_u[4][4];
    for (int g = 0;; ++g) {
        const int slot = g % STAGES;
        if (!wait_phase(&ctl->full[slot], (g / STAGES) & 1, ctl, a.ctr, DEV_TIMEOUT_FULL)) return;
        const StageHdr h = ctl->hdr[slot];
        if (h.type == UNIT_END) return;
        if (h.s == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc_g[j][c] = acc_u[j][c] = 0.0f;
        }
        const uint32_t wbase = smem_u32(slots + slot * SLOT_BYTES);
        const uint32_t obase = wbase + W_BYTES;
        const int nt = (h.n + 7) >> 3;
        switch (nt) {
            case 1: stage_dispatch<1>(h, wbase, obase, a, warp, lane, acc_g, acc_u); break;
            case 2: stage_dispatch<2>(h, wbase, obase, a, warp, lane, acc_g, acc_u); break;
            case 3: stage_dispatch<3>(h, wbase, obase, a, warp, lane, acc_g, acc_u); break;
            default: stage_dispatch<4>(h, wbase, obase, a, warp, lane, acc_g, acc_u); break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->empty[slot]);
        if (ct == 0) ctl->consumed = g + 1;
        if (h.s != h.ns - 1) continue;

        // ---- unit epilogue
        const int row = lane >> 2, col = (lane & 3) * 2;
        if (h.type == UNIT_D) {
            const int i_base = h.row0 + warp * 16 + row;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j >= nt) break;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int n = j * 8 + col + (c & 1);
                    if (n < h.n) {
                        const int pair = h.p0 + n;
                        const int t = __ldg(a.tok + pair);
                        const float wt = __ldg(a.w + pair);
                        const int i = i_base + ((c >> 1) << 3);
                        atomicAdd(a.y + static_cast<size_t>(t) * a.d + i, wt * acc_g[j][c]);
                    }
                }
            }
        } else {
            // partial sums of this warp's k-steps -> shared, then reduce in a
            // fixed warp order and apply silu(g) * u
            float *pg = part + (warp * 2 + 0) * 16 * TN;
            float *pu = part + (warp * 2 + 1) * 16 * TN;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j >= nt) break;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int r = row + ((c >> 1) << 3);
                    const int n = j * 8 + col + (c & 1);
                    pg[r * TN + n] = acc_g[j][c];
                    pu[r * TN + n] = acc_u[j][c];
                }
            }
            consumer_bar();
            for (int idx = ct; idx < 16 * h.n; idx += NCW * 32) {
                const int r = idx & 15, n = idx >> 4;
                float gs = 0.0f, us = 0.0f;
#pragma unroll
                for (int wv = 0; wv < NCW; ++wv) {
                    gs += part[(wv * 2 + 0) * 16 * TN + r * TN + n];
                    us += part[(wv * 2 + 1) * 16 * TN + r * TN + n];
                }
                const float hv = gs / (1.0f + __expf(-gs)) * us;
                a.h[static_cast<size_t>(h.p0 + n) * a.F + h.row0 + r] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(hv));
            }
            __threadfence();
            asm volatile("fence.proxy.async.global;" ::: "memory");
            consumer_bar();
            if (ct == 0) {
                __threadfence();
                atomicAdd(&a.ctr->gu_done[h.i_act], 1);
            }
        }
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    expert_ffn_kernel(const __grid_constant__ ExpertMaps maps, const ExpertArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char *slots = base;
    float *part = reinterpret_cast<float *>(base + STAGES * SLOT_BYTES);
    SharedCtl *ctl = reinterpret_cast<SharedCtl *>(part + PART_FLOATS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], NCW);
        }
        ctl->abort_flag = 0;
        ctl->consumed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == NCW && lane == 0) {
        prefetch_tmap(&maps.gate);
        prefetch_tmap(&maps.up);
        prefetch_tmap(&maps.down);
        prefetch_tmap(&maps.h);
    }
    // everything above overlaps the re-selection kernel; the lists are read
    // only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == NCW) {
        // tile table: active expert i owns tiles [tile_start[i], tile_start[i+1])
        const int na = *a.n_active;
        int run = 0;
        for (int base_i = 0; base_i < na; base_i += 32) {
            const int i = base_i + lane;
            int nt = 0;
            if (i < na) nt = (__ldg(a.offsets + i + 1) - __ldg(a.offsets + i) + TN - 1) / TN;
            int incl = nt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (i < na) ctl->tile_start[i] = run + incl - nt;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            ctl->tile_start[na] = run;
            ctl->n_active = na;
            ctl->total_tiles = (na > 0 && na <= a.E) ? run : 0;
            if (na < 0 || na > a.E) atomicCAS(&a.ctr->error, 0, DEV_BAD_LISTS);
        }
    }
    __syncthreads();
    if (warp == NCW) {
        producer(a, maps, ctl, slots);
    } else {
        consumer(a, ctl, slots, part);
    }
}

// ------------------------------------------------------------------ prep --
__global__ void __launch_bounds__(256) ffn_prep_kernel(const float *__restrict__ x, int n4, uint16_t *__restrict__ xb,
                                                       float *__restrict__ y, Counters *ctr) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(x) + i);
        const unsigned lo = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x))) |
                            (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
        const unsigned hi = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.z))) |
                            (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.w))) << 16);
        reinterpret_cast<uint2 *>(xb)[i] = make_uint2(lo, hi);
        reinterpret_cast<float4 *>(y)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) ctr->ticket = 0;
        for (int i = threadIdx.x; i < E_MAX; i += blockDim.x) ctr->gu_done[i] = 0;
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

int g_num_sms[64] = {0};

}  // namespace

int expert_ffn_h_rows() { return TN; }

cudaError_t launch_ffn_prep(const float *x, const moe_dims_t &d, uint16_t *xb, float *y, Counters *ctr,
                            cudaStream_t s) {
    const int n4 = d.B * d.d / 4;
    const int blocks = (n4 + 255) / 256 > 0 ? min((n4 + 255) / 256, 1024) : 1;
    ffn_prep_kernel<<<blocks, 256, 0, s>>>(x, n4, xb, y, ctr);
    return cudaGetLastError();
}

cudaError_t launch_expert_ffn(const ExpertMaps &maps, const uint16_t *xb, const moe_dims_t &d,
                              const moe_lists_t &l, float *y, uint16_t *h, Counters *ctr, bool pdl,
                              cudaStream_t s) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (g_num_sms[dev] == 0) {
        int n = 0;
        err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(expert_ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (err != cudaSuccess) return err;
        g_num_sms[dev] = n;
    }
    ExpertArgs a;
    a.xb = xb;
    a.B = d.B;
    a.d = d.d;
    a.E = d.E;
    a.k = d.k;
    a.F = d.d_ff;
    a.n_active = l.n_active;
    a.active = l.active;
    a.offsets = l.offsets;
    a.tok = l.tok;
    a.w = l.w;
    a.y = y;
    a.h = h;
    a.ctr = ctr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g_num_sms[dev]);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, expert_ffn_kernel, maps, a);
}

}  // namespace moe
