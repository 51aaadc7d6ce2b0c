// Grouped SwiGLU expert kernel (sm_100a) and its input preparation.
//
// Streams only the activated experts' bf16 weights from HBM, each byte once
// per call: decode is bandwidth-bound and its latency follows the number of
// distinct activated experts ("Lynx: Enabling Efficient MoE Inference
// through Dynamic Batch-Aware Expert Selection", section 1; "Opportunistic
// Expert Activation: Batch-Aware Expert Routing for Faster Decode Without
// Retraining", abstract).
//
// Work units, dealt round robin to persistent CTAs (one per SM):
//   GU unit (expert e, token tile, 32 rows of d_ff; 16 on the warp-MMA path):
//       g = Wgate[e][rows] x_t, u = Wup[e][rows] x_t over all of d,
//       h = silu(g) * u -> H scratch (bf16);
//   D unit (expert e, token tile, 64-row block of d):
//       y[t][rows] += w_t * Wdown[e][rows] h_t over all of d_ff.
// Every CTA takes all its GU units before its D units; a D unit's producer
// waits (bounded) until its expert's GU units are published done.
//
// Dense mode (B <= 64): every unit works on all B tokens of the batch, so
// gate/up stages load x for all tokens in one swizzled box, H is indexed by
// (active slot, token), and the down epilogue weighs each token by a dense
// [slot][B] weight matrix (0 for tokens that did not choose the expert).
// Gate/up work then needs only the activated set, which the fused layer
// kernel has before the token lists exist: its CTAs rank the tokens' first
// experts themselves (OEA, plain top-k) or read the set the selection CTA
// publishes (the batch-wide rules), and start streaming at once.
// Larger batches (tile mode) use tiles of up to 64 (token, expert) pairs:
// the input preparation copies each pair's x row (bf16) into a pair-indexed
// buffer in the lists' order, so a tile's x rows are one swizzled box like
// H's, and the down epilogue weighs each pair by its list weight.
//
// Per CTA: one producer warp issues TMA tensor copies (boxes of 64-column
// chunks, 128-byte swizzle; a gate/up stage in one box of Wgate and Wup
// seen as one tensor) into a ring of 32 KB weight
// stages plus operand tiles, each guarded by a full/empty mbarrier pair.
// The math runs on the 5th-generation tensor cores: four issuer warps
// (one thread each) issue, per stage, tcgen05 MMAs of 64 weight rows (a
// gate/up chunk is 32 gate rows and the same 32 up rows) by the tile's
// token columns into partial TMEM accumulators, two buffers deep so that a
// unit's epilogue overlaps the next unit's MMAs; the MMA completion itself
// frees the stage.  Eight epilogue warps read the accumulators out (silu *
// u -> H, or weighted atomics into y) and publish gate/up completions.
// Batches of up to 8 tokens run the warp-MMA variant of the same roles
// instead: 16-row gate/up units, and eight consumer warps that do each
// stage's math with mma.sync and the epilogues themselves.
// Every wait is bounded by a time limit; on expiry the CTA records an error
// code in the workspace, drains its in-flight copies and MMAs and returns.
// The last CTA to finish puts the workspace counters of the call back to
// zero.
#include <cstring>
#include <mutex>

#include <cuda_bf16.h>

#include "internal.h"
#include "route_dev.cuh"
#include "tcgen05.cuh"

namespace moe {
namespace {

constexpr int NCW = 8;  // epilogue warps
// The MMAs are issued by NISSUE warps (one per SM sub-partition: a single
// thread issues at most about one tcgen05.mma per 165 cycles, whatever its
// shape, measured), each taking every NISSUE-th k-step of a stage into a
// partial accumulator of its own.
constexpr int NISSUE = 4;
constexpr int NTHREADS = (NCW + 1 + NISSUE) * 32;  // + one producer warp
constexpr int TN = 64;         // pairs per token tile (batches above 64 tokens)
constexpr int DENSE_MAX = 64;  // dense mode (every unit takes the whole batch) up to 64 tokens
// GU units of 32 gate rows and the same 32 up rows; a stage holds 4 chunks
// of 64 columns, each chunk as the gate tile [32][64] followed by the up
// tile [32][64], so that one chunk is a single 64-row MMA operand (1 KiB row
// groups throughout).
constexpr int UM_ROWS = 32;
constexpr int UM_CHUNKS = 4;
constexpr int UM_TILE = UM_ROWS * 128;       // one gate (or up) tile of a chunk
constexpr int UM_CHUNK_BYTES = 2 * UM_TILE;  // gate + up tiles of a chunk
constexpr int D_ROWS = 64;                   // rows of Wdown per D unit
constexpr int D_CHUNKS = 4;                  // 64-column chunks of d_ff per D stage (at most)
constexpr int MAX_STAGES = 5;
constexpr int W_BYTES = 32768;               // weight bytes per stage (both kinds)
// Ring shapes: stages of 32 KB of weights plus an operand region for the
// token rows of 4 chunks (x for gate/up, H for down): bpad rows in dense
// mode (8, 16 or 32 KB for up to 16, 32 or 64 tokens), 64 pair rows in tile
// mode; PARTB: the epilogue's accumulator copy, [rows][64] fp32.
template <int ST, int OPB, int PARTB>
struct Ring {
    static constexpr int STAGES = ST;
    static constexpr int OP_BYTES = OPB;
    static constexpr int SLOT_BYTES = W_BYTES + OPB;
    static constexpr int PART_BYTES = PARTB;
};
constexpr int CTL_BYTES = 6144;  // reserved for SharedCtl (checked below)
// The fused layer kernel adds static shared memory of its own (router and
// selection state, under 7 KB); the budget below keeps room for it.
constexpr int STATIC_SMEM_RESERVE = 7168;
template <class RG>
constexpr int smem_bytes() {
    return 1024 /*align slack*/ + RG::STAGES * RG::SLOT_BYTES + RG::PART_BYTES + CTL_BYTES;
}
using RingB16 = Ring<5, 8192, 16 * 64 * 4>;
using RingB32 = Ring<4, 16384, 32 * 64 * 4>;
using RingB64 = Ring<3, 32768, 64 * 64 * 4>;
// Batches of up to WM_MAX tokens that activate at most WM_ACTIVE_MAX
// experts take the warp-MMA path instead (mma.sync m16n8k16, the tokens one
// 8-column tile): its gate/up units are 16 rows, a stage the gate box
// [WM_CHUNKS][16 rows][64 cols] and the up box after it.  With so few
// tokens the work per weight byte is small enough for the warps, and the
// finer units spread the few activated experts over more CTAs; a 64-row
// tensor-core MMA cannot take a 16-row unit without reading rows it does
// not use.  With more experts the stream is long enough for 32-row units,
// and those are cheaper per byte (measured: at Qwen3-30B shape, 8 tokens,
// top-8 the warp-MMA path took 54 us against 51 us; with OEA k0 = 4, at
// most 32 experts, 35 us against 36 us).
constexpr int WM_MAX = 8;
constexpr int WM_ACTIVE_MAX = 32;
constexpr int WM_ROWS = 16;
constexpr int WM_CHUNKS = 8;
constexpr int WM_UP_OFF = WM_ROWS * 128 * WM_CHUNKS;  // the up box after the gate box
constexpr int SIG_SLOTS = 4;  // gate/up completions queued for the signal warp (warp-MMA path)
static_assert(2 * WM_UP_OFF == W_BYTES, "warp-MMA gate/up boxes must fill the weight region");
static_assert(WM_MAX * 128 * WM_CHUNKS <= RingB16::OP_BYTES, "warp-MMA x rows do not fit");
static_assert(4 * 2 * WM_ROWS * WM_MAX * 4 <= RingB16::PART_BYTES, "warp-MMA gate/up partial sums do not fit");
static_assert(UM_CHUNKS * UM_CHUNK_BYTES == W_BYTES, "gate/up chunks must fill the weight region");
static_assert(2 * UM_ROWS == UMMA_M && D_ROWS == UMMA_M && D_ROWS * 128 == UM_CHUNK_BYTES,
              "a gate/up chunk and a down chunk are one 64-row MMA operand each");
static_assert(16 * 128 * UM_CHUNKS <= RingB16::OP_BYTES && 32 * 128 * UM_CHUNKS <= RingB32::OP_BYTES &&
                  DENSE_MAX * 128 * UM_CHUNKS <= RingB64::OP_BYTES && DENSE_MAX * 128 * D_CHUNKS <= RingB64::OP_BYTES,
              "token rows do not fit");
static_assert(TN * 128 * UM_CHUNKS <= RingB64::OP_BYTES && TN * 64 * 4 <= RingB64::PART_BYTES,
              "tile mode uses the 64-row ring");
static_assert(D_ROWS * 128 * D_CHUNKS <= W_BYTES, "down tile does not fit");
static_assert(DENSE_MAX * 64 * 4 <= RingB64::PART_BYTES, "accumulator copy does not fit");
static_assert(RingB16::SLOT_BYTES % 1024 == 0 && RingB32::SLOT_BYTES % 1024 == 0 && RingB64::SLOT_BYTES % 1024 == 0,
              "slots must keep 1 KiB alignment for 128B swizzle");
static_assert(RingB16::STAGES <= MAX_STAGES && RingB32::STAGES <= MAX_STAGES && RingB64::STAGES <= MAX_STAGES,
              "too many stages");
static_assert(smem_bytes<RingB16>() + STATIC_SMEM_RESERVE <= 232448 &&
                  smem_bytes<RingB32>() + STATIC_SMEM_RESERVE <= 232448 &&
                  smem_bytes<RingB64>() + STATIC_SMEM_RESERVE <= 232448,
              "shared memory budget");

// Bounded waits: a wait on another CTA, another kernel or a copy gives up
// after the call's wait limit (ExpertArgs::wait_ns, 1 s unless the caller
// set another with moe_set_wait_limit_ns), records an error code and ends
// the CTA's work; copies already in flight into its shared memory are then
// drained, with a fixed limit, before the CTA exits.
constexpr unsigned long long DRAIN_LIMIT_NS = 1000000000ull;  // 1 s
constexpr int SPLIT_TABLE_MAX = 256;  // tile counts covered by the split table

enum : int { UNIT_GU = 0, UNIT_D = 1, UNIT_END = 2 };

struct StageHdr {
    int type, e, i_act, p0, n, row0, s, ns;
    int k;  // the stage's k-range (s, or k0 + s for a split down unit)
};

// One work unit, decoded: kind, expert id and active index, first pair and
// pair count of its token tile, first row, stage count, and (down units)
// the gate/up units of its expert that must be published first.
struct UnitRec {
    int type, e, i_act, p0, n, row0, ns, need;
    int k0;  // first k-range (split down units; 0 otherwise)
};
constexpr int UNIT_WINDOW = 32;  // units a producer decodes at once (one per lane)

// The unit an accumulator buffer holds (tensor-core path).
struct AccHdr {
    int type, i_act, row0, p0, n;
};

struct SharedCtl {
    unsigned long long wait_ns;  // limit of every bounded wait of this call
    unsigned long long full[MAX_STAGES];
    unsigned long long empty[MAX_STAGES];
    StageHdr hdr[MAX_STAGES];
    volatile int abort_flag;
    volatile int consumed;
    int n_active, total_tiles;
    int split;  // last-round down units cut into k-ranges
    int last_cta;
    int tile_start[E_MAX + 1];
    UnitRec urec[UNIT_WINDOW];  // the producer's decoded window of its own units
    int act_e[E_MAX];       // active expert ids (copied once per CTA)
    int off[E_MAX + 1];     // list offsets (copied once per CTA)
    // tensor-core path: accumulator buffers (TMEM columns 64 b ..) full /
    // released, completion of the MMAs issued, the unit each buffer holds
    unsigned long long acc_full[2];
    unsigned long long acc_empty[2];
    unsigned long long mma_done;
    AccHdr acc_hdr[2];
    uint32_t tmem;  // TMEM base address of the CTA's allocation
    volatile int epi_go, epi_lists;  // outcomes of the epilogue's waits (its thread 0)
    // warp-MMA path: outcome of a stage's wait (by stage parity); the
    // queue of gate/up completions the signal warp publishes
    volatile int wm_go[2];
    unsigned long long sig_full[SIG_SLOTS];
    unsigned long long sig_empty[SIG_SLOTS];
    int sig_iact[SIG_SLOTS];
};

static_assert(sizeof(SharedCtl) <= CTL_BYTES, "SharedCtl does not fit its reservation");

struct ExpertArgs {
    const uint16_t *xb;
    int B, d, E, k, F;
    unsigned long long wait_ns;  // limit of the bounded waits
    int unit_ctas;               // CTAs the work units are dealt to (0 .. unit_ctas-1)
    // early mode: the dense weights are ready once *lists_flag >= 1 (fused
    // layer kernel); null: once the previous kernel has completed
    const int32_t *lists_flag;
    // dense mode (B <= DENSE_MAX): every stage works on all B tokens; gate/up
    // stages load all token rows of x in one box, H is token-indexed
    // [slot][B][d_ff] and the down epilogue weighs tokens by wd[slot][B]
    int dense;
    int gu_rows;  // rows of Wgate / Wup per GU unit
    int gc;       // 64-column chunks of d per GU stage
    int bpad;   // B rounded up to a multiple of 8 (dense mode)
    int hrows;  // rows of one H box (bpad in dense mode, TN otherwise)
    int early;       // start when ctr->pubs[c].pub reaches pub_target, not at the previous kernel's end
    int pub_target;
    // host-computed unit geometry: gate/up and down units per tile, their
    // stage counts, and the reciprocals of the unit counts (dense decode)
    int gu_per_tile, d_per_tile, ns_gu, ns_d;
    float inv_gu, inv_d, inv_nsd;
    // last-round down units to cut into k-ranges, per total tile count
    unsigned char split_for[SPLIT_TABLE_MAX + 1];
    const float *wd;
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
// Adds to the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_add_tx(unsigned long long *bar, unsigned bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
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
// one box of a (chunk, row, chunk index) map: `nch` tiles of [rows][64]
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}
// The same for a tensor read once per call (the expert weights): marked
// evict-first in L2 so that the stream does not push out what the next call
// reuses (router weights, code, the small per-call buffers).
__device__ __forceinline__ unsigned long long evict_first_policy() {
    unsigned long long p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_3d_stream(void *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                                   unsigned long long *bar, unsigned long long policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// one box of the 4-D gate/up map (both matrices of a stage), evict-first
__device__ __forceinline__ void tma_load_4d_stream(void *dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                                   unsigned long long *bar, unsigned long long policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)),
        "l"(policy)
        : "memory");
}
__device__ __forceinline__ int d_chunks_of(int F) { return min(D_CHUNKS, F / 64); }
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<unsigned long long>(map)) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory"); }

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
        if (global_ns() - t0 > ctl->wait_ns) {
            record_error(ctr, ctl, code);
            return false;
        }
    }
}

// ------------------------------------------------------------ producer --
// The producer keeps one unit decoded ahead: while it issues the stages of
// the current unit, the next unit's gate/up completion count (down units)
// is already in flight, so no global round trip sits between two stages.
struct UnitInfo : UnitRec {
    int dep;  // D (lane 0): gate/up units of the expert already published
};

// q = floor(u / per) for 0 <= u < 2^22 from a float reciprocal, corrected
// to the exact quotient.
__device__ __forceinline__ int div_by(int u, int per, float inv) {
    int q = __float2int_rz(__fmul_rn(static_cast<float>(u), inv));
    if ((q + 1) * per <= u) ++q;
    else if (q * per > u) --q;
    return q;
}

// The unit sequence: all gate/up units, then the down units.  Units are
// dealt round robin, so the last, partial round decides when the kernel
// ends.  When that round holds only down units and cutting each of them
// into its k-ranges (one stage each, their sums meet in y's atomic adds)
// lowers the largest per-CTA stage count by two or more, the round is cut.
struct UnitCounts {
    int n_gu, d_main, split, total;  // split: down units cut into k-ranges
};
__device__ __forceinline__ UnitCounts unit_counts(const ExpertArgs &a, int total_tiles, int split) {
    UnitCounts c;
    c.n_gu = total_tiles * a.gu_per_tile;
    c.split = split;
    c.d_main = total_tiles * a.d_per_tile - split;
    c.total = c.n_gu + c.d_main + split * a.ns_d;
    return c;
}
// DENSE: dense mode known at compile time (the fused layer kernel), which
// leaves the tile-mode code out of the persistent kernel.
template <bool DENSE>
__device__ __forceinline__ void decode_rec(int u, int n_units, const ExpertArgs &a, const SharedCtl *ctl,
                                           UnitRec &ui) {
    if (u >= n_units) {
        ui.type = UNIT_END;
        return;
    }
    const UnitCounts uc = unit_counts(a, ctl->total_tiles, ctl->split);
    ui.k0 = 0;
    if (u >= uc.n_gu + uc.d_main) {
        // a k-range of one of the last round's down units
        const int j = u - uc.n_gu - uc.d_main;
        const int q = div_by(j, a.ns_d, a.inv_nsd);
        ui.k0 = j - q * a.ns_d;
        u = uc.n_gu + uc.d_main + q;
    }
    if (DENSE || a.dense) {
        // one tile per active expert: slot i's units are consecutive
        const bool gu = u < uc.n_gu;
        const int v = gu ? u : u - uc.n_gu;
        const int per = gu ? a.gu_per_tile : a.d_per_tile;
        const int i = div_by(v, per, gu ? a.inv_gu : a.inv_d);
        ui.type = gu ? UNIT_GU : UNIT_D;
        ui.ns = gu ? a.ns_gu : (ui.k0 > 0 || u - uc.n_gu >= uc.d_main ? 1 : a.ns_d);
        ui.row0 = (v - i * per) * (gu ? a.gu_rows : D_ROWS);
        ui.i_act = i;
        ui.e = ctl->act_e[i];
        ui.p0 = i * a.B;
        ui.n = a.B;
        ui.need = a.gu_per_tile;
        return;
    }
    const int gu_per_tile = a.gu_per_tile;
    const int n_gu = ctl->total_tiles * gu_per_tile;
    int per, v;
    if (u < n_gu) {
        ui.type = UNIT_GU;
        per = gu_per_tile;
        v = u;
        ui.ns = a.ns_gu;
    } else {
        ui.type = UNIT_D;
        per = a.d_per_tile;
        v = u - n_gu;
        ui.ns = v >= uc.d_main ? 1 : a.ns_d;
    }
    // active expert owning this unit: largest i with tile_start[i] <= v / per
    const int tile = v / per;
    int lo = 0, hi = ctl->n_active - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ctl->tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int i = lo;
    // an expert's units: row block major, token tile minor, so the tiles of
    // one weight block run back to back (a re-read then hits L2)
    const int nt_i = ctl->tile_start[i + 1] - ctl->tile_start[i];
    const int local = v - ctl->tile_start[i] * per;
    const int blk = local / nt_i;
    const int tt = local - blk * nt_i;
    ui.row0 = blk * (ui.type == UNIT_GU ? a.gu_rows : D_ROWS);
    ui.i_act = i;
    ui.e = ctl->act_e[i];
    ui.p0 = ctl->off[i] + tt * TN;
    ui.n = min(TN, ctl->off[i + 1] - ui.p0);
    ui.need = nt_i * gu_per_tile;
}

// The j-th unit of this CTA's round-robin sequence (units blockIdx.x +
// j * unit_ctas).  The producer's lanes decode UNIT_WINDOW units at a time
// into shared memory; the prefetches of the unit's first stage are issued
// here and first used when that stage is issued.
template <bool DENSE>
__device__ bool fetch_unit(int j, int &win_base, int n_units, const ExpertArgs &a, SharedCtl *ctl, int lane,
                           UnitInfo &ui) {
    if (j >= win_base + UNIT_WINDOW) {
        __syncwarp();
        decode_rec<DENSE>(blockIdx.x + (j + lane) * a.unit_ctas, n_units, a, ctl, ctl->urec[lane]);
        __syncwarp();
        win_base = j;
    }
    static_cast<UnitRec &>(ui) = ctl->urec[j - win_base];
    if (ui.type == UNIT_END) return false;
    ui.dep = 0;
    if (ui.type == UNIT_D && lane == 0) ui.dep = ld_acquire(&a.ctr->gu_done[ui.i_act]);
    return true;
}

// A gate/up stage of the tensor-core path is one box of the 4-D gate/up
// map where the two weight buffers allow it (the whole 32 KB stage,
// measured about 8 % faster in steady state than per-chunk boxes), else
// UM_CHUNKS chunk copies of each matrix, interleaved per chunk (the
// tensor-core operand layout); on the warp-MMA path (WM) one gate box and
// one up box of gc chunks each.
template <class RG, bool DENSE, bool WM>
__device__ void producer(const ExpertArgs &a, const ExpertMaps &m, SharedCtl *ctl, unsigned char *slots) {
    constexpr int STAGES = RG::STAGES;
    const int lane = threadIdx.x & 31;
    // host-computed per tile count: the producer's set-up code runs once per
    // call on the critical path, so it does no arithmetic it can avoid
    const int t = ctl->total_tiles;
    const int split = t <= SPLIT_TABLE_MAX ? a.split_for[t] : 0;
    if (lane == 0) ctl->split = split;
    __syncwarp();
    const int n_units = unit_counts(a, t, split).total;
    const unsigned long long policy = evict_first_policy();
    // units are dealt round robin: CTA c takes c, c + grid, c + 2 grid, ...
    // (all CTAs start together when the lists are ready; every gate/up unit
    // precedes every down unit in each CTA's sequence)
    int j_next = 0, win_base = -UNIT_WINDOW;
    UnitInfo cur;
    bool have = fetch_unit<DENSE>(j_next++, win_base, n_units, a, ctl, lane, cur);
    int g = 0;  // stages issued
    bool ok = true;
    while (have && ok) {
        UnitInfo nxt;
        bool have_nxt = false;
        for (int s = 0; s < cur.ns; ++s) {
            const int slot = g % STAGES;
            if (g >= STAGES &&
                !wait_phase(&ctl->empty[slot], ((g / STAGES) - 1) & 1, ctl, a.ctr, DEV_TIMEOUT_EMPTY)) {
                ok = false;
                break;
            }
            unsigned char *wdst = slots + slot * RG::SLOT_BYTES;
            unsigned char *odst = wdst + W_BYTES;
            const int gc = a.gc, dc = d_chunks_of(a.F);
            // chunks of d this gate/up stage covers (the last stage may hold fewer)
            const int gcv = min(gc, (a.d >> 6) - (cur.k0 + s) * gc);
            // x tile: all B token rows (dense mode) or the tile's TN pair rows
            const unsigned xbytes = static_cast<unsigned>(gc) * (a.dense ? a.bpad : TN) * 128u;
            // (whole-stage boxes and the warp-MMA boxes always hold gc
            // chunks; the tail of d reads as zeros)
            const unsigned wbytes = (WM || m.gu_mode) ? 2u * gc * static_cast<unsigned>(a.gu_rows * 128) : 2u * gcv * UM_TILE;
            const unsigned bytes = cur.type == UNIT_GU ? wbytes + xbytes : dc * (D_ROWS * 128u) + dc * (a.hrows * 128u);
            if (lane == 0) {
                StageHdr &h = ctl->hdr[slot];
                h.type = cur.type;
                h.e = cur.e;
                h.i_act = cur.i_act;
                h.p0 = cur.p0;
                h.n = cur.n;
                h.row0 = cur.row0;
                h.s = s;
                h.ns = cur.ns;
                h.k = cur.k0 + s;
                mbar_expect_tx(&ctl->full[slot], bytes);
            }
            __syncwarp();
            if (cur.type == UNIT_GU) {
                const int grow = cur.e * a.F + cur.row0;
                if (!WM && m.gu_mode) {
                    // the whole stage in one box of the 4-D gate/up map:
                    // [chunk][gate rows][up rows] (halves swapped when Wup
                    // is the lower buffer)
                    if (lane == 0) tma_load_4d_stream(wdst, &m.gu, 0, grow, 0, s * gc, &ctl->full[slot], policy);
                } else if constexpr (WM) {
                    // the gate box of gc chunks, the up box at WM_UP_OFF
                    if (lane == 0)
                        tma_load_3d_stream(wdst, &m.gate, 0, grow, s * gc, &ctl->full[slot], policy);
                    else if (lane == 8)
                        tma_load_3d_stream(wdst + WM_UP_OFF, &m.up, 0, grow, s * gc, &ctl->full[slot], policy);
                } else {
                    // chunk c: gate tile at 8 KB c, up tile 4 KB after it
                    if (lane < gcv)
                        tma_load_3d_stream(wdst + lane * UM_CHUNK_BYTES, &m.gate, 0, grow, s * gc + lane,
                                           &ctl->full[slot], policy);
                    else if (lane >= 8 && lane < 8 + gcv)
                        tma_load_3d_stream(wdst + (lane - 8) * UM_CHUNK_BYTES + UM_TILE, &m.up, 0, grow,
                                           s * gc + lane - 8, &ctl->full[slot], policy);
                }
                // x rows for this column range, one swizzled box: all B
                // tokens (dense mode) or the tile's pairs of the dispatched x
                if (lane == 16) tma_load_3d(odst, &m.x, 0, (DENSE || a.dense) ? 0 : cur.p0, s * gc, &ctl->full[slot]);
            } else {
                if (lane == 0)
                    tma_load_3d_stream(wdst, &m.down, 0, cur.e * a.d + cur.row0, (cur.k0 + s) * dc, &ctl->full[slot],
                                       policy);
                if (s == 0) {
                    // this expert's gate/up units must be complete before H is read
                    if (lane == 0) {
                        // the prefetched count was read with acquire semantics;
                        // if it is short, poll (acquire) until complete
                        int v = cur.dep;
                        if (v < cur.need) {
                            const unsigned long long t0 = global_ns();
                            while ((v = ld_acquire(&a.ctr->gu_done[cur.i_act])) < cur.need) {
                                if (ctl->abort_flag) { ok = false; break; }
                                if (global_ns() - t0 > a.wait_ns) {
                                    record_error(a.ctr, ctl, DEV_TIMEOUT_DEP);
                                    ok = false;
                                    break;
                                }
                                __nanosleep(64);
                            }
                        }
                        // H was written through the generic proxy; it is read by TMA
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                }
                if (ok && lane == 1) tma_load_3d(odst, &m.h, 0, cur.p0, (cur.k0 + s) * dc, &ctl->full[slot]);
            }
            ++g;
            if (!ok) break;
            if (s == 0) have_nxt = fetch_unit<DENSE>(j_next++, win_base, n_units, a, ctl, lane, nxt);
        }
        cur = nxt;
        have = have_nxt;
    }
    if (ok) {
        // end marker for the issuers (and, through them, the epilogue) or
        // the warp-MMA consumers
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
                if (global_ns() - t0 > DRAIN_LIMIT_NS) break;
            }
        }
    }
}

// ------------------------------------------------ tensor-core path (dense) --
// TMEM columns of the CTA's allocation: two accumulator buffers, each
// NISSUE partial accumulators of bpad columns (a power of two, at least 32).
__device__ __forceinline__ int tmem_cols_for(int bpad) {
    int c = 32;
    while (c < 2 * NISSUE * bpad) c <<= 1;
    return c;
}

// Issuer p (one thread of each issuer warp): for every stage it waits for
// the copies, issues k-steps p, p + NISSUE, ... of the stage (64-row x
// bpad-column MMAs, K = 16 each) into its partial accumulator of the unit's
// buffer, and commits them to the stage's empty barrier (the slot is free
// once every issuer's MMAs have read it).  At a unit's last stage it commits
// to the buffer's full barrier as well.  A gate/up chunk is [32 gate rows]
// [32 up rows] of 64 columns and a down chunk 64 rows of Wdown, both one
// 8 KB operand; the token rows (x, or H) are the B operand, bpad rows per
// chunk.  Issuer 0 also hands the unit's header to the epilogue.
__device__ void umma_issuer(const ExpertArgs &a, SharedCtl *ctl, unsigned char *slots, int stages, int slot_bytes,
                            uint32_t tmem, int p) {
    const uint32_t idesc = umma_idesc_bf16(a.hrows);
    const uint32_t b_chunk = static_cast<uint32_t>(a.hrows) * 128u;
    const uint32_t buf_stride = static_cast<uint32_t>(tmem_cols_for(a.hrows) / 2);
    const int gk = 64 * a.gc, dk = 64 * d_chunks_of(a.F);
    int unit = 0;  // units started
    for (int g = 0;; ++g) {
        const int slot = g % stages;
        if (!wait_phase(&ctl->full[slot], (g / stages) & 1, ctl, a.ctr, DEV_TIMEOUT_FULL)) break;
        if (p == 0) ctl->consumed = g + 1;  // the copies have landed
        const StageHdr h = ctl->hdr[slot];
        const int b = unit & 1;
        if (h.type == UNIT_END || h.s == 0) {
            // the buffer's previous unit must have been read out
            if (unit >= 2 && !wait_phase(&ctl->acc_empty[b], ((unit >> 1) - 1) & 1, ctl, a.ctr, DEV_TIMEOUT_EMPTY))
                break;
            tc_fence_after();
            if (p == 0) {
                AccHdr &ah = ctl->acc_hdr[b];
                ah.type = h.type;
                ah.i_act = h.i_act;
                ah.row0 = h.row0;
                ah.p0 = h.p0;
                ah.n = h.n;
                // the extra arrival of the buffer's phase; releases the header
                mbar_arrive(&ctl->acc_full[b]);
            }
            if (h.type == UNIT_END) {
                mbar_arrive(&ctl->acc_full[b]);
                break;
            }
        }
        const uint32_t wbase = smem_u32(slots + slot * slot_bytes);
        const uint32_t obase = wbase + W_BYTES;
        const int nks = (h.type == UNIT_GU ? min(gk, a.d - h.k * gk) : min(dk, a.F - h.k * dk)) >> 4;
        const uint32_t dcol = tmem + static_cast<uint32_t>(b) * buf_stride + static_cast<uint32_t>(p * a.hrows);
        // nks >= 4 = NISSUE (d and d_ff are multiples of 64): every issuer
        // starts its partial sum at stage 0
        for (int ks = p; ks < nks; ks += NISSUE) {
            const uint32_t c = static_cast<uint32_t>(ks >> 2), kk = static_cast<uint32_t>(ks & 3) * 32u;
            umma_bf16(dcol, umma_desc(wbase + c * UM_CHUNK_BYTES + kk), umma_desc(obase + c * b_chunk + kk), idesc,
                      (h.s > 0 || ks >= NISSUE) ? 1u : 0u);
        }
        umma_commit(smem_u32(&ctl->empty[slot]));
        if (h.s == h.ns - 1) {
            umma_commit(smem_u32(&ctl->acc_full[b]));
            ++unit;
        }
    }
    // every MMA issued must have completed before the CTA's shared memory
    // and tensor memory are released
    umma_commit(smem_u32(&ctl->mma_done));
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(&ctl->mma_done, 0)) {
        if (global_ns() - t0 > DRAIN_LIMIT_NS) break;
    }
}

// The eight epilogue warps, one accumulator buffer per unit in turn: warp w
// reads TMEM lanes 32 (w % 4) .. (rows 16 (w % 4) ..) for the column groups
// of 8 tokens g = w / 4, w / 4 + 2, ..., adds the issuers' partial sums in
// issuer order, releases the buffer and copies the values to shared memory
// as [token][64 rows]; then
//   gate/up unit: rows 0..31 are g, rows 32..63 u (the other way round
//     when gu_swap): h = silu(g) u -> H
//     (bf16, two rows per thread), and thread 0 publishes the completion;
//   down unit:    y[t][row0 + r] += wd[slot][t] acc[t][r], four rows per
//     vector atomic.
template <bool DENSE>
__device__ void umma_epilogue(const ExpertArgs &a, SharedCtl *ctl, float *xch, uint32_t tmem, bool gu_swap) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ct = threadIdx.x;  // 0 .. NCW*32-1
    const int q = warp & 3, half = warp >> 2;
    const int ncg = a.hrows >> 3;
    const uint32_t buf_stride = static_cast<uint32_t>(tmem_cols_for(a.hrows) / 2);
    bool lists_ready = !a.early;
    // Thread 0 takes every wait and passes its outcome through shared
    // memory, so that all epilogue threads leave together (none is left at a
    // barrier): epi_go is read between the first and second barrier of a
    // unit, epi_lists after the second.
    for (int u = 0;; ++u) {
        const int b = u & 1;
        if (ct == 0) ctl->epi_go = wait_phase(&ctl->acc_full[b], (u >> 1) & 1, ctl, a.ctr, DEV_TIMEOUT_FULL) ? 1 : 0;
        consumer_bar();  // also: the previous unit's readers of xch are done
        if (!ctl->epi_go) return;
        const AccHdr ah = ctl->acc_hdr[b];
        if (ah.type == UNIT_END) return;
        tc_fence_after();
        // the issuers' partial accumulators, summed in issuer order
        float v[4][8];
        const uint32_t tb = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b) * buf_stride;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cg = half + 2 * j;
            if (cg < ncg) {
                tmem_ld8(tb + static_cast<uint32_t>(cg * 8), v[j]);
#pragma unroll
                for (int pi = 1; pi < NISSUE; ++pi) {
                    float w8[8];
                    tmem_ld8(tb + static_cast<uint32_t>(pi * a.hrows + cg * 8), w8);
#pragma unroll
                    for (int c = 0; c < 8; ++c) v[j][c] += w8[c];
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->acc_empty[b]);
        if (ah.type == UNIT_D && !lists_ready) {
            // the dense weights are the selection's last output: in early
            // mode wait for them before the first down epilogue
            if (a.lists_flag == nullptr) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                if (ct == 0) ctl->epi_lists = 1;
            } else if (ct == 0) {
                int ok = 1;
                const unsigned long long t0 = global_ns();
                while (ld_acquire(a.lists_flag) < 1) {
                    if (ctl->abort_flag) { ok = 0; break; }
                    if (global_ns() - t0 > a.wait_ns) {
                        record_error(a.ctr, ctl, DEV_TIMEOUT_DEP);
                        ok = 0;
                        break;
                    }
                    __nanosleep(64);
                }
                ctl->epi_lists = ok;
            }
            lists_ready = true;
        }
        if (lane < 16) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int cg = half + 2 * j;
                if (cg < ncg) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) xch[(cg * 8 + c) * 64 + 16 * q + lane] = v[j][c];
                }
            }
        }
        consumer_bar();
        if (ah.type == UNIT_GU) {
            // column t: token t (dense mode) or the tile's pair t; H row p0 + t
            const int goff = gu_swap ? UM_ROWS : 0, uoff = gu_swap ? 0 : UM_ROWS;
            for (int idx = ct; idx < 16 * ah.n; idx += NCW * 32) {
                const int t = idx >> 4, r = (idx & 15) * 2;
                const float2 gs = *reinterpret_cast<const float2 *>(xch + t * 64 + goff + r);
                const float2 us = *reinterpret_cast<const float2 *>(xch + t * 64 + uoff + r);
                const float h0 = gs.x / (1.0f + __expf(-gs.x)) * us.x;
                const float h1 = gs.y / (1.0f + __expf(-gs.y)) * us.y;
                const unsigned packed = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(h0))) |
                                        (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(h1))) << 16);
                *reinterpret_cast<unsigned *>(a.h + static_cast<size_t>(ah.p0 + t) * a.F + ah.row0 + r) = packed;
            }
            // H is read by other CTAs through TMA (the async proxy)
            asm volatile("fence.proxy.async.global;" ::: "memory");
            consumer_bar();
            if (ct == 0) {
                __threadfence();
                atomicAdd(&a.ctr->gu_done[ah.i_act], 1);
            }
        } else {
            if (!ctl->epi_lists) return;
            for (int idx = ct; idx < 16 * ah.n; idx += NCW * 32) {
                const int n = idx >> 4, r = (idx & 15) * 4;
                // dense mode: token n, weight wd[slot][n]; tile mode: the
                // pair's token and weight from the lists (a token outside the
                // batch is skipped and reported)
                int t = n;
                float w;
                if (DENSE || a.dense) {
                    w = __ldcg(a.wd + static_cast<size_t>(ah.i_act) * a.B + n);
                } else {
                    t = __ldg(a.tok + ah.p0 + n);
                    const bool v = t >= 0 && t < a.B;
                    if (!v && r == 0) atomicCAS(&a.ctr->error, 0, DEV_BAD_LISTS);
                    w = v ? __ldg(a.w + ah.p0 + n) : 0.0f;
                }
                if (w != 0.0f) {
                    const float4 s4 = *reinterpret_cast<const float4 *>(xch + n * 64 + r);
                    atomicAdd(reinterpret_cast<float4 *>(a.y + static_cast<size_t>(t) * a.d + ah.row0 + r),
                              make_float4(w * s4.x, w * s4.y, w * s4.z, w * s4.w));
                }
            }
        }
    }
}

// ------------------------------------------------ warp-MMA path (B <= 8) --
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// c += A (16 x 16, row-major fragments a0..a3) * B (16 x 8, column fragments b0, b1), fp32 accumulate
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Address of (row r, 16-byte column group c) in a 128B-swizzled tile of
// 128-byte rows whose base is 1 KiB aligned (the TMA's swizzle pattern).
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int c) {
    return base + r * 128 + ((c ^ (r & 7)) << 4);
}
// The B operand fragment of k-step ks (16 columns) of an [8 rows][64 cols]
// token tile: lanes 0..7 address the rows' first 8 columns, lanes 8..15
// the next 8.
__device__ __forceinline__ void wm_b_frag(uint32_t tile, int ks, int lane, uint32_t &b0, uint32_t &b1) {
    ldsm_x2(swz(tile, lane & 7, ((ks & 3) << 1) + ((lane >> 3) & 1)), b0, b1);
}

// Gate/up stage: warp w takes k-steps w, w + NCW, ... (16 columns each) of
// the stage's 16 gate and 16 up rows against the 8 token columns.
__device__ __forceinline__ void wm_gu_stage(uint32_t gbase, uint32_t ubase, uint32_t xbase, int nks, int warp, int lane,
                                            float (&cg)[4], float (&cu)[4]) {
#pragma unroll 4
    for (int ks = warp; ks < nks; ks += NCW) {
        const int c = ks >> 2;  // 64-column chunk
        const int col = ((ks & 3) << 1) + (lane >> 4);
        uint32_t g0, g1, g2, g3, u0, u1, u2, u3, b0, b1;
        ldsm_x4(swz(gbase + c * (WM_ROWS * 128), lane & 15, col), g0, g1, g2, g3);
        ldsm_x4(swz(ubase + c * (WM_ROWS * 128), lane & 15, col), u0, u1, u2, u3);
        wm_b_frag(xbase + c * (WM_MAX * 128), ks, lane, b0, b1);
        mma_bf16(cg, g0, g1, g2, g3, b0, b1);
        mma_bf16(cu, u0, u1, u2, u3, b0, b1);
    }
}
// Down stage: warp w takes rows 16 (w % 4) .. + 16 of the 64-row unit over
// the k-steps of its half of the stage, (w / 4) * 2 D_CHUNKS ...
__device__ __forceinline__ void wm_d_stage(uint32_t wbase, uint32_t hbase, int nks, int warp, int lane,
                                           float (&acc)[4]) {
    const int r = (warp & 3) * 16 + (lane & 15);
    const int k0 = (warp >> 2) * (2 * D_CHUNKS);
    const int k1 = min(nks, k0 + 2 * D_CHUNKS);
#pragma unroll 4
    for (int ks = k0; ks < k1; ++ks) {
        const int c = ks >> 2;
        uint32_t a0, a1, a2, a3, b0, b1;
        ldsm_x4(swz(wbase + c * (D_ROWS * 128), r, ((ks & 3) << 1) + (lane >> 4)), a0, a1, a2, a3);
        wm_b_frag(hbase + c * (WM_MAX * 128), ks, lane, b0, b1);
        mma_bf16(acc, a0, a1, a2, a3, b0, b1);
    }
}

// Queue one gate/up completion (i >= 0) or the end marker (i < 0) for the
// signal warp (consumer thread 0).  A wait that expires has recorded the
// error and raised the abort flag, which ends the consumers at their next
// stage.
__device__ void wm_post(SharedCtl *ctl, Counters *ctr, int q, int i) {
    const int slot = q % SIG_SLOTS;
    if (q >= SIG_SLOTS && !wait_phase(&ctl->sig_empty[slot], ((q / SIG_SLOTS) - 1) & 1, ctl, ctr, DEV_TIMEOUT_EMPTY))
        return;
    ctl->sig_iact[slot] = i;
    mbar_arrive(&ctl->sig_full[slot]);
}
// Signal warp (one thread): turns the queued completions into gate/up
// counts visible to the whole GPU.  The consumers wrote H and passed a CTA
// barrier before the completion was queued; this thread's fence is
// cumulative over those writes, so the count is raised after H is visible.
__device__ void wm_signaller(const ExpertArgs &a, SharedCtl *ctl) {
    for (int q = 0;; ++q) {
        const int slot = q % SIG_SLOTS;
        if (!wait_phase(&ctl->sig_full[slot], (q / SIG_SLOTS) & 1, ctl, a.ctr, DEV_TIMEOUT_FULL)) return;
        const int i = ctl->sig_iact[slot];
        mbar_arrive(&ctl->sig_empty[slot]);
        if (i < 0) return;
        __threadfence();
        atomicAdd(&a.ctr->gu_done[i], 1);
    }
}

// The eight consumer warps of the warp-MMA path (dense mode, B <= WM_MAX):
// every stage's math and, at a unit's last stage, its epilogue
//   gate/up: the warps' k-slices are summed in a fixed order (warp w + 4
//     into warp w, then the four sums), h = silu(g) u -> H (bf16), and the
//     completion is queued for the signal warp, so that no consumer waits
//     for the GPU-wide fence;
//   down:    y[t][row] += wd[slot][t] acc[t][row], each warp its k-half.
// Thread 0 takes every wait and passes the outcome on through shared
// memory (by stage parity), so all consumer threads leave together.
template <class RG>
__device__ void wm_consumer(const ExpertArgs &a, SharedCtl *ctl, unsigned char *slots, float *part) {
    constexpr int STAGES = RG::STAGES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ct = threadIdx.x;  // 0 .. NCW*32-1
    const int row = lane >> 2, col = (lane & 3) * 2;
    const int gk = 64 * a.gc, dk = 64 * d_chunks_of(a.F);
    float acc_g[4], acc_u[4], wk[2] = {0.0f, 0.0f};
    bool lists_ready = !a.early;
    int nsig = 0;  // completions queued (thread 0)
    for (int g = 0;; ++g) {
        const int slot = g % STAGES;
        const unsigned parity = (g / STAGES) & 1;
        if (ct == 0) ctl->wm_go[g & 1] = wait_phase(&ctl->full[slot], parity, ctl, a.ctr, DEV_TIMEOUT_FULL) ? 1 : 0;
        consumer_bar();
        if (!ctl->wm_go[g & 1]) return;
        // the phase is complete: this thread's own observation of it orders
        // the copies' data before its reads
        (void)mbar_try_wait(&ctl->full[slot], parity);
        if (ct == 0) ctl->consumed = g + 1;
        const StageHdr h = ctl->hdr[slot];
        if (h.type == UNIT_END) {
            if (ct == 0) wm_post(ctl, a.ctr, nsig, -1);
            return;
        }
        if (h.s == 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c) acc_g[c] = acc_u[c] = 0.0f;
            if (h.type == UNIT_D) {
                if (!lists_ready) {
                    // the dense weights are the selection's last output: in
                    // early mode wait for them before the first down unit
                    if (a.lists_flag == nullptr) {
                        asm volatile("griddepcontrol.wait;" ::: "memory");
                    } else if (ct == 0) {
                        int ok = 1;
                        const unsigned long long t0 = global_ns();
                        while (ld_acquire(a.lists_flag) < 1) {
                            if (ctl->abort_flag) { ok = 0; break; }
                            if (global_ns() - t0 > a.wait_ns) {
                                record_error(a.ctr, ctl, DEV_TIMEOUT_DEP);
                                ok = 0;
                                break;
                            }
                            __nanosleep(64);
                        }
                        ctl->epi_lists = ok;
                    }
                    consumer_bar();
                    if (!ctl->epi_lists) return;
                    lists_ready = true;
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int t = col + c;
                    wk[c] = t < a.B ? __ldcg(a.wd + static_cast<size_t>(h.i_act) * a.B + t) : 0.0f;
                }
            }
        }
        const uint32_t wbase = smem_u32(slots + slot * RG::SLOT_BYTES);
        const uint32_t obase = wbase + W_BYTES;
        if (h.type == UNIT_GU)
            wm_gu_stage(wbase, wbase + WM_UP_OFF, obase, min(gk, a.d - h.k * gk) >> 4, warp, lane, acc_g, acc_u);
        else wm_d_stage(wbase, obase, min(dk, a.F - h.k * dk) >> 4, warp, lane, acc_g);
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->empty[slot]);
        if (h.s != h.ns - 1) continue;

        // ---- unit epilogue (accumulator c: row lane/4 + 8 (c/2), token 2 (lane%4) + c%2)
        if (h.type == UNIT_D) {
            const int i_base = h.row0 + (warp & 3) * 16 + row;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int t = col + (c & 1);
                if (t < a.B && wk[c & 1] != 0.0f)
                    atomicAdd(a.y + static_cast<size_t>(t) * a.d + i_base + ((c >> 1) << 3), wk[c & 1] * acc_g[c]);
            }
            continue;
        }
        // gate/up: part holds, per warp pair (w, w + 4), g then u as [16 rows][8 tokens]
        float *pg = part + (warp & 3) * (2 * WM_ROWS * WM_MAX);
        float *pu = pg + WM_ROWS * WM_MAX;
        if (warp >= 4) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int o = (row + ((c >> 1) << 3)) * WM_MAX + col + (c & 1);
                pg[o] = acc_g[c];
                pu[o] = acc_u[c];
            }
        }
        consumer_bar();
        if (warp < 4) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int o = (row + ((c >> 1) << 3)) * WM_MAX + col + (c & 1);
                pg[o] = acc_g[c] + pg[o];
                pu[o] = acc_u[c] + pu[o];
            }
        }
        consumer_bar();
        for (int idx = ct; idx < WM_ROWS * h.n; idx += NCW * 32) {
            const int r = idx & (WM_ROWS - 1), t = idx >> 4;
            float gs = 0.0f, us = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                gs += part[q * (2 * WM_ROWS * WM_MAX) + r * WM_MAX + t];
                us += part[q * (2 * WM_ROWS * WM_MAX) + WM_ROWS * WM_MAX + r * WM_MAX + t];
            }
            const float hv = gs / (1.0f + __expf(-gs)) * us;
            a.h[static_cast<size_t>(h.p0 + t) * a.F + h.row0 + r] = __bfloat16_as_ushort(__float2bfloat16_rn(hv));
        }
        // H is read by other CTAs through TMA (the async proxy)
        asm volatile("fence.proxy.async.global;" ::: "memory");
        consumer_bar();
        if (ct == 0) wm_post(ctl, a.ctr, nsig++, h.i_act);
    }
}

// n_active of caller-supplied lists, checked by the producer warp before
// any list value is used as an index: 0 <= n_active <= min(E, B*k) (the H
// and dense-weight slots), every active id an expert, and offsets
// non-decreasing within [0, B*k] with at most B pairs per expert (a token
// chooses an expert once).  Inconsistent lists record DEV_BAD_LISTS and
// run as an empty call (n_active = 0).  Token ids are checked where they
// are used.
__device__ int checked_n_active(const ExpertArgs &a, int lane) {
    const int na = __ldcg(a.n_active);
    const int pairs = a.B * a.k;
    bool bad = na < 0 || na > min(a.E, pairs);
    if (!bad) {
        for (int i = lane; i < na; i += 32) {
            const int e = __ldcg(a.active + i);
            const int o0 = __ldcg(a.offsets + i), o1 = __ldcg(a.offsets + i + 1);
            bad = bad || e < 0 || e >= a.E || o0 < 0 || o1 < o0 || o1 > pairs || o1 - o0 > a.B;
        }
    }
    bad = __any_sync(0xffffffffu, bad);
    if (bad && lane == 0) atomicCAS(&a.ctr->error, 0, DEV_BAD_LISTS);
    return bad ? 0 : na;
}

// Shared memory of an expert CTA: the ring slots, the gate/up epilogue
// buffer and the control block, from a 1024-byte aligned base.
template <class RG>
struct CtaSmem {
    unsigned char *slots;
    float *part;
    SharedCtl *ctl;
    __device__ explicit CtaSmem(unsigned char *raw) {
        unsigned char *base = reinterpret_cast<unsigned char *>(
            (reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
        slots = base;
        part = reinterpret_cast<float *>(base + RG::STAGES * RG::SLOT_BYTES);
        ctl = reinterpret_cast<SharedCtl *>(base + RG::STAGES * RG::SLOT_BYTES + RG::PART_BYTES);
    }
};

// Barriers and flags of a CTA (thread 0).  A stage is released by the
// issuers' MMA commits (warp-MMA path: by the consumer warps).
template <class RG, bool WM>
__device__ void ctl_init(SharedCtl *ctl, unsigned long long wait_ns) {
    for (int s = 0; s < RG::STAGES; ++s) {
        mbar_init(&ctl->full[s], 1);
        mbar_init(&ctl->empty[s], WM ? NCW : NISSUE);  // one MMA commit per issuer, or one arrival per warp
    }
    for (int b = 0; b < 2; ++b) {
        mbar_init(&ctl->acc_full[b], NISSUE + 1);  // the first issuer's arrive + every issuer's commit
        mbar_init(&ctl->acc_empty[b], NCW);
    }
    if (WM) {
        for (int q = 0; q < SIG_SLOTS; ++q) {
            mbar_init(&ctl->sig_full[q], 1);
            mbar_init(&ctl->sig_empty[q], 1);
        }
    }
    mbar_init(&ctl->mma_done, NISSUE);
    ctl->epi_lists = 1;
    ctl->wait_ns = wait_ns;
    ctl->abort_flag = 0;
    ctl->consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void prefetch_expert_maps(const ExpertMaps &maps) {
    if (maps.gu_mode) {
        prefetch_tmap(&maps.gu);
    } else {
        prefetch_tmap(&maps.gate);
        prefetch_tmap(&maps.up);
    }
    prefetch_tmap(&maps.down);
    prefetch_tmap(&maps.h);
    prefetch_tmap(&maps.x);
}

// Dense mode from an activated-set bit mask (producer warp; lane l holds
// word l, experts 32 l .. 32 l + 31): one tile per active expert in
// ascending expert order, the slot order the selection uses for H and the
// dense weights; H rows of slot i start at i * B.
__device__ void table_from_mask(const ExpertArgs &a, SharedCtl *ctl, unsigned word, int lane) {
    if (32 * lane >= a.E) word = 0u;
    else if (a.E - 32 * lane < 32) word &= (1u << (a.E - 32 * lane)) - 1u;
    int incl = __popc(word);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int pos = incl - __popc(word);
    while (word != 0u) {
        const int bit = __ffs(word) - 1;
        word &= word - 1u;
        ctl->act_e[pos] = 32 * lane + bit;
        ctl->tile_start[pos] = pos;
        ctl->off[pos] = pos * a.B;
        ++pos;
    }
    const int na = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) {
        ctl->tile_start[na] = na;
        ctl->off[na] = na * a.B;
        ctl->n_active = na;
        ctl->total_tiles = na;
    }
}

// Early mode: wait (bounded) until the activated set is published in the
// CTA's copy of the publication line, then build the table from its mask.
__device__ void table_from_publication(const ExpertArgs &a, SharedCtl *ctl, int lane) {
    bool ok = true;
    uint4 m0 = make_uint4(0u, 0u, 0u, 0u), m1 = m0;
    const PubLine *pl = &a.ctr->pubs[blockIdx.x % PUB_COPIES];
    if (lane == 0) {
        const unsigned long long t0 = global_ns();
        while (ld_acquire(&pl->pub) < a.pub_target) {
            if (global_ns() - t0 > a.wait_ns) {
                record_error(a.ctr, ctl, DEV_TIMEOUT_DEP);
                ok = false;
                break;
            }
            __nanosleep(64);
        }
        if (ok) {
            m0 = __ldcg(reinterpret_cast<const uint4 *>(pl->mask));
            m1 = __ldcg(reinterpret_cast<const uint4 *>(pl->mask) + 1);
        }
    }
    const unsigned mw[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    unsigned word = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const unsigned v = __shfl_sync(0xffffffffu, mw[i], 0);
        if (lane == i) word = v;
    }
    table_from_mask(a, ctl, word, lane);
}

// Lists from the caller (or the selection kernel): checked, then the tile
// table (producer warp).
__device__ void table_from_lists(const ExpertArgs &a, SharedCtl *ctl, int lane) {
    const int na = checked_n_active(a, lane);
    if (a.dense) {
        // one tile per active expert; H rows of slot i start at i * B
        for (int i = lane; i < na; i += 32) {
            ctl->tile_start[i] = i;
            ctl->act_e[i] = __ldcg(a.active + i);
            ctl->off[i] = i * a.B;
        }
        if (lane == 0) {
            ctl->tile_start[na] = na;
            ctl->off[na] = na * a.B;
            ctl->n_active = na;
            ctl->total_tiles = na;
        }
        return;
    }
    // tile table: active expert i owns tiles [tile_start[i], tile_start[i+1])
    int run = 0;
    for (int base_i = 0; base_i < na; base_i += 32) {
        const int i = base_i + lane;
        int nt = 0;
        if (i < na) nt = (__ldcg(a.offsets + i + 1) - __ldcg(a.offsets + i) + TN - 1) / TN;
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (i < na) {
            ctl->tile_start[i] = run + incl - nt;
            ctl->act_e[i] = __ldcg(a.active + i);
            ctl->off[i] = __ldcg(a.offsets + i);
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        ctl->off[na] = na > 0 ? __ldcg(a.offsets + na) : 0;
        ctl->tile_start[na] = run;
        ctl->n_active = na;
        ctl->total_tiles = run;
    }
}

// Allocation of the CTA's TMEM columns by the first issuer warp at kernel
// entry, off the critical path; the address is read after the CTA barrier
// that follows (with the tcgen05 fences around it).
__device__ __forceinline__ void tmem_alloc_cta(const ExpertArgs &a, SharedCtl *ctl) {
    if ((threadIdx.x >> 5) == NCW + 1) tmem_alloc(smem_u32(&ctl->tmem), tmem_cols_for(a.hrows));
}

// The roles of an expert CTA: the producer, NISSUE MMA issuer warps (one
// thread each; the first holds the CTA's TMEM allocation) and eight
// epilogue warps; on the warp-MMA path (WM) the producer, eight consumer
// warps and a signal warp (the other issuer warps idle).
template <class RG, bool DENSE, bool WM>
__device__ __forceinline__ void run_roles(const ExpertArgs &a, const ExpertMaps &maps, const CtaSmem<RG> &sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if constexpr (WM) {
        if (warp == NCW) producer<RG, DENSE, true>(a, maps, sm.ctl, sm.slots);
        else if (warp < NCW) wm_consumer<RG>(a, sm.ctl, sm.slots, sm.part);
        else if (warp == NCW + 1 && lane == 0) wm_signaller(a, sm.ctl);
        __syncthreads();
        return;
    }
    // the TMEM columns were allocated at kernel entry (tmem_alloc_cta)
    const int cols = tmem_cols_for(a.hrows);
    const uint32_t tmem = sm.ctl->tmem;
    if (warp == NCW) {
        producer<RG, DENSE, false>(a, maps, sm.ctl, sm.slots);
    } else if (warp > NCW) {
        if (lane == 0) umma_issuer(a, sm.ctl, sm.slots, RG::STAGES, RG::SLOT_BYTES, tmem, warp - NCW - 1);
    } else {
        umma_epilogue<DENSE>(a, sm.ctl, sm.part, tmem, maps.gu_mode == 2);
    }
    // the issuers have waited for their MMAs, the epilogue for its loads
    tc_fence_before();
    __syncthreads();
    if (warp == NCW + 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, cols);
    }
}

// The last CTA to finish puts the call's counters back to zero (every CTA
// has passed the grid barrier, read the published set and awaits no
// gate/up count any more); the next call's kernels start after this grid
// completes.
__device__ void cta_exit(const ExpertArgs &a, SharedCtl *ctl) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        ctl->last_cta = atomicAdd(&a.ctr->k3_exit, 1) == static_cast<int>(gridDim.x) - 1 ? 1 : 0;
    }
    __syncthreads();
    if (ctl->last_cta) {
        __threadfence();
        for (int i = threadIdx.x; i < E_MAX; i += blockDim.x) a.ctr->gu_done[i] = 0;
        for (int i = threadIdx.x; i < PUB_COPIES * (E_MAX / 32); i += blockDim.x)
            a.ctr->pubs[i / (E_MAX / 32)].mask[i % (E_MAX / 32)] = 0u;
        if (threadIdx.x < PUB_COPIES) a.ctr->pubs[threadIdx.x].pub = 0;
        if (threadIdx.x == 0) {
            a.ctr->k3_exit = 0;
            a.ctr->arrive = 0;
            a.ctr->lists_ready = 0;
        }
    }
}

template <class RG, bool WM>
__global__ void __launch_bounds__(NTHREADS, 1)
    expert_ffn_kernel(const __grid_constant__ ExpertMaps maps, const ExpertArgs a) {
    extern __shared__ unsigned char smem_raw[];
    const CtaSmem<RG> sm(smem_raw);
    SharedCtl *ctl = sm.ctl;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) ctl_init<RG, WM>(ctl, a.wait_ns);
    if (warp == NCW && lane == 0) prefetch_expert_maps(maps);
    if (!WM) tmem_alloc_cta(a, ctl);
    // everything above overlaps the previous kernel (selection or input
    // preparation); the lists are complete once it has
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == NCW) table_from_lists(a, ctl, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    run_roles<RG, false, WM>(a, maps, sm);
    cta_exit(a, ctl);
}

// ------------------------------------------------------ fused layer kernel --
// One persistent grid for the whole layer call when B <= 64 (dense mode),
// one CTA per SM, launched cooperatively so that every CTA is resident:
//  1. router: the CTAs compute the logits in items of (epb experts) x (tpb
//     tokens) with the router's fixed-order dot products (rows staged by
//     TMA in the ring's shared memory); meanwhile every CTA writes its share
//     of x in bf16 and zeroes its share of y;
//  2. grid barrier: each CTA counts itself in (release) and waits (acquire,
//     bounded) until all have;
//  3. the last CTA runs the batch selection (softmax, re-selection, weights,
//     lists, dense weights) and raises a flag when the dense weights are
//     written; for the batch-wide rules it publishes the activated set as
//     soon as that is fixed;
//  4. every other CTA takes the activated set -- OEA and plain top-k: it
//     ranks every token's first r1 experts itself (the union of the kept
//     sets, resp. of the top-k sets, is final before any fill is chosen);
//     the batch-wide rules: from the selection CTA's publication -- and
//     streams its share of the activated experts' units as the standalone
//     expert kernel does, waiting for the flag only before its first down
//     epilogue.
struct LayerArgs {
    const float *x;     // [B][d] fp32
    const float *bias;  // [E] or null
    float *logits;      // [B][E]
    int epb, tpb;       // experts (one warp each) and tokens per router item
    int n_eg, n_items;  // expert groups; items = expert groups x token groups
    int row_bytes;      // shared-memory stride of one staged row (multiple of 1024)
    int box_lines, boxes;
    int r1;             // first ranks per token forming the set (OEA: k0, top-k: k); 0: published
    int residual;       // y = x + the experts' output (a layer of a residual stack) instead of y = 0 + ...
    // launched with programmatic dependent launch after the previous layer
    // of a stack: x (its output) and the shared workspace are read only
    // after the previous kernel has completed; the router weights of this
    // layer are staged before that
    int chained;
    ReselectArgs sel;   // the selection CTA's arguments
};

// OR each token's first r1 experts (r1 <= R) into s_set (bit e of word
// e / 32): warp w takes tokens w, w + NCW, ...
template <int NI, int R>
__device__ __forceinline__ void rank_union(const ExpertArgs &a, const LayerArgs &L, int warp, int lane,
                                           unsigned *s_set) {
#pragma unroll 1
    for (int b = warp; b < a.B; b += 2 * NCW) {
        const int b2 = b + NCW;
        const bool two = b2 < a.B;
        float l[NI], l2[NI];
        unsigned ord[NI], ord2[NI];
        load_row<NI>(L.logits + static_cast<size_t>(b) * a.E, a.E, lane, l);
        load_row<NI>(L.logits + static_cast<size_t>(two ? b2 : b) * a.E, a.E, lane, l2);
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            ord[i] = ord_of(l[i]);
            ord2[i] = ord_of(l2[i]);
        }
        unsigned long long top[R], top2[R];
        warp_top_r<NI, R>(ord, a.E, lane, top);
        warp_top_r<NI, R>(ord2, a.E, lane, top2);
        unsigned mine = 0u;  // bits of expert word `lane`
#pragma unroll
        for (int j = 0; j < R; ++j) {
            if (j >= L.r1) break;
            const int e = topr_expert(top[j]), e2 = topr_expert(top2[j]);
            if (e >= 0 && (e >> 5) == lane) mine |= 1u << (e & 31);
            if (two && e2 >= 0 && (e2 >> 5) == lane) mine |= 1u << (e2 & 31);
        }
        if (lane < E_MAX / 32 && mine != 0u) atomicOr(&s_set[lane], mine);
    }
}

template <class RG, int NI, bool WM>
__global__ void __launch_bounds__(NTHREADS, 1)
    layer_kernel(const __grid_constant__ ExpertMaps maps, const __grid_constant__ RouterMaps rmaps,
                 const ExpertArgs a, const LayerArgs L) {
    extern __shared__ unsigned char smem_raw[];
    const CtaSmem<RG> sm(smem_raw);
    SharedCtl *ctl = sm.ctl;
    __shared__ __align__(8) unsigned long long s_rbar;  // router row staging
    __shared__ unsigned s_set[E_MAX / 32];
    __shared__ int s_ok;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *wrows = sm.slots;
    unsigned char *xrows = sm.slots + L.epb * L.row_bytes;
    const int lines = a.d >> 5;  // 128-byte lines per row
    // the router's row copies of this CTA's first item come first: they are
    // the head of the call's critical path (the router weights do not depend
    // on a previous layer; the token rows, in a stack, do)
    auto issue_rows = [&](int item, bool weights, bool tokens) {
        const int eg = item % L.n_eg, tg = item / L.n_eg;
        const int e0 = eg * L.epb, b0 = tg * L.tpb;
        const int ne = min(L.epb, a.E - e0), nb = min(L.tpb, a.B - b0);
        if (weights) {
            for (int r = 0; r < ne; ++r)
                for (int bx = 0; bx < L.boxes; ++bx)
                    tma_rows(wrows + r * L.row_bytes + bx * L.box_lines * 128, &rmaps.wg,
                                  (e0 + r) * lines + bx * L.box_lines, &s_rbar);
        }
        if (tokens)
            for (int r = 0; r < nb; ++r)
                for (int bx = 0; bx < L.boxes; ++bx)
                    tma_rows(xrows + r * L.row_bytes + bx * L.box_lines * 128, &rmaps.x,
                             (b0 + r) * lines + bx * L.box_lines, &s_rbar);
    };
    auto item_bytes = [&](int item, bool weights) {
        const int eg = item % L.n_eg, tg = item / L.n_eg;
        const int n = weights ? min(L.epb, a.E - eg * L.epb) : min(L.tpb, a.B - tg * L.tpb);
        return static_cast<unsigned>(n * L.boxes * L.box_lines * 128);
    };
    bool waited = !L.chained;
    if (threadIdx.x == 0) {
        mbar_init(&s_rbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (static_cast<int>(blockIdx.x) < L.n_items) {
            const int item = blockIdx.x;
            if (waited) {
                mbar_expect_tx(&s_rbar, item_bytes(item, true) + item_bytes(item, false));
                issue_rows(item, true, true);
            } else {
                mbar_add_tx(&s_rbar, item_bytes(item, true));
                issue_rows(item, true, false);
            }
        }
        ctl_init<RG, WM>(ctl, a.wait_ns);
        s_ok = 1;
    }
    if (threadIdx.x < E_MAX / 32) s_set[threadIdx.x] = 0u;
    if (warp == NCW && lane == 0) {
        prefetch_expert_maps(maps);
        prefetch_tmap(&rmaps.x);
        prefetch_tmap(&rmaps.wg);
    }
    // the expert CTAs' TMEM columns (the selection CTA runs no MMAs, the
    // warp-MMA path none on the tensor-core pipe)
    if (!WM && blockIdx.x != gridDim.x - 1) tmem_alloc_cta(a, ctl);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // a layer of a stack may start while the previous layer's last CTAs
    // still run: let the next layer's CTAs launch as SMs free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- 1. router items (one per CTA when there are no more items than CTAs)
    bool prepped = false;
    int phase = 0;
    for (int item = blockIdx.x; item < L.n_items; item += gridDim.x) {
        const int eg = item % L.n_eg, tg = item / L.n_eg;
        const int e0 = eg * L.epb, b0 = tg * L.tpb;
        const int ne = min(L.epb, a.E - e0), nb = min(L.tpb, a.B - b0);
        if (item != static_cast<int>(blockIdx.x) && threadIdx.x == 0) {
            // a later item: the staging area was freed at the end of the last one
            mbar_expect_tx(&s_rbar, item_bytes(item, true) + item_bytes(item, false));
            issue_rows(item, true, true);
        }
        if (!waited) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            waited = true;
            if (threadIdx.x == 0) {
                mbar_expect_tx(&s_rbar, item_bytes(item, false));
                issue_rows(item, false, true);
            }
        }
        if (!prepped) {
            // x -> bf16 (read by the gate/up copies) and y = 0 or x (the
            // down epilogues add into it), grid-stride: overlaps the row loads
            layer_prep(L.x, a.B, a.d, const_cast<uint16_t *>(a.xb), a.y, L.residual != 0);
            prepped = true;
        }
        // every thread waits for the rows; on expiry the rows are still
        // awaited (drained) before the shared memory is used for anything else
        if (!mbar_try_wait(&s_rbar, phase)) {
            const unsigned long long t0 = global_ns();
            bool late = false;
            while (!mbar_try_wait(&s_rbar, phase)) {
                const unsigned long long dt = global_ns() - t0;
                if (!late && dt > a.wait_ns) {
                    late = true;
                    s_ok = 0;
                    atomicCAS(&a.ctr->error, 0, DEV_TIMEOUT_FULL);
                }
                if (dt > a.wait_ns + DRAIN_LIMIT_NS) break;
            }
        }
        __syncthreads();
        if (warp < ne && s_ok) {
            const int e = e0 + warp;
            float acc[GEMV_TPB_MAX];
#pragma unroll
            for (int t = 0; t < GEMV_TPB_MAX; ++t) acc[t] = 0.0f;
            if ((a.d & 255) == 0) gemv_rows<true>(wrows + warp * L.row_bytes, xrows, L.row_bytes, a.d, nb, lane, acc);
            else gemv_rows<false>(wrows + warp * L.row_bytes, xrows, L.row_bytes, a.d, nb, lane, acc);
            float mine = 0.0f;
#pragma unroll
            for (int t = 0; t < GEMV_TPB_MAX; ++t) {
                const float v = warp_butterfly_sum(acc[t]);
                if (lane == t) mine = v;
            }
            if (lane < nb) {
                const float v = L.bias ? __fadd_rn(mine, __ldg(L.bias + e)) : mine;
                L.logits[static_cast<size_t>(b0 + lane) * a.E + e] = v;
            }
        }
        __syncthreads();  // the staging area is free again
        phase ^= 1;
    }
    if (!waited) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!prepped) layer_prep(L.x, a.B, a.d, const_cast<uint16_t *>(a.xb), a.y, L.residual != 0);
    // x in bf16 is read by the async proxy (TMA) of other CTAs
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncthreads();

    // ---- 2. grid barrier
    if (threadIdx.x == 0) {
        // the CTA barrier above orders the CTA's writes before this thread's
        // release, which makes them visible at gpu scope
        asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(&a.ctr->arrive), "r"(1) : "memory");
        const unsigned long long t0 = global_ns();
        while (ld_acquire(&a.ctr->arrive) < static_cast<int>(gridDim.x)) {
            if (global_ns() - t0 > a.wait_ns) {
                atomicCAS(&a.ctr->error, 0, DEV_TIMEOUT_DEP);
                s_ok = 0;
                break;
            }
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncthreads();
    const bool ok = s_ok != 0;

    // ---- 3. the selection CTA
    if (blockIdx.x == gridDim.x - 1) {
        if (ok) reselect_body<NI>(L.sel, sm.slots);
        __syncthreads();
        if (threadIdx.x == 0)
            asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(&a.ctr->lists_ready), "r"(1) : "memory");
        cta_exit(a, ctl);
        return;
    }

    // ---- 4. the activated set, then the expert stream
    if (L.r1 > 0) {
        // each warp ranks tokens warp, warp + NCW, ... (two at a time, their
        // butterfly merges independent); only the union of the tokens' first
        // r1 experts is kept, so the order within a token does not matter
        if (warp < NCW && ok) {
            if (L.r1 <= 4) rank_union<NI, 4>(a, L, warp, lane, s_set);
            else if (L.r1 <= 8) rank_union<NI, 8>(a, L, warp, lane, s_set);
            else rank_union<NI, 16>(a, L, warp, lane, s_set);
        }
        __syncthreads();
        if (warp == NCW) table_from_mask(a, ctl, lane < E_MAX / 32 ? s_set[lane] : 0u, lane);
    } else if (warp == NCW) {
        if (ok) table_from_publication(a, ctl, lane);
        else table_from_mask(a, ctl, 0u, lane);
    }
    // only the producer warp, which built it, reads the unit table: the
    // other roles start at once
    run_roles<RG, true, WM>(a, maps, sm);
    cta_exit(a, ctl);
}

// ------------------------------------------------------------------ prep --
// Input preparation of the expert kernel, chained before it:
//  - x in bf16 [B][d] (dense mode) or, for larger batches, each pair's x
//    row in bf16 at its list position p: xd[p] = x[tok[p]] (the dispatch);
//  - y = 0 (standalone path; the layer path's router already zeroed it);
//  - dense mode: the weight matrix wd[slot][B] from the lists;
//  - the gate/up completion counts cleared (standalone path).
struct PrepArgs {
    const float *x;
    int B, d, k;
    int slots;     // active-expert slots: min(E, B*k)
    uint16_t *xb;  // dense mode: x in bf16, or null
    uint16_t *xd;  // larger batches: dispatched x rows, or null
    float *y;      // zeroed when non-null
    Counters *ctr; // gate/up counts cleared when non-null
    const int32_t *n_active, *offsets, *tok;
    const float *w;
    float *wd;  // dense weights [slot][B] (B <= 64), or null
    int32_t *err;  // error word for inconsistent lists, or null
};

__device__ __forceinline__ uint2 bf16x4(float4 v) {
    const unsigned lo = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x))) |
                        (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
    const unsigned hi = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.z))) |
                        (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v.w))) << 16);
    return make_uint2(lo, hi);
}

__global__ void __launch_bounds__(256) ffn_prep_kernel(PrepArgs p) {
    // the lists may come from the previous kernel (the layer path's selection)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = blockIdx.x * blockDim.x + threadIdx.x, nthreads = gridDim.x * blockDim.x;
    const int n4 = p.B * p.d / 4;
    if (p.xb || p.y) {
        for (int i = tid; i < n4; i += nthreads) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(p.x) + i);
            if (p.xb) reinterpret_cast<uint2 *>(p.xb)[i] = bf16x4(v);
            if (p.y) reinterpret_cast<float4 *>(p.y)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // the lists may come from the caller: n_active and the offsets are
    // clamped to the buffers they index (min(E, B*k) active slots, B*k
    // pairs) and tokens outside the batch are skipped; the expert kernel
    // checks the same lists and reports inconsistent ones
    const int pairs = p.B * p.k;
    if (p.xd) {
        // one thread per 4 columns of a pair row; rows of unused pairs skipped
        const int na = *p.n_active;
        const int total = (na > 0 && na <= p.slots) ? min(max(p.offsets[na], 0), pairs) : 0;
        const int q4 = p.d / 4;
        for (int i = tid; i < total * q4; i += nthreads) {
            const int pr = i / q4, c = i - pr * q4;
            const int t = p.tok[pr];
            if (t < 0 || t >= p.B) continue;
            const float4 v = __ldg(reinterpret_cast<const float4 *>(p.x) + static_cast<size_t>(t) * q4 + c);
            reinterpret_cast<uint2 *>(p.xd)[static_cast<size_t>(pr) * q4 + c] = bf16x4(v);
        }
    }
    if (p.wd) {
        // wd[i][t] = weight of token t in active expert i's list, else 0:
        // one warp per active expert (its list holds at most B <= 64 pairs)
        const int na0 = *p.n_active;
        const int na = (na0 > 0 && na0 <= p.slots) ? na0 : 0;
        const int lane = threadIdx.x & 31;
        for (int i = tid >> 5; i < na; i += nthreads >> 5) {
            const int j0 = min(max(p.offsets[i], 0), pairs);
            const int n = min(min(max(p.offsets[i + 1], j0), pairs) - j0, p.B);
            for (int t = lane; t < p.B; t += 32) p.wd[static_cast<size_t>(i) * p.B + t] = 0.0f;
            __syncwarp();
            for (int q = lane; q < n; q += 32) {
                const int t = p.tok[j0 + q];
                if (t >= 0 && t < p.B) p.wd[static_cast<size_t>(i) * p.B + t] = p.w[j0 + q];
                else if (p.err) atomicCAS(p.err, 0, DEV_BAD_LISTS);  // pair skipped
            }
        }
    }
    if (p.ctr && blockIdx.x == 0)
        for (int i = threadIdx.x; i < E_MAX; i += blockDim.x) p.ctr->gu_done[i] = 0;
}

// Host side of the last-round cut (see unit_counts): the largest per-CTA
// stage count when consecutive slices of the unit sequence (start, length,
// stages per unit) are dealt round robin over P CTAs.  Every CTA takes
// floor(len / P) units of a slice and the len % P CTAs from start % P on
// (cyclically) one more; the largest sum of extras is reached at the start
// of one of the slices' extra runs.
struct Slice {
    long long start, len, w;
};
long long max_stages_host(const Slice *sl, int ns, long long P) {
    long long base = 0, best = 0;
    for (int i = 0; i < ns; ++i) base += sl[i].w * (sl[i].len / P);
    for (int i = 0; i < ns; ++i) {
        if (sl[i].len % P == 0) continue;
        const long long c = sl[i].start % P;
        long long extra = 0;
        for (int j = 0; j < ns; ++j)
            if (((c - sl[j].start % P) % P + P) % P < sl[j].len % P) extra += sl[j].w;
        best = best > extra ? best : extra;
    }
    return base + best;
}
// Last-round down units to cut for `tiles` tiles: only when that round
// holds down units alone and the cut lowers the largest stage count by two
// or more (one stage does not pay for the extra epilogues, measured).
int split_for_tiles(long long tiles, int gu_per_tile, int d_per_tile, int ns_gu, int ns_d, long long P) {
    const long long n_gu = tiles * gu_per_tile, n_d = tiles * d_per_tile;
    const long long r = (n_gu + n_d) % P;
    if (ns_d <= 1 || r == 0 || r > n_d) return 0;
    const Slice whole[2] = {{0, n_gu, ns_gu}, {n_gu, n_d, ns_d}};
    const Slice cut[3] = {{0, n_gu, ns_gu}, {n_gu, n_d - r, ns_d}, {n_gu + n_d - r, r * ns_d, 1}};
    return max_stages_host(cut, 3, P) + 2 <= max_stages_host(whole, 2, P) ? static_cast<int>(r) : 0;
}

int g_num_sms[MAX_DEVICES] = {0};

}  // namespace

int expert_ffn_h_rows(int B) { return B <= DENSE_MAX ? (B + 7) / 8 * 8 : TN; }
int expert_ffn_dense_batch(int B) { return B <= DENSE_MAX ? 1 : 0; }
int expert_ffn_warp_mma(const moe_dims_t &d, int max_active) {
    return d.B <= WM_MAX && max_active <= WM_ACTIVE_MAX ? 1 : 0;
}
int expert_ffn_gu_rows(int wm) { return wm ? WM_ROWS : UM_ROWS; }
int expert_ffn_d_rows() { return D_ROWS; }
int expert_ffn_gu_chunks(int d, int wm) {
    const int c = wm ? WM_CHUNKS : UM_CHUNKS;
    return d / 64 < c ? d / 64 : c;
}
int expert_ffn_gu_box_chunks(int d, int wm) { return wm ? expert_ffn_gu_chunks(d, wm) : 1; }
int expert_ffn_d_chunks(int F) { return F / 64 < D_CHUNKS ? F / 64 : D_CHUNKS; }

cudaError_t launch_ffn_prep(const float *x, const moe_dims_t &d, uint16_t *xb, uint16_t *xd, float *y,
                            Counters *ctr, const moe_lists_t &l, float *wd, bool chained, cudaStream_t s) {
    PrepArgs p;
    p.x = x;
    p.B = d.B;
    p.d = d.d;
    p.k = d.k;
    p.slots = active_slots(d);
    p.err = ctr ? &ctr->error : nullptr;
    p.xb = xb;
    p.xd = xd;
    p.y = y;
    p.ctr = ctr;
    p.n_active = l.n_active;
    p.offsets = l.offsets;
    p.tok = l.tok;
    p.w = l.w;
    p.wd = wd;
    const long long work = xd ? static_cast<long long>(d.B) * d.k * d.d / 4 : static_cast<long long>(d.B) * d.d / 4;
    const int blocks = static_cast<int>(work / 256 + 1 < 1024 ? work / 256 + 1 : 1024);
    if (!chained) {
        ffn_prep_kernel<<<blocks, 256, 0, s>>>(p);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ffn_prep_kernel, p);
}

namespace {

// Number of SMs of the current device (cached per device).
cudaError_t device_sms(int *dev_out, int *sms) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    if (g_num_sms[dev] == 0) {
        int n = 0;
        err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        g_num_sms[dev] = n;
    }
    *dev_out = dev;
    *sms = g_num_sms[dev];
    return cudaSuccess;
}

// Sets the dynamic shared-memory limit of a kernel once per device (keyed
// by the kernel's address: template instances share a type).
template <class K>
cudaError_t configure_smem(K kernel, int bytes, int dev) {
    static std::mutex mu;
    static const void *done[64][MAX_DEVICES] = {};
    const void *key = reinterpret_cast<const void *>(kernel);
    std::lock_guard<std::mutex> lock(mu);
    int slot = 0;
    for (; slot < 64 && done[slot][dev] != nullptr; ++slot)
        if (done[slot][dev] == key) return cudaSuccess;
    const cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err == cudaSuccess && slot < 64) done[slot][dev] = key;
    return err;
}

// Expert-stream arguments for dims d, units dealt to `unit_ctas` CTAs.
ExpertArgs make_expert_args(const uint16_t *xb, const moe_dims_t &d, const moe_lists_t &l, float *y, uint16_t *h,
                            const float *wd, Counters *ctr, int unit_ctas, int wm) {
    ExpertArgs a;
    a.xb = xb;
    a.B = d.B;
    a.d = d.d;
    a.E = d.E;
    a.k = d.k;
    a.F = d.d_ff;
    a.wait_ns = wait_limit_ns();
    a.unit_ctas = unit_ctas;
    a.lists_flag = nullptr;
    a.dense = d.B <= DENSE_MAX ? 1 : 0;
    a.gu_rows = expert_ffn_gu_rows(wm);
    a.gc = expert_ffn_gu_chunks(d.d, wm);
    a.bpad = (d.B + 7) / 8 * 8;
    a.hrows = expert_ffn_h_rows(d.B);
    a.early = 0;
    a.pub_target = 0;
    a.gu_per_tile = d.d_ff / a.gu_rows;
    a.d_per_tile = d.d / D_ROWS;
    {
        const int gk = 64 * a.gc, dk = 64 * expert_ffn_d_chunks(d.d_ff);
        a.ns_gu = (d.d + gk - 1) / gk;
        a.ns_d = (d.d_ff + dk - 1) / dk;
    }
    a.inv_gu = 1.0f / static_cast<float>(a.gu_per_tile);
    a.inv_d = 1.0f / static_cast<float>(a.d_per_tile);
    a.inv_nsd = 1.0f / static_cast<float>(a.ns_d);
    {
        // cached per unit geometry and grid size (one GPU and shape at a time
        // in practice; recomputed when either changes)
        static std::mutex mu;
        static int key[5] = {-1, -1, -1, -1, -1};
        static unsigned char table[SPLIT_TABLE_MAX + 1];
        const int k[5] = {a.gu_per_tile, a.d_per_tile, a.ns_gu, a.ns_d, unit_ctas};
        std::lock_guard<std::mutex> lock(mu);
        if (std::memcmp(k, key, sizeof(k)) != 0) {
            for (int t = 0; t <= SPLIT_TABLE_MAX; ++t)
                table[t] = static_cast<unsigned char>(split_for_tiles(t, k[0], k[1], k[2], k[3], unit_ctas));
            std::memcpy(key, k, sizeof(k));
        }
        std::memcpy(a.split_for, table, sizeof(table));
    }
    a.wd = wd;
    a.n_active = l.n_active;
    a.active = l.active;
    a.offsets = l.offsets;
    a.tok = l.tok;
    a.w = l.w;
    a.y = y;
    a.h = h;
    a.ctr = ctr;
    return a;
}

// Router items of the fused layer kernel: tokens per item up to 4, experts
// per item 4 (8 when 4 would give more items than CTAs), both cut back
// while the staged rows exceed the ring's shared memory.
LayerArgs make_layer_router(const moe_dims_t &d, int grid, int ring_bytes) {
    LayerArgs L;
    const int lines = d.d / 32;
    L.box_lines = router_box_lines(d.d);
    L.boxes = (lines + L.box_lines - 1) / L.box_lines;
    L.row_bytes = (L.boxes * L.box_lines * 128 + 1023) / 1024 * 1024;
    L.tpb = d.B < GEMV_TPB_MAX ? d.B : GEMV_TPB_MAX;
    const int n_tg = (d.B + L.tpb - 1) / L.tpb;
    L.epb = ((d.E + 3) / 4) * n_tg > grid ? NCW : 4;
    while ((L.epb + L.tpb) * L.row_bytes > ring_bytes) {
        if (L.epb > 1) --L.epb;
        else if (L.tpb > 1) --L.tpb;
        else break;
    }
    L.n_eg = (d.E + L.epb - 1) / L.epb;
    L.n_items = L.n_eg * ((d.B + L.tpb - 1) / L.tpb);
    return L;
}

template <class RG, int NI, bool WM>
cudaError_t launch_layer_ni(const ExpertMaps &maps, const RouterMaps &rmaps, const ExpertArgs &a,
                            const LayerArgs &L, int grid, int dev, cudaStream_t s) {
    cudaError_t err = configure_smem(layer_kernel<RG, NI, WM>, smem_bytes<RG>(), dev);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem_bytes<RG>();
    cfg.stream = s;
    // every CTA must be resident: the CTAs wait for one another at the
    // grid barrier.  A chained layer may launch before the previous one has
    // finished (its CTAs take SMs as the previous layer's CTAs leave them).
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = L.chained ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, layer_kernel<RG, NI, WM>, maps, rmaps, a, L);
}

}  // namespace

namespace {
template <class RG, bool WM>
cudaError_t launch_expert_ffn_rg(const ExpertMaps &maps, const ExpertArgs &a, int sms, int dev, cudaStream_t s) {
    cudaError_t err = configure_smem(expert_ffn_kernel<RG, WM>, smem_bytes<RG>(), dev);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem_bytes<RG>();
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;  // always chained to the previous kernel with programmatic dependent launch
    return cudaLaunchKernelEx(&cfg, expert_ffn_kernel<RG, WM>, maps, a);
}
}  // namespace

cudaError_t launch_expert_ffn(const ExpertMaps &maps, const uint16_t *xb, const moe_dims_t &d,
                              const moe_lists_t &l, float *y, uint16_t *h, const float *wd, Counters *ctr, int wm,
                              cudaStream_t s) {
    if (wm && d.B > WM_MAX) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t err = device_sms(&dev, &sms);
    if (err != cudaSuccess) return err;
    const ExpertArgs a = make_expert_args(xb, d, l, y, h, wd, ctr, sms, wm);
    // the warp-MMA path, or the ring sized for the token rows: dense mode
    // up to 16, 32 or 64 tokens, tile mode (64 pair rows) above
    if (wm) return launch_expert_ffn_rg<RingB16, true>(maps, a, sms, dev, s);
    if (d.B <= 16) return launch_expert_ffn_rg<RingB16, false>(maps, a, sms, dev, s);
    if (d.B <= 32) return launch_expert_ffn_rg<RingB32, false>(maps, a, sms, dev, s);
    return launch_expert_ffn_rg<RingB64, false>(maps, a, sms, dev, s);
}

cudaError_t launch_layer_fused(const ExpertMaps &maps, const RouterMaps &rmaps, const moe_dims_t &d,
                               const moe_reselect_t &rule, const float *x, const float *bias, float *logits,
                               float *probs, uint16_t *xb, float *y, uint16_t *h, float *wd, int32_t *sel_idx,
                               float *sel_w, const moe_lists_t &lists, int32_t *n_active_copy, Counters *ctr,
                               int wm, bool residual, bool chained, cudaStream_t s) {
    if (d.B > DENSE_MAX || (wm && d.B > WM_MAX)) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t err = device_sms(&dev, &sms);
    if (err != cudaSuccess) return err;
    if (sms < 2) return cudaErrorInvalidConfiguration;
    // the last CTA runs the selection; the others stream the experts
    ExpertArgs a = make_expert_args(xb, d, lists, y, h, wd, ctr, sms - 1, wm);
    a.early = 1;
    a.lists_flag = &ctr->lists_ready;
    const bool batch_rule = rule.mode == MOE_RESELECT_XSHARE || rule.mode == MOE_RESELECT_AFFINITY ||
                            rule.mode == MOE_RESELECT_XSHARE_HIER;
    a.pub_target = 1;
    const int ring = d.B <= 16 ? RingB16::STAGES * RingB16::SLOT_BYTES
                     : d.B <= 32 ? RingB32::STAGES * RingB32::SLOT_BYTES
                                 : RingB64::STAGES * RingB64::SLOT_BYTES;
    LayerArgs L = make_layer_router(d, sms, ring);
    L.x = x;
    L.bias = bias;
    L.logits = logits;
    L.r1 = rule.mode == MOE_RESELECT_OEA ? rule.k0 : (rule.mode == MOE_RESELECT_NONE ? d.k : 0);
    L.residual = residual ? 1 : 0;
    L.chained = chained ? 1 : 0;
    L.sel = make_reselect_args(logits, probs, true, d, rule, sel_idx, sel_w, lists, n_active_copy);
    L.sel.ctr = ctr;
    L.sel.wd = wd;
    L.sel.publish_set = batch_rule ? 1 : 0;
    const size_t sel_smem = reselect_smem(d, rule, &L.sel.cache_rows);
    if (sel_smem > static_cast<size_t>(ring)) return cudaErrorInvalidValue;
    // instantiated for the warp-MMA path (up to WM_MAX tokens) and per ring
    // (up to 16, 32 or 64 tokens), and for logit rows of up to 128 or 256
    // experts per warp
    const bool ni8 = ni_for(d.E) > 4;
#define MOE_LAYER_CASE(RGT, WMV)                                                                       \
    return ni8 ? launch_layer_ni<RGT, 8, WMV>(maps, rmaps, a, L, sms, dev, s)                         \
               : launch_layer_ni<RGT, 4, WMV>(maps, rmaps, a, L, sms, dev, s)
    if (wm) MOE_LAYER_CASE(RingB16, true);
    if (d.B <= 16) MOE_LAYER_CASE(RingB16, false);
    if (d.B <= 32) MOE_LAYER_CASE(RingB32, false);
    MOE_LAYER_CASE(RingB64, false);
#undef MOE_LAYER_CASE
}

}  // namespace moe
