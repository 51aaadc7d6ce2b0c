// Host side of the C ABI declared in include/moe_decode.h: argument
// validation, workspace layout, TMA descriptor encoding and launch chaining.
// Nothing here allocates device memory; every failure is reported as a
// status code before anything is enqueued.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace moe {
namespace {

constexpr size_t ALIGN = 256;
constexpr unsigned long long DEFAULT_WAIT_NS = 1000000000ull;  // 1 s

std::atomic<unsigned long long> g_wait_ns{DEFAULT_WAIT_NS};

size_t round_up(size_t v) { return (v + ALIGN - 1) / ALIGN * ALIGN; }

// B, E, k: every entry point; d: all but moe_reselect; d_ff: the FFN paths.
bool dims_ok_reselect(const moe_dims_t &d) {
    if (d.B < 1 || d.B > B_MAX) return false;
    if (d.k < 1 || d.k > K_MAX) return false;
    if (d.E < d.k || d.E > E_MAX) return false;
    return true;
}

bool dims_ok_route(const moe_dims_t &d) {
    return dims_ok_reselect(d) && d.d >= D_MIN && d.d <= D_MAX && d.d % 64 == 0;
}

bool dims_ok(const moe_dims_t &d) {
    return dims_ok_route(d) && d.d_ff >= F_MIN && d.d_ff <= F_MAX && d.d_ff % 64 == 0;
}

bool rule_ok(const moe_dims_t &d, const moe_reselect_t &r) {
    switch (r.mode) {
        case MOE_RESELECT_NONE: return true;
        case MOE_RESELECT_OEA: return r.k0 >= 1 && r.k0 <= d.k;
        case MOE_RESELECT_XSHARE: return r.budget >= d.k && r.budget <= d.E;
        case MOE_RESELECT_AFFINITY: return true;
        case MOE_RESELECT_XSHARE_HIER:
            return r.budget >= d.k && r.budget <= d.E && r.group >= 1 && r.group <= B_MAX;
        default: return false;
    }
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

moe_status_t check_lists(const moe_lists_t &l) {
    if (!l.n_active || !l.active || !l.offsets || !l.tok || !l.w) return MOE_ERR_INVALID_ARG;
    if (!al16(l.n_active) || !al16(l.active) || !al16(l.offsets) || !al16(l.tok) || !al16(l.w))
        return MOE_ERR_MISALIGNED;
    return MOE_OK;
}

moe_status_t check_ws(const moe_dims_t &d, void *ws, size_t ws_bytes) {
    if (!ws) return MOE_ERR_WORKSPACE;
    if (!al256(ws)) return MOE_ERR_MISALIGNED;
    if (ws_bytes < ws_layout(d).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

// The current device must be an sm_100 part (B200).  Cached per device.
moe_status_t check_device() {
    static int cached[MAX_DEVICES] = {0};  // 0 unknown, 1 ok, 2 unsupported
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (dev < 0 || dev >= MAX_DEVICES) return MOE_ERR_UNSUPPORTED;
    if (cached[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    return cached[dev] == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

// A failed launch leaves its error as the thread's last error: clear it, so
// that the next call's launch check does not report it again.
moe_status_t from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    cudaGetLastError();
    return MOE_ERR_CUDA;
}

// ---------------------------------------------------------- tensor maps --
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// bf16 matrix [rows][cols] (row-major, cols % 64 == 0) seen as a 3-D tensor
// (64-element column chunk, row, chunk index).  One box of box_rows rows and
// box_chunks chunks lands in shared memory as box_chunks consecutive tiles of
// [box_rows][64], each with the 128-byte swizzle.  Elements past the end of
// the matrix read as zero.
bool encode_bf16_chunked(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                         uint32_t box_chunks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {64, rows, cols / 64};
    cuuint64_t gstride[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_chunks};
    cuuint32_t estride[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), gdim, gstride, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 matrix [rows][cols] (cols % 32 == 0) seen as rows * cols / 32
// lines of 32 floats; boxes of box_lines whole lines, 128-byte swizzle.
// Lines past the end read as zero.
bool encode_f32_lines(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_lines) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {32, rows * (cols / 32)};
    cuuint64_t gstride[1] = {128};
    cuuint32_t box[2] = {32, box_lines};
    cuuint32_t estride[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(ptr), gdim, gstride, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
T *seg(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

moe_lists_t ws_lists(void *ws, const WsLayout &L) {
    moe_lists_t l;
    l.n_active = seg<int32_t>(ws, L.n_active);
    l.active = seg<int32_t>(ws, L.active);
    l.offsets = seg<int32_t>(ws, L.offsets);
    l.tok = seg<int32_t>(ws, L.tok);
    l.w = seg<float>(ws, L.w);
    return l;
}

// The most experts a call under `rule` can activate: the union of every
// token's candidates (OEA: its first k0; top-k and the affinity rule: its
// k), at most the budget for the XShare rules, at most E.
int max_activated(const moe_dims_t &d, const moe_reselect_t &rule) {
    int per_token = d.k;
    if (rule.mode == MOE_RESELECT_OEA) per_token = rule.k0;
    long long n = static_cast<long long>(d.B) * per_token;
    if ((rule.mode == MOE_RESELECT_XSHARE || rule.mode == MOE_RESELECT_XSHARE_HIER) && rule.budget < n)
        n = rule.budget;
    return static_cast<int>(n < d.E ? n : d.E);
}

// One layer call (arguments validated): up to 64 tokens the fused kernel,
// above the four chained kernels.  residual: y = x + the experts' output;
// chained: the layer follows the previous layer of a stack on the stream.
moe_status_t layer_call(const float *x, const moe_layer_weights_t &w, const moe_dims_t &dims,
                        const moe_reselect_t &rule, float *y, int32_t *sel_idx, float *sel_w, int32_t *n_active,
                        void *ws, cudaStream_t s, bool residual, bool chained);

}  // namespace

// Wgate and Wup [rows][cols] (same shape) as one 4-D tensor (64 columns,
// row, matrix, chunk) with box (64, box_rows, 2, box_chunks): a stage as
// [chunk][matrix][row][64].  The matrix dimension's stride is the distance
// from the lower buffer to the higher.  Returns 0 when that distance is no
// valid stride (or the encoding fails), 1 when Wgate is the lower buffer,
// 2 when Wup is.
int encode_gate_up(CUtensorMap *map, const void *Wgate, const void *Wup, uint64_t rows, uint64_t cols,
                   uint32_t box_rows, uint32_t box_chunks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return 0;
    const uintptr_t g = reinterpret_cast<uintptr_t>(Wgate), u = reinterpret_cast<uintptr_t>(Wup);
    const uintptr_t lo = g < u ? g : u, dist = g < u ? u - g : g - u;
    // a TMA stride is a positive multiple of 16 below 2^40
    if (dist == 0 || dist % 16 != 0 || dist >= (uint64_t{1} << 40)) return 0;
    cuuint64_t gdim[4] = {64, rows, 2, cols / 64};
    cuuint64_t gstride[3] = {cols * 2, dist, 128};
    cuuint32_t box[4] = {64, box_rows, 2, box_chunks};
    cuuint32_t estride[4] = {1, 1, 1, 1};
    if (fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, reinterpret_cast<void *>(lo), gdim, gstride, box, estride,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return 0;
    return g < u ? 1 : 2;
}

bool encode_expert_maps(ExpertMaps *m, const moe_dims_t &d, const uint16_t *Wgate, const uint16_t *Wup,
                        const uint16_t *Wdown, const uint16_t *h, const uint16_t *x, int wm) {
    std::memset(m, 0, sizeof(*m));
    const uint64_t E = d.E, F = d.d_ff, D = d.d;
    const uint32_t gu_chunks = expert_ffn_gu_chunks(d.d, wm), d_chunks = expert_ffn_d_chunks(d.d_ff);
    const uint32_t gu_box = expert_ffn_gu_box_chunks(d.d, wm);
    // the tensor cores' gate/up stage in one box, [chunk][gate rows][up
    // rows]; the warp-MMA path keeps one box per matrix (a single box of
    // its 16-row stage measured slower: 4 tokens, OEA k0 = 4, 30.3 ->
    // 31.6 us)
    m->gu_mode = wm ? 0 : encode_gate_up(&m->gu, Wgate, Wup, E * F, D, expert_ffn_gu_rows(wm), gu_chunks);
    return encode_bf16_chunked(&m->gate, Wgate, E * F, D, expert_ffn_gu_rows(wm), gu_box) &&
           encode_bf16_chunked(&m->up, Wup, E * F, D, expert_ffn_gu_rows(wm), gu_box) &&
           encode_bf16_chunked(&m->down, Wdown, E * D, F, expert_ffn_d_rows(), d_chunks) &&
           encode_bf16_chunked(&m->h, h,
                               expert_ffn_dense_batch(d.B) ? static_cast<uint64_t>(active_slots(d)) * d.B
                                                           : static_cast<uint64_t>(d.B) * d.k,
                               F, expert_ffn_h_rows(d.B), d_chunks) &&
           (expert_ffn_dense_batch(d.B)
                ? encode_bf16_chunked(&m->x, x, static_cast<uint64_t>(d.B), D, (d.B + 7) / 8 * 8, gu_chunks)
                : encode_bf16_chunked(&m->x, x, static_cast<uint64_t>(d.B) * d.k, D, expert_ffn_h_rows(d.B),
                                      gu_chunks));
}

bool encode_router_maps(RouterMaps *m, const moe_dims_t &d, const float *x, const float *Wg) {
    std::memset(m, 0, sizeof(*m));
    const uint32_t bl = static_cast<uint32_t>(router_box_lines(d.d));
    return encode_f32_lines(&m->x, x, static_cast<uint64_t>(d.B), static_cast<uint64_t>(d.d), bl) &&
           encode_f32_lines(&m->wg, Wg, static_cast<uint64_t>(d.E), static_cast<uint64_t>(d.d), bl);
}

unsigned long long wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

WsLayout ws_layout(const moe_dims_t &d) {
    WsLayout L;
    size_t o = 0;
    const size_t B = d.B, E = d.E, k = d.k, D = d.d;
    L.counters = o; o += round_up(sizeof(Counters));
    L.logits = o;   o += round_up(B * E * 4);
    L.probs = o;    o += round_up(B * E * 4);
    L.sel_idx = o;  o += round_up(B * k * 4);
    L.sel_w = o;    o += round_up(B * k * 4);
    L.n_active = o; o += round_up(4);
    L.active = o;   o += round_up(E * 4);
    L.offsets = o;  o += round_up((E + 1) * 4);
    L.tok = o;      o += round_up(B * k * 4);
    L.w = o;        o += round_up(B * k * 4);
    L.xb = o;       o += round_up(B * D * 2);
    L.xd = o;       o += round_up(xd_bytes(d));
    L.h = o;        o += round_up(h_scratch_bytes(d));
    L.wd = o;       o += round_up(wd_bytes(d));
    L.total = o;
    return L;
}

namespace {

moe_status_t layer_call(const float *x, const moe_layer_weights_t &w, const moe_dims_t &dims,
                        const moe_reselect_t &rule, float *y, int32_t *sel_idx, float *sel_w, int32_t *n_active,
                        void *ws, cudaStream_t s, bool residual, bool chained) {
    const WsLayout L = ws_layout(dims);
    const bool dense = expert_ffn_dense_batch(dims.B) != 0;
    // the expert kernel's x: bf16 x (B <= 64) or the dispatched pair rows
    uint16_t *xk = dense ? seg<uint16_t>(ws, L.xb) : seg<uint16_t>(ws, L.xd);
    const int wm = expert_ffn_warp_mma(dims, max_activated(dims, rule));
    ExpertMaps maps;
    if (!encode_expert_maps(&maps, dims, w.Wgate, w.Wup, w.Wdown, seg<uint16_t>(ws, L.h), xk, wm))
        return MOE_ERR_CUDA;
    RouterMaps rmaps;
    if (!encode_router_maps(&rmaps, dims, x, w.Wg)) return MOE_ERR_CUDA;
    Counters *ctr = seg<Counters>(ws, L.counters);
    float *logits = seg<float>(ws, L.logits);
    float *probs = seg<float>(ws, L.probs);
    int32_t *si = sel_idx ? sel_idx : seg<int32_t>(ws, L.sel_idx);
    float *sw = sel_w ? sel_w : seg<float>(ws, L.sel_w);
    const moe_lists_t lists = ws_lists(ws, L);
    if (dense) {
        // B <= 64: one persistent kernel for the whole call
        return from_cuda(launch_layer_fused(maps, rmaps, dims, rule, x, w.bias, logits, probs, xk, y,
                                            seg<uint16_t>(ws, L.h), seg<float>(ws, L.wd), si, sw, lists, n_active,
                                            ctr, wm, residual, chained, s));
    }
    // larger batches: router, selection (lists), the dispatch of each
    // pair's x row, then the expert kernel, chained with programmatic
    // dependent launch
    moe_status_t st = from_cuda(launch_layer_route(rmaps, x, w.bias, dims, logits, y, ctr, residual, chained, s));
    if (st != MOE_OK) return st;
    st = from_cuda(launch_layer_select(logits, probs, dims, rule, si, sw, lists, n_active, s));
    if (st != MOE_OK) return st;
    st = from_cuda(launch_ffn_prep(x, dims, nullptr, xk, nullptr, nullptr, lists, nullptr, true, s));
    if (st != MOE_OK) return st;
    return from_cuda(launch_expert_ffn(maps, xk, dims, lists, y, seg<uint16_t>(ws, L.h), nullptr, ctr, wm, s));
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(moe_dims_t dims) {
    if (!dims_ok(dims)) return 0;
    return ws_layout(dims).total;
}

const char *moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument (null pointer, dimension or rule parameter)";
        case MOE_ERR_MISALIGNED: return "misaligned buffer (device buffers 16-byte, workspace 256-byte)";
        case MOE_ERR_WORKSPACE: return "workspace missing or smaller than moe_workspace_bytes()";
        case MOE_ERR_UNSUPPORTED: return "unsupported: outside the implemented limits or not an sm_100 device";
        case MOE_ERR_CUDA: return "a CUDA call or kernel launch failed";
        case MOE_ERR_INTERNAL: return "a kernel recorded an internal error (bounded wait expired or bad lists)";
        default: return "unknown status";
    }
}

moe_status_t moe_route(const float *x, const float *Wg, const float *bias, moe_dims_t dims, float *logits,
                       float *probs, int32_t *topk_idx, float *topk_w, void *stream) {
    if (!dims_ok_route(dims)) return MOE_ERR_INVALID_ARG;
    if (!x || !Wg || !logits || !probs || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(Wg) || (bias && !al16(bias)) || !al16(logits) || !al16(probs) || !al16(topk_idx) ||
        !al16(topk_w))
        return MOE_ERR_MISALIGNED;
    moe_status_t st = check_device();
    if (st != MOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    RouterMaps rmaps;
    if (!encode_router_maps(&rmaps, dims, x, Wg)) return MOE_ERR_CUDA;
    st = from_cuda(launch_router_logits(rmaps, bias, dims, logits, s));
    if (st != MOE_OK) return st;
    return from_cuda(launch_route_topk(logits, dims, probs, topk_idx, topk_w, s));
}

moe_status_t moe_reselect(const float *logits, const float *probs, moe_dims_t dims, moe_reselect_t rule,
                          int32_t *sel_idx, float *sel_w, moe_lists_t lists, void *stream) {
    if (!dims_ok_reselect(dims) || !rule_ok(dims, rule)) return MOE_ERR_INVALID_ARG;
    if (!logits || !probs || !sel_idx || !sel_w) return MOE_ERR_INVALID_ARG;
    moe_status_t st = check_lists(lists);
    if (st != MOE_OK) return st;
    if (!al16(logits) || !al16(probs) || !al16(sel_idx) || !al16(sel_w)) return MOE_ERR_MISALIGNED;
    st = check_device();
    if (st != MOE_OK) return st;
    return from_cuda(launch_reselect(logits, probs, dims, rule, sel_idx, sel_w, lists,
                                     static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn(const float *x, const uint16_t *Wgate, const uint16_t *Wup, const uint16_t *Wdown,
                            moe_dims_t dims, moe_lists_t lists, float *y, void *ws, size_t ws_bytes,
                            void *stream) {
    if (!dims_ok(dims)) return MOE_ERR_INVALID_ARG;
    if (!x || !Wgate || !Wup || !Wdown || !y) return MOE_ERR_INVALID_ARG;
    moe_status_t st = check_lists(lists);
    if (st != MOE_OK) return st;
    if (!al16(x) || !al16(Wgate) || !al16(Wup) || !al16(Wdown) || !al16(y)) return MOE_ERR_MISALIGNED;
    st = check_ws(dims, ws, ws_bytes);
    if (st != MOE_OK) return st;
    st = check_device();
    if (st != MOE_OK) return st;
    const WsLayout L = ws_layout(dims);
    const bool dense = expert_ffn_dense_batch(dims.B) != 0;
    // the expert kernel's x: bf16 x (B <= 64) or the dispatched pair rows
    uint16_t *xk = dense ? seg<uint16_t>(ws, L.xb) : seg<uint16_t>(ws, L.xd);
    // caller-supplied lists: any union of the tokens' k choices
    const int wm = expert_ffn_warp_mma(dims, dims.B * dims.k);
    ExpertMaps maps;
    if (!encode_expert_maps(&maps, dims, Wgate, Wup, Wdown, seg<uint16_t>(ws, L.h), xk, wm)) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Counters *ctr = seg<Counters>(ws, L.counters);
    float *wd = dense ? seg<float>(ws, L.wd) : nullptr;
    st = from_cuda(launch_ffn_prep(x, dims, dense ? xk : nullptr, dense ? nullptr : xk, y, ctr, lists, wd, false, s));
    if (st != MOE_OK) return st;
    return from_cuda(launch_expert_ffn(maps, xk, dims, lists, y, seg<uint16_t>(ws, L.h), wd, ctr, wm, s));
}

moe_status_t moe_layer_decode(const float *x, const float *Wg, const float *bias, const uint16_t *Wgate,
                              const uint16_t *Wup, const uint16_t *Wdown, moe_dims_t dims, moe_reselect_t rule,
                              float *y, int32_t *sel_idx, float *sel_w, int32_t *n_active, void *ws,
                              size_t ws_bytes, void *stream) {
    if (!dims_ok(dims) || !rule_ok(dims, rule)) return MOE_ERR_INVALID_ARG;
    if (!x || !Wg || !Wgate || !Wup || !Wdown || !y) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(Wg) || (bias && !al16(bias)) || !al16(Wgate) || !al16(Wup) || !al16(Wdown) ||
        !al16(y) || (sel_idx && !al16(sel_idx)) || (sel_w && !al16(sel_w)) || (n_active && !al16(n_active)))
        return MOE_ERR_MISALIGNED;
    moe_status_t st = check_ws(dims, ws, ws_bytes);
    if (st != MOE_OK) return st;
    st = check_device();
    if (st != MOE_OK) return st;
    const moe_layer_weights_t w = {Wg, bias, Wgate, Wup, Wdown};
    return layer_call(x, w, dims, rule, y, sel_idx, sel_w, n_active, ws, static_cast<cudaStream_t>(stream), false,
                      false);
}

moe_status_t moe_decode_stack(const moe_layer_weights_t *layers, int32_t n_layers, moe_dims_t dims,
                              moe_reselect_t rule, int32_t phase, float *xs, int32_t *sel_idx, int32_t *n_active,
                              void *ws, size_t ws_bytes, void *stream) {
    if (!layers || n_layers < 1 || n_layers > MOE_STACK_MAX_LAYERS || !xs) return MOE_ERR_INVALID_ARG;
    if (phase != MOE_PHASE_DECODE && phase != MOE_PHASE_PREFILL) return MOE_ERR_INVALID_ARG;
    // prefill bypasses the re-selection: standard top-k routing
    const moe_reselect_t r = phase == MOE_PHASE_PREFILL ? moe_reselect_t{MOE_RESELECT_NONE, 0, 0, 1} : rule;
    if (!dims_ok(dims) || !rule_ok(dims, r)) return MOE_ERR_INVALID_ARG;
    if (!al16(xs) || (sel_idx && !al16(sel_idx)) || (n_active && !al16(n_active))) return MOE_ERR_MISALIGNED;
    for (int32_t l = 0; l < n_layers; ++l) {
        const moe_layer_weights_t &w = layers[l];
        if (!w.Wg || !w.Wgate || !w.Wup || !w.Wdown) return MOE_ERR_INVALID_ARG;
        if (!al16(w.Wg) || (w.bias && !al16(w.bias)) || !al16(w.Wgate) || !al16(w.Wup) || !al16(w.Wdown))
            return MOE_ERR_MISALIGNED;
    }
    moe_status_t st = check_ws(dims, ws, ws_bytes);
    if (st != MOE_OK) return st;
    st = check_device();
    if (st != MOE_OK) return st;
    const size_t act = static_cast<size_t>(dims.B) * dims.d;
    const size_t sel = static_cast<size_t>(dims.B) * dims.k;
    for (int32_t l = 0; l < n_layers; ++l) {
        st = layer_call(xs + l * act, layers[l], dims, r, xs + (l + 1) * act, sel_idx ? sel_idx + l * sel : nullptr,
                        nullptr, n_active ? n_active + l : nullptr, ws, static_cast<cudaStream_t>(stream), true,
                        l > 0);
        if (st != MOE_OK) return st;
    }
    return MOE_OK;
}

moe_status_t moe_down_channel_major(const uint16_t *Wdown, moe_dims_t dims, uint16_t *WdownT, void *stream) {
    if (!dims_ok(dims) || !Wdown || !WdownT) return MOE_ERR_INVALID_ARG;
    if (!al16(Wdown) || !al16(WdownT)) return MOE_ERR_MISALIGNED;
    const moe_status_t st = check_device();
    if (st != MOE_OK) return st;
    return from_cuda(launch_down_transpose(Wdown, dims, WdownT, static_cast<cudaStream_t>(stream)));
}

size_t moe_channels_workspace_bytes(moe_dims_t dims) {
    if (!dims_ok(dims) || dims.B > MOE_CHANNELS_B_MAX || channels_stages(dims) < 2) return 0;
    return channels_workspace_bytes(dims);
}

moe_status_t moe_expert_ffn_channels(const float *x, const uint16_t *Wgate, const uint16_t *Wup,
                                     const uint16_t *WdownT, moe_dims_t dims, const int32_t *sel_idx,
                                     const float *sel_w, const float *score, int32_t c, float *y, uint32_t *keep,
                                     void *ws, size_t ws_bytes, void *stream) {
    if (!dims_ok(dims)) return MOE_ERR_INVALID_ARG;
    if (!x || !Wgate || !Wup || !WdownT || !sel_idx || !sel_w || !score || !y) return MOE_ERR_INVALID_ARG;
    if (c < 1 || c > dims.d_ff) return MOE_ERR_INVALID_ARG;
    if (dims.B > MOE_CHANNELS_B_MAX || channels_stages(dims) < 2) return MOE_ERR_UNSUPPORTED;
    if (!al16(x) || !al16(Wgate) || !al16(Wup) || !al16(WdownT) || !al16(sel_idx) || !al16(sel_w) ||
        !al16(score) || !al16(y) || (keep && !al16(keep)))
        return MOE_ERR_MISALIGNED;
    if (!ws) return MOE_ERR_WORKSPACE;
    if (!al256(ws)) return MOE_ERR_MISALIGNED;
    if (ws_bytes < channels_workspace_bytes(dims)) return MOE_ERR_WORKSPACE;
    const moe_status_t st = check_device();
    if (st != MOE_OK) return st;
    return from_cuda(launch_channels(x, Wgate, Wup, WdownT, dims, sel_idx, sel_w, score, c, y, keep, ws,
                                     static_cast<cudaStream_t>(stream)));
}

void moe_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns == 0 ? DEFAULT_WAIT_NS : ns, std::memory_order_relaxed); }

moe_status_t moe_check_error(void *ws, size_t ws_bytes, void *stream) {
    // every workspace of this library starts with its error word
    if (!ws || ws_bytes < sizeof(int32_t)) return MOE_ERR_WORKSPACE;
    if (!al256(ws)) return MOE_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Counters *ctr = seg<Counters>(ws, 0);
    int32_t err = 0;
    if (cudaMemcpyAsync(&err, &ctr->error, sizeof(err), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (err != 0) {
        if (cudaMemsetAsync(&ctr->error, 0, sizeof(int32_t), s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        return MOE_ERR_INTERNAL;
    }
    return MOE_OK;
}

}  // extern "C"
