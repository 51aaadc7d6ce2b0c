// moe_expert_ffn_noalloc: the grouped SwiGLU expert FFN for callers that
// cannot allocate device memory and have no workspace to pass.
//
// Its scratch (the expert kernel's counters, the bf16 copy of x and the
// SwiGLU activations H) lives in one file-scope static device array of
// MOE_NOALLOC_SCRATCH_BYTES.  Every GPU that loads this library holds that
// array until the process exits.  Host code cannot use the array's name as
// a device address, so the first call on each device looks the address up
// with cudaGetSymbolAddress (with that device current) and caches it; the
// kernels receive that pointer.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
unsigned char *g_scratch_addr[MAX_DEVICES] = {};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct NoallocLayout {
    size_t counters, xb, xd, h, wd, total;
};

NoallocLayout noalloc_layout(const moe_dims_t &d) {
    NoallocLayout L;
    size_t o = 0;
    L.counters = o; o += align256(sizeof(Counters));
    L.xb = o;       o += align256(expert_ffn_dense_batch(d.B) ? static_cast<size_t>(d.B) * d.d * 2 : 0);
    L.xd = o;       o += align256(xd_bytes(d));
    L.h = o;        o += align256(h_scratch_bytes(d));
    L.wd = o;       o += align256(wd_bytes(d));
    L.total = o;
    return L;
}

// Device address of the static scratch on the current device; looked up
// once per device.
moe_status_t scratch_address(unsigned char **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (dev < 0 || dev >= MAX_DEVICES) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<unsigned char *>(p);
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_expert_ffn_noalloc(const float *x, const uint16_t *Wgate, const uint16_t *Wup,
                                               const uint16_t *Wdown, moe_dims_t dims, moe_lists_t lists,
                                               float *y, void *stream) {
    if (dims.B < 1 || dims.B > B_MAX || dims.k < 1 || dims.k > K_MAX || dims.E < dims.k || dims.E > E_MAX ||
        dims.d < D_MIN || dims.d > D_MAX || dims.d % 64 != 0 || dims.d_ff < F_MIN || dims.d_ff > F_MAX ||
        dims.d_ff % 64 != 0)
        return MOE_ERR_INVALID_ARG;
    if (!x || !Wgate || !Wup || !Wdown || !y) return MOE_ERR_INVALID_ARG;
    if (!lists.n_active || !lists.active || !lists.offsets || !lists.tok || !lists.w) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(Wgate) || !al16(Wup) || !al16(Wdown) || !al16(y) || !al16(lists.n_active) ||
        !al16(lists.active) || !al16(lists.offsets) || !al16(lists.tok) || !al16(lists.w))
        return MOE_ERR_MISALIGNED;
    const NoallocLayout L = noalloc_layout(dims);
    if (L.total > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;
    unsigned char *scratch = nullptr;
    moe_status_t st = scratch_address(&scratch);
    if (st != MOE_OK) return st;

    Counters *ctr = reinterpret_cast<Counters *>(scratch + L.counters);
    const bool dense = expert_ffn_dense_batch(dims.B) != 0;
    // the expert kernel's x: bf16 x (B <= 64) or the dispatched pair rows
    uint16_t *xk = reinterpret_cast<uint16_t *>(scratch + (dense ? L.xb : L.xd));
    uint16_t *h = reinterpret_cast<uint16_t *>(scratch + L.h);
    float *wd = dense ? reinterpret_cast<float *>(scratch + L.wd) : nullptr;
    // caller-supplied lists: any union of the tokens' k choices
    const int wm = expert_ffn_warp_mma(dims, dims.B * dims.k);
    ExpertMaps maps;
    if (!encode_expert_maps(&maps, dims, Wgate, Wup, Wdown, h, xk, wm)) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the prep kernel clears the per-expert counters the expert kernel needs
    // at zero and rebuilds x, the dense weights and (in the kernel) H
    if (launch_ffn_prep(x, dims, dense ? xk : nullptr, dense ? nullptr : xk, y, ctr, lists, wd, false, s) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if (launch_expert_ffn(maps, xk, dims, lists, y, h, wd, ctr, wm, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}
