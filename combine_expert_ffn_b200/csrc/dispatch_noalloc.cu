// dispatch_noalloc.cu -- moe_dispatch without a caller-provided workspace.
//
// Some callers cannot allocate device memory for us: a serving runtime that
// reserves the whole HBM budget up front and owns every device allocation
// through its own pool, or a latency-critical host path on which cudaMalloc's
// implicit device synchronisation is not acceptable.  For them this entry
// point runs the same four dispatch kernels as moe_dispatch, with their
// scratch (block histograms, block bases, partial send matrices) in a fixed
// file-scope device array instead of the workspace.  The array is
// kNoAllocScratchBytes (4 MiB) on every GPU that loads the library and stays
// there until the process exits.
//
// Host code may not hand the array's name to a kernel: on the host it is only
// a stand-in symbol.  The device address is looked up with
// cudaGetSymbolAddress on the first call made with that device current, and
// kept once the lookup has succeeded; a lookup that failed (for example one
// made while the stream was being captured) is not kept, so the next call
// tries again.
#include <mutex>

#include "kernels.h"

namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_dispatch_scratch[kNoAllocScratchBytes];

// Per device: the array's device address once a lookup has succeeded.
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices];

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

// Byte offsets of the dispatch scratch inside the static array.
struct NoAllocLayout {
    size_t status, hist_t, base_t, send_part, sendtok_part, total;
};

NoAllocLayout noalloc_layout(const moe_config &c) {
    const size_t nblk = (size_t)dispatch_nblk(c.T), E = (size_t)c.E, G = (size_t)c.G;
    NoAllocLayout L{};
    L.status = 0;
    L.hist_t = 256;
    L.base_t = L.hist_t + up256(4 * E * nblk);
    L.send_part = L.base_t + up256(4 * E * nblk);
    L.sendtok_part = L.send_part + up256(4 * nblk * G * G);
    L.total = L.sendtok_part + up256(4 * nblk * G * G);
    return L;
}

// Device address of the static scratch on the current device (set up once per device).
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
        if (e != cudaSuccess) return e;  // not cached: the next call looks it up again
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dispatch_noalloc(const moe_config *c, const void *x,
                                           const int32_t *topk_idx, int32_t *counts,
                                           int32_t *offsets, int32_t *send, int32_t *send_tok,
                                           int32_t *perm_token, int32_t *inv_perm, void *x_perm,
                                           int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!counts || !offsets || !send) return MOE_ERR_INVALID_ARG;
    if (c->T > 0 && (!topk_idx || !perm_token || !inv_perm)) return MOE_ERR_INVALID_ARG;
    if (x_perm && (!x || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
    const NoAllocLayout L = noalloc_layout(*c);
    if (L.total > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;

    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        major != 10)
        return MOE_ERR_NO_DEVICE;
    void *base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return MOE_ERR_CUDA;
    char *b = static_cast<char *>(base);
    DispatchWs dw{reinterpret_cast<int32_t *>(b + L.hist_t), reinterpret_cast<int32_t *>(b + L.base_t),
                  reinterpret_cast<int32_t *>(b + L.send_part),
                  reinterpret_cast<int32_t *>(b + L.sendtok_part)};
    int32_t *status = device_status ? device_status : reinterpret_cast<int32_t *>(b + L.status);
    cudaError_t e = launch_dispatch(x, topk_idx, c->T, c->d, c->E, c->G, c->K, counts, offsets,
                                    send, send_tok, perm_token, inv_perm, x_perm, dw, status,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
