// api.cu -- the C ABI of libmoe (declared in include/moe.h).
//
// Host code only: argument validation, the workspace layout, and the launch
// sequence of each entry point.  Every compute entry point enqueues kernels
// on the caller's stream and returns; nothing here allocates device memory,
// synchronises, or copies between host and device (except
// moe_read_device_status, whose purpose is that copy).
#include <atomic>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include <nvtx3/nvToolsExt.h>

#include "kernels.h"

namespace moe {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

constexpr int64_t kWaitTimeoutNs = 2000000000LL;  // 2 s per device wait

// NVTX range ("moe.route", "moe.dispatch", ...) around the enqueue of one stage:
// a timeline profiler shows it over the stage's kernels.  NVTX v3 is header
// only; without a profiler attached a push or pop is a call to an empty hook.
class StageRange {
  public:
    explicit StageRange(const char *name) { nvtxRangePushA(name); }
    ~StageRange() { nvtxRangePop(); }
    void next(const char *name) {  // close this stage's range and open the next one
        nvtxRangePop();
        nvtxRangePushA(name);
    }
    StageRange(const StageRange &) = delete;
    StageRange &operator=(const StageRange &) = delete;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
    size_t status, scores, e_split, router_part, hist_t, base_t, send_part, sendtok_part;
    size_t topk_idx, topk_w, counts, offsets, send, send_tok, perm_token, inv_perm;
    size_t x_perm, h, y_perm, h_sh, y_sh;
    size_t total;
};

Layout layout(const moe_config &c) {
    Layout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    };
    const size_t T = (size_t)c.T, E = (size_t)c.E, K = (size_t)c.K, G = (size_t)c.G;
    const size_t nblk = (size_t)dispatch_nblk(c.T);
    L.status = take(256);
    L.scores = take(4 * T * E);
    L.e_split = take(2 * 3 * E * (size_t)c.d);
    // router partial logits: splits * T * E <= splits * tiles * 128 * 128 <= 148 * 128 * 128
    // floats (router_splits keeps splits * tiles <= 148), reserved whole so that the
    // workspace stays monotone in T
    L.router_part = take(c.T > 0 ? 4 * (size_t)148 * 128 * 128 : 0);
    L.hist_t = take(4 * E * nblk);
    L.base_t = take(4 * E * nblk);
    L.send_part = take(4 * nblk * G * G);
    L.sendtok_part = take(4 * nblk * G * G);
    L.topk_idx = take(4 * T * K);
    L.topk_w = take(4 * T * K);
    L.counts = take(4 * E);
    L.offsets = take(4 * (E + 1));
    L.send = take(4 * G * G);
    L.send_tok = take(4 * G * G);
    L.perm_token = take(4 * T * K);
    L.inv_perm = take(4 * T * K);
    L.x_perm = take(2 * T * K * (size_t)c.d);
    L.h = take(2 * T * K * (size_t)c.d_ff);
    L.y_perm = take(2 * T * K * (size_t)c.d);
    L.h_sh = take(2 * T * (size_t)c.n_shared * (size_t)c.d_ff_shared);
    L.y_sh = take(2 * T * (size_t)c.d);
    L.total = off;
    return L;
}

template <typename T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The current device must be an sm_100 part (checked once per device).
moe_status check_device() {
    static std::atomic<int> ok_cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
    if (dev < 0 || dev >= 64) return MOE_ERR_NO_DEVICE;
    int v = ok_cache[dev].load();
    if (v == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return MOE_ERR_NO_DEVICE;
        v = (major == 10 && minor == 0) ? 1 : 2;
        ok_cache[dev].store(v);
    }
    return v == 1 ? MOE_OK : MOE_ERR_NO_DEVICE;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Affinity router + node-limited top-K.  Up to 256 experts (G <= 32, E/G <= 32)
// one fused kernel keeps the affinities on chip and writes `scores` only when
// the caller asks for them; larger layers take the tensor-core logits kernel
// (affinities into `scores` or the workspace) and the warp-per-token select.
cudaError_t route_affinity(const moe_config &c, const void *x, const float *router_w,
                           const float *logit_offset, const float *bias, int32_t *topk_idx,
                           float *topk_w, float *scores, void *ws, const Layout &L,
                           cudaStream_t s) {
    int32_t *status = at<int32_t>(ws, L.status);
    void *e_split = at<void>(ws, L.e_split);
    if (router_fused_supported(c.E, c.G, c.K)) {
        cudaError_t err = launch_router_split(router_w, c.E, c.d, e_split, s);
        if (err != cudaSuccess) return err;
        return launch_router_select_fused(x, e_split, logit_offset, bias, c.T, c.d, c.E, c.G, c.K,
                                          c.M, c.router, scores, topk_idx, topk_w, status,
                                          kWaitTimeoutNs, s);
    }
    if (!scores) scores = at<float>(ws, L.scores);
    cudaError_t err = launch_router_logits_tc(x, router_w, logit_offset, c.T, c.d, c.E, c.router,
                                              e_split, at<float>(ws, L.router_part), scores,
                                              status, kWaitTimeoutNs, s);
    if (err != cudaSuccess) return err;
    return launch_route_select(scores, bias, c.T, c.E, c.G, c.K, c.M, topk_idx, topk_w, s);
}

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

}  // namespace
}  // namespace moe

using namespace moe;

namespace {
// cuMemGetAddressRange through the runtime's driver entry point (no
// link-time libcuda): the allocation that holds a device pointer
using AddrRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);
bool ipc_addr_range(const void *p, CUdeviceptr *base, size_t *bytes) {
    static AddrRangeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddrRangeFn>(f);
    });
    return fn && fn(base, bytes, reinterpret_cast<CUdeviceptr>(p)) == CUDA_SUCCESS;
}
// pointers handed out by moe_ipc_open_handle -> the mapping they lie in and
// how many successful opens returned them (the runtime hands back the same
// mapping, reference counted, when one handle is opened twice in a process)
struct IpcOpened {
    void *base;
    int opens;
};
std::mutex &ipc_mutex() {
    static std::mutex m;
    return m;
}
std::unordered_map<void *, IpcOpened> &ipc_opened() {
    static std::unordered_map<void *, IpcOpened> m;
    return m;
}
}  // namespace

extern "C" {

moe_status moe_check_config(const moe_config *c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->T < 0 || c->d <= 0 || c->E <= 0 || c->G <= 0 || c->K <= 0 || c->M <= 0 ||
        c->d_ff <= 0 || c->n_shared < 0 || c->d_ff_shared < 0)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->router < MOE_ROUTER_SIGMOID || c->router > MOE_ROUTER_HASH)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->payload < MOE_PAYLOAD_BF16 || c->payload > MOE_PAYLOAD_FP8)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->payload == MOE_PAYLOAD_FP8 && c->d % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->E % c->G || c->K % c->M || c->M > c->G || c->K / c->M > c->E / c->G)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->K > 32 || c->E > 1024 || c->G > 64) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T % c->G) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->d % 64 || c->d_ff % 64) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->n_shared > 0 && (c->d_ff_shared <= 0 || c->d_ff_shared % 64))
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)c->T * c->K >= (1LL << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)c->n_shared * c->d_ff_shared >= (1LL << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

size_t moe_workspace_size(const moe_config *c) {
    if (moe_check_config(c) != MOE_OK) return 0;
    return layout(*c).total;
}

const char *moe_status_string(int s) {
    switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (NULL required pointer or misaligned buffer)";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported layer sizes";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than moe_workspace_size()";
    case MOE_ERR_CUDA: return "a CUDA call failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
    case MOE_ERR_DEVICE_FAULT: return "a kernel found an invalid index in its inputs";
    case MOE_ERR_NO_DEVICE: return "no sm_100 device is current";
    default: return "unknown status";
    }
}

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status moe_read_device_status(const void *ws, int32_t *host_status, void *stream) {
    if (!ws || !host_status) return MOE_ERR_INVALID_ARG;
    moe_status st = check_device();
    if (st) return st;
    cudaStream_t s = as_stream(stream);
    if (cudaMemcpyAsync(host_status, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(s));
}

moe_status moe_last_device_status(const void *ws, void *stream) {
    int32_t word = MOE_OK;
    const moe_status st = moe_read_device_status(ws, &word, stream);
    return st != MOE_OK ? st : static_cast<moe_status>(word);
}

moe_status moe_clear_device_status(void *ws, void *stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    moe_status st = check_device();
    if (st) return st;
    return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), as_stream(stream)));
}

moe_status moe_route_select(const moe_config *c, const float *scores, const float *bias,
                            int32_t *topk_idx, float *topk_w, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->T > 0 && (!scores || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    return cuda_status(launch_route_select(scores, bias, c->T, c->E, c->G, c->K, c->M, topk_idx,
                                           topk_w, as_stream(stream)));
}

moe_status moe_route(const moe_config *c, const void *x, const float *router_w,
                     const float *logit_offset, const float *bias, int32_t *topk_idx,
                     float *topk_w, float *scores, void *ws, size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (c->router == MOE_ROUTER_HASH) return MOE_ERR_INVALID_ARG;
    if (c->T > 0 && (!x || !router_w || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    StageRange range("moe.route");
    return cuda_status(route_affinity(*c, x, router_w, logit_offset, bias, topk_idx, topk_w,
                                      scores, ws, L, as_stream(stream)));
}

moe_status moe_route_hash(const moe_config *c, const int64_t *token_ids, int32_t *topk_idx,
                          float *topk_w, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->T > 0 && (!topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    return cuda_status(launch_hash_route(token_ids, c->T, c->E, c->G, c->K, c->M, topk_idx, topk_w,
                                         as_stream(stream)));
}

moe_status moe_bias_update(const moe_config *c, const int32_t *counts, float gamma, float *bias,
                           void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!counts || !bias || !(gamma - gamma == 0.0f)) return MOE_ERR_INVALID_ARG;  // finite
    if ((st = check_device())) return st;
    return cuda_status(launch_bias_update(counts, c->E, c->T, c->K, gamma, bias, as_stream(stream)));
}

moe_status moe_dispatch(const moe_config *c, const void *x, const int32_t *topk_idx,
                        int32_t *counts, int32_t *offsets, int32_t *send, int32_t *send_tok,
                        int32_t *perm_token, int32_t *inv_perm, void *x_perm, void *ws,
                        size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!counts || !offsets || !send || !ws) return MOE_ERR_INVALID_ARG;
    if (c->T > 0 && (!topk_idx || !perm_token || !inv_perm)) return MOE_ERR_INVALID_ARG;
    if (x_perm && (!x || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    StageRange range("moe.dispatch");
    DispatchWs dw{at<int32_t>(ws, L.hist_t), at<int32_t>(ws, L.base_t),
                  at<int32_t>(ws, L.send_part), at<int32_t>(ws, L.sendtok_part)};
    return cuda_status(launch_dispatch(x, topk_idx, c->T, c->d, c->E, c->G, c->K, counts, offsets,
                                       send, send_tok, perm_token, inv_perm, x_perm, dw,
                                       at<int32_t>(ws, L.status), as_stream(stream)));
}

moe_status moe_permute(const moe_config *c, const void *x, const int32_t *inv_perm, void *x_perm,
                       void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->T > 0 && (!x || !inv_perm || !x_perm)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    StageRange range("moe.permute");
    return cuda_status(launch_permute(x, inv_perm, c->T, c->d, c->K, x_perm, as_stream(stream)));
}

moe_status moe_dispatch_fp8(const moe_config *c, const void *x, const int32_t *topk_idx,
                            int32_t *counts, int32_t *offsets, int32_t *send, int32_t *send_tok,
                            int32_t *perm_token, int32_t *inv_perm, uint8_t *x_perm_q,
                            float *x_scale, void *ws, size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->d % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!counts || !offsets || !send || !ws) return MOE_ERR_INVALID_ARG;
    if (c->T > 0 && (!x || !topk_idx || !perm_token || !inv_perm || !x_perm_q || !x_scale))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm_q) || !aligned16(x_scale)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    cudaStream_t s = as_stream(stream);
    DispatchWs dw{at<int32_t>(ws, L.hist_t), at<int32_t>(ws, L.base_t),
                  at<int32_t>(ws, L.send_part), at<int32_t>(ws, L.sendtok_part)};
    if (launch_dispatch(x, topk_idx, c->T, c->d, c->E, c->G, c->K, counts, offsets, send, send_tok,
                        perm_token, inv_perm, nullptr, dw, at<int32_t>(ws, L.status), s))
        return MOE_ERR_CUDA;
    return cuda_status(launch_gather_fp8(x, inv_perm, c->T, c->d, c->K, x_perm_q, x_scale, s));
}

moe_status moe_expert_ffn_fp8(const moe_config *c, const uint8_t *x_perm_q, const float *x_scale,
                              const int32_t *offsets, const void *w_gate, const void *w_up,
                              const void *w_down, void *y_perm, const void *x, const void *ws_gate,
                              const void *ws_up, const void *ws_down, void *y_shared, void *ws,
                              size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->d % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (c->T > 0) {
        if (!x_perm_q || !x_scale || !offsets || !w_gate || !w_up || !w_down || !y_perm || !x)
            return MOE_ERR_INVALID_ARG;
        if (c->n_shared > 0 && (!ws_gate || !ws_up || !ws_down || !y_shared))
            return MOE_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {x_perm_q, x_scale, w_gate, w_up, w_down, y_perm, x, ws_gate, ws_up,
                          ws_down, y_shared};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    FfnArgs a{};
    a.T = c->T; a.d = c->d; a.E = c->E; a.K = c->K; a.d_ff = c->d_ff;
    a.n_shared = c->n_shared; a.d_ff_shared = c->d_ff_shared;
    a.x_perm_q = x_perm_q; a.x_scale = x_scale; a.offsets = offsets;
    a.w_gate = w_gate; a.w_up = w_up; a.w_down = w_down;
    a.h = at<void>(ws, L.h); a.y_perm = y_perm;
    a.x = x; a.ws_gate = ws_gate; a.ws_up = ws_up; a.ws_down = ws_down;
    a.h_shared = at<void>(ws, L.h_sh); a.y_shared = y_shared;
    a.status = at<int32_t>(ws, L.status);
    a.timeout_ns = kWaitTimeoutNs;
    return cuda_status(launch_expert_ffn(a, as_stream(stream)));
}

moe_status moe_expert_ffn(const moe_config *c, const void *x_perm, const int32_t *offsets,
                          const void *w_gate, const void *w_up, const void *w_down, void *y_perm,
                          const void *x, const void *ws_gate, const void *ws_up,
                          const void *ws_down, void *y_shared, void *ws, size_t ws_bytes,
                          void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (c->T > 0) {
        if (!x_perm || !offsets || !w_gate || !w_up || !w_down || !y_perm) return MOE_ERR_INVALID_ARG;
        if (c->n_shared > 0 && (!x || !ws_gate || !ws_up || !ws_down || !y_shared))
            return MOE_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {x_perm, w_gate, w_up, w_down, y_perm, x, ws_gate, ws_up, ws_down, y_shared};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    StageRange range("moe.expert_ffn");
    FfnArgs a{};
    a.T = c->T; a.d = c->d; a.E = c->E; a.K = c->K; a.d_ff = c->d_ff;
    a.n_shared = c->n_shared; a.d_ff_shared = c->d_ff_shared;
    a.x_perm = x_perm; a.offsets = offsets;
    a.w_gate = w_gate; a.w_up = w_up; a.w_down = w_down;
    a.h = at<void>(ws, L.h); a.y_perm = y_perm;
    a.x = x; a.ws_gate = ws_gate; a.ws_up = ws_up; a.ws_down = ws_down;
    a.h_shared = at<void>(ws, L.h_sh); a.y_shared = y_shared;
    a.status = at<int32_t>(ws, L.status);
    a.timeout_ns = kWaitTimeoutNs;
    return cuda_status(launch_expert_ffn(a, as_stream(stream)));
}

moe_status moe_expert_ffn_gather(const moe_config *c, const void *x, const int32_t *perm_token,
                                 const int32_t *offsets, const void *w_gate, const void *w_up,
                                 const void *w_down, void *y_perm, const void *ws_gate,
                                 const void *ws_up, const void *ws_down, void *y_shared, void *ws,
                                 size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (c->T > 0) {
        if (!x || !perm_token || !offsets || !w_gate || !w_up || !w_down || !y_perm)
            return MOE_ERR_INVALID_ARG;
        if (c->n_shared > 0 && (!ws_gate || !ws_up || !ws_down || !y_shared))
            return MOE_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {x, w_gate, w_up, w_down, y_perm, ws_gate, ws_up, ws_down, y_shared};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    FfnArgs a{};
    a.T = c->T; a.d = c->d; a.E = c->E; a.K = c->K; a.d_ff = c->d_ff;
    a.n_shared = c->n_shared; a.d_ff_shared = c->d_ff_shared;
    a.x_perm = nullptr; a.perm_token = perm_token; a.offsets = offsets;
    a.w_gate = w_gate; a.w_up = w_up; a.w_down = w_down;
    a.h = at<void>(ws, L.h); a.y_perm = y_perm;
    a.x = x; a.ws_gate = ws_gate; a.ws_up = ws_up; a.ws_down = ws_down;
    a.h_shared = at<void>(ws, L.h_sh); a.y_shared = y_shared;
    a.status = at<int32_t>(ws, L.status);
    a.timeout_ns = kWaitTimeoutNs;
    return cuda_status(launch_expert_ffn(a, as_stream(stream)));
}

moe_status moe_combine(const moe_config *c, const void *y_perm, const int32_t *inv_perm,
                       const float *topk_w, const void *y_shared, void *out, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->T > 0 && (!y_perm || !inv_perm || !topk_w || !out)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_perm) || !aligned16(y_shared) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    StageRange range("moe.combine");
    return cuda_status(launch_combine(y_perm, inv_perm, topk_w, y_shared, c->T, c->d, c->K,
                                      (int64_t)c->T * c->K, out, as_stream(stream)));
}

}  // extern "C"

// The layer forward over row-major weights (packed == null) or the packed ones.
static moe_status forward_impl(const moe_config *c, const void *x, const float *router_w,
                               const float *logit_offset, const float *bias,
                               const int64_t *token_ids, const void *w_gate, const void *w_up,
                               const void *w_down, const void *ws_gate, const void *ws_up,
                               const void *ws_down, const void *packed, void *out,
                               int32_t *topk_idx, float *topk_w, int32_t *counts,
                               int32_t *offsets, int32_t *send, int32_t *send_tok, void *ws,
                               size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (packed && c->payload == MOE_PAYLOAD_FP8) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0) {
        if (!x || !out) return MOE_ERR_INVALID_ARG;
        if (!packed && (!w_gate || !w_up || !w_down)) return MOE_ERR_INVALID_ARG;
        if (c->router != MOE_ROUTER_HASH && !router_w) return MOE_ERR_INVALID_ARG;
        if (!packed && c->n_shared > 0 && (!ws_gate || !ws_up || !ws_down))
            return MOE_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {x, router_w, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, out, packed};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    if (c->T == 0) return MOE_OK;

    cudaStream_t s = as_stream(stream);
    if (!topk_idx) topk_idx = at<int32_t>(ws, L.topk_idx);
    if (!topk_w) topk_w = at<float>(ws, L.topk_w);
    if (!counts) counts = at<int32_t>(ws, L.counts);
    if (!offsets) offsets = at<int32_t>(ws, L.offsets);
    if (!send) send = at<int32_t>(ws, L.send);
    if (!send_tok) send_tok = at<int32_t>(ws, L.send_tok);
    int32_t *perm_token = at<int32_t>(ws, L.perm_token);
    int32_t *inv_perm = at<int32_t>(ws, L.inv_perm);
    void *y_perm = at<void>(ws, L.y_perm);
    void *y_sh = c->n_shared > 0 ? at<void>(ws, L.y_sh) : nullptr;
    int32_t *status = at<int32_t>(ws, L.status);

    StageRange layer("moe.forward");
    StageRange stage("moe.route");
    if (c->router == MOE_ROUTER_HASH) {
        if (launch_hash_route(token_ids, c->T, c->E, c->G, c->K, c->M, topk_idx, topk_w, s))
            return MOE_ERR_CUDA;
    } else {
        if (route_affinity(*c, x, router_w, logit_offset, bias, topk_idx, topk_w, nullptr, ws, L,
                           s))
            return MOE_ERR_CUDA;
    }
    stage.next("moe.dispatch");
    DispatchWs dw{at<int32_t>(ws, L.hist_t), at<int32_t>(ws, L.base_t),
                  at<int32_t>(ws, L.send_part), at<int32_t>(ws, L.sendtok_part)};
    // Two steps: the dispatch writes x_perm, GEMM1 reads it with tiled TMA loads.
    // (Gathering the rows inside GEMM1, moe_expert_ffn_gather, is bit-identical
    // but measured about 13% slower for dispatch + expert FFN at V3 sizes: its
    // 16-byte row copies feed the tensor core more slowly than whole-tile TMA
    // loads of the contiguous x_perm rows.)
    // With the FP8 payload the x_perm region holds the codes [T*K, d] and, after
    // them, the scales [T*K, d/128] (together at most half of its 2*T*K*d bytes + 16).
    void *x_perm = at<void>(ws, L.x_perm);
    const bool fp8 = c->payload == MOE_PAYLOAD_FP8;
    uint8_t *x_perm_q = static_cast<uint8_t *>(x_perm);
    float *x_scale = reinterpret_cast<float *>(x_perm_q + (size_t)c->T * c->K * c->d);
    if (launch_dispatch(x, topk_idx, c->T, c->d, c->E, c->G, c->K, counts, offsets, send, send_tok,
                        perm_token, inv_perm, fp8 ? nullptr : x_perm, dw, status, s))
        return MOE_ERR_CUDA;
    if (fp8 && launch_gather_fp8(x, inv_perm, c->T, c->d, c->K, x_perm_q, x_scale, s))
        return MOE_ERR_CUDA;
    stage.next("moe.expert_ffn");
    FfnArgs a{};
    a.T = c->T; a.d = c->d; a.E = c->E; a.K = c->K; a.d_ff = c->d_ff;
    a.n_shared = c->n_shared; a.d_ff_shared = c->d_ff_shared;
    a.x_perm = fp8 ? nullptr : x_perm; a.perm_token = nullptr; a.offsets = offsets;
    a.x_perm_q = fp8 ? x_perm_q : nullptr; a.x_scale = fp8 ? x_scale : nullptr;
    a.w_gate = w_gate; a.w_up = w_up; a.w_down = w_down;
    a.h = at<void>(ws, L.h); a.y_perm = y_perm;
    a.x = x; a.ws_gate = ws_gate; a.ws_up = ws_up; a.ws_down = ws_down;
    a.h_shared = at<void>(ws, L.h_sh); a.y_shared = y_sh;
    a.packed = packed;
    a.status = status;
    a.timeout_ns = kWaitTimeoutNs;
    if (launch_expert_ffn(a, s)) return MOE_ERR_CUDA;
    stage.next("moe.combine");
    return cuda_status(launch_combine(y_perm, inv_perm, topk_w, y_sh, c->T, c->d, c->K,
                                      (int64_t)c->T * c->K, out, s));
}

extern "C" {

moe_status moe_forward(const moe_config *c, const void *x, const float *router_w,
                       const float *logit_offset, const float *bias, const int64_t *token_ids,
                       const void *w_gate,
                       const void *w_up, const void *w_down, const void *ws_gate,
                       const void *ws_up, const void *ws_down, void *out, int32_t *topk_idx,
                       float *topk_w, int32_t *counts, int32_t *offsets, int32_t *send,
                       int32_t *send_tok, void *ws, size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->T > 0 && (!w_gate || !w_up || !w_down)) return MOE_ERR_INVALID_ARG;
    return forward_impl(c, x, router_w, logit_offset, bias, token_ids, w_gate, w_up, w_down,
                        ws_gate, ws_up, ws_down, nullptr, out, topk_idx, topk_w, counts, offsets,
                        send, send_tok, ws, ws_bytes, stream);
}

moe_status moe_forward_packed(const moe_config *c, const void *x, const float *router_w,
                              const float *logit_offset, const float *bias,
                              const int64_t *token_ids, const void *packed, void *out,
                              int32_t *topk_idx, float *topk_w, int32_t *counts, int32_t *offsets,
                              int32_t *send, int32_t *send_tok, void *ws, size_t ws_bytes,
                              void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (c->T > 0 && !packed) return MOE_ERR_INVALID_ARG;
    return forward_impl(c, x, router_w, logit_offset, bias, token_ids, nullptr, nullptr, nullptr,
                        nullptr, nullptr, nullptr, packed, out, topk_idx, topk_w, counts, offsets,
                        send, send_tok, ws, ws_bytes, stream);
}

size_t moe_packed_weights_size(const moe_config *c) {
    if (moe_check_config(c) != MOE_OK) return 0;
    return packed_layout(c->E, c->d, c->d_ff, c->n_shared, c->d_ff_shared).total;
}

moe_status moe_pack_weights(const moe_config *c, const void *w_gate, const void *w_up,
                            const void *w_down, const void *ws_gate, const void *ws_up,
                            const void *ws_down, void *packed, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!w_gate || !w_up || !w_down || !packed) return MOE_ERR_INVALID_ARG;
    if (c->n_shared > 0 && (!ws_gate || !ws_up || !ws_down)) return MOE_ERR_INVALID_ARG;
    const void *ptrs[] = {w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    return cuda_status(launch_pack_weights(c->E, c->d, c->d_ff, c->n_shared, c->d_ff_shared,
                                           w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed,
                                           as_stream(stream)));
}

moe_status moe_expert_ffn_packed(const moe_config *c, const void *x_perm, const int32_t *offsets,
                                 const void *packed, void *y_perm, const void *x, void *y_shared,
                                 void *ws, size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (c->T > 0) {
        if (!x_perm || !offsets || !packed || !y_perm) return MOE_ERR_INVALID_ARG;
        if (c->n_shared > 0 && (!x || !y_shared)) return MOE_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {x_perm, packed, y_perm, x, y_shared};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout(*c);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    StageRange range("moe.expert_ffn");
    FfnArgs a{};
    a.T = c->T; a.d = c->d; a.E = c->E; a.K = c->K; a.d_ff = c->d_ff;
    a.n_shared = c->n_shared; a.d_ff_shared = c->d_ff_shared;
    a.x_perm = x_perm; a.offsets = offsets; a.packed = packed;
    a.h = at<void>(ws, L.h); a.y_perm = y_perm;
    a.x = x; a.h_shared = at<void>(ws, L.h_sh); a.y_shared = y_shared;
    a.status = at<int32_t>(ws, L.status);
    a.timeout_ns = kWaitTimeoutNs;
    return cuda_status(launch_expert_ffn(a, as_stream(stream)));
}

// ----------------------------------------------------------------- expert parallelism
namespace {
bool ep_args_ok(const moe_config *c, int32_t world) {
    // every rank's copies may land on one owner: world * T * K rows there,
    // indexed in int32 like the single-GPU x_perm
    return world >= 1 && world <= 64 && c->E % world == 0 &&
           (int64_t)world * c->T * c->K < (1LL << 31);
}
moe_config ep_global(const moe_config *c, int32_t world) {
    moe_config g = *c;
    g.T = c->T * world;
    return g;
}
}  // namespace

size_t moe_ep_workspace_size(const moe_config *c, int32_t world) {
    if (moe_check_config(c) != MOE_OK || !ep_args_ok(c, world)) return 0;
    const moe_config g = ep_global(c, world);
    return moe_workspace_size(&g);
}

moe_status moe_ep_plan(const moe_config *c, int32_t world, int32_t rank, const int32_t *counts_all,
                       int32_t *base, int32_t *local_offsets, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world) || rank < 0 || rank >= world) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!counts_all || !base || !local_offsets) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    return cuda_status(launch_ep_plan(counts_all, world, c->E, rank, base, local_offsets,
                                      as_stream(stream)));
}

moe_status moe_ep_dispatch(const moe_config *c, int32_t world, const void *x,
                           const int32_t *topk_idx, const int32_t *offsets, const int32_t *inv_perm,
                           const int32_t *base, void *const *recv_x, int32_t *device_status,
                           void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!x || !topk_idx || !offsets || !inv_perm || !base || !recv_x))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t cap = (int64_t)world * c->T * c->K;
    return cuda_status(launch_ep_dispatch(x, topk_idx, offsets, inv_perm, base, recv_x, cap, c->T,
                                          c->d, c->E, c->K, world, device_status,
                                          as_stream(stream)));
}

moe_status moe_ep_dispatch_fp8(const moe_config *c, int32_t world, const void *x,
                               const int32_t *topk_idx, const int32_t *offsets,
                               const int32_t *inv_perm, const int32_t *base, void *const *recv_q,
                               void *const *recv_scale, int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world) || c->d % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!x || !topk_idx || !offsets || !inv_perm || !base || !recv_q || !recv_scale))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t cap = (int64_t)world * c->T * c->K;
    return cuda_status(launch_ep_dispatch_fp8(x, topk_idx, offsets, inv_perm, base, recv_q,
                                              recv_scale, cap, c->T, c->d, c->E, c->K, world,
                                              device_status, as_stream(stream)));
}

moe_status moe_ep_token_plan(const moe_config *c, int32_t world, const int32_t *topk_idx,
                             int32_t *tok_slot, int32_t *tok_counts, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!tok_counts || (c->T > 0 && (!topk_idx || !tok_slot))) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    return cuda_status(launch_ep_token_plan(topk_idx, c->T, c->E, c->K, world, tok_slot,
                                            tok_counts, as_stream(stream)));
}

moe_status moe_ep_token_base(const moe_config *c, int32_t world, int32_t rank,
                             const int32_t *tok_counts_all, int32_t *tok_base, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world) || rank < 0 || rank >= world) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!tok_counts_all || !tok_base) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    return cuda_status(launch_ep_token_base(tok_counts_all, world, rank, tok_base,
                                            as_stream(stream)));
}

moe_status moe_ep_dispatch_dedup(const moe_config *c, int32_t world, const void *x,
                                 const int32_t *topk_idx, const int32_t *offsets,
                                 const int32_t *inv_perm, const int32_t *base,
                                 const int32_t *tok_slot, const int32_t *tok_base,
                                 void *const *recv_tok, int32_t *const *recv_idx,
                                 int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!x || !topk_idx || !offsets || !inv_perm || !base || !tok_slot ||
                     !tok_base || !recv_tok || !recv_idx))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t tok_rows = (int64_t)world * c->T;
    const int64_t cap = tok_rows * c->K;
    return cuda_status(launch_ep_dispatch_dedup(x, topk_idx, offsets, inv_perm, base, tok_slot,
                                                tok_base, recv_tok, recv_idx, tok_rows, cap, c->T,
                                                c->d, c->E, c->K, world, device_status,
                                                as_stream(stream)));
}

moe_status moe_ep_dispatch_dedup_plan(const moe_config *c, int32_t world, const void *x,
                                      const int32_t *topk_idx, const float *topk_w,
                                      const int32_t *offsets, const int32_t *inv_perm,
                                      const int32_t *base, const int32_t *tok_slot,
                                      const int32_t *tok_base, void *const *recv_tok,
                                      int32_t *const *recv_idx, int32_t *const *list,
                                      float *const *lw, int32_t *const *lcnt,
                                      int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!x || !topk_idx || !topk_w || !offsets || !inv_perm || !base ||
                     !tok_slot || !tok_base || !recv_tok || !recv_idx || !list || !lw || !lcnt))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t tok_rows = (int64_t)world * c->T;
    return cuda_status(launch_ep_dispatch_dedup(x, topk_idx, offsets, inv_perm, base, tok_slot,
                                                tok_base, recv_tok, recv_idx, tok_rows,
                                                tok_rows * c->K, c->T, c->d, c->E, c->K, world,
                                                device_status, as_stream(stream), topk_w, list,
                                                lw, lcnt));
}

moe_status moe_ep_fanout(const moe_config *c, int32_t world, const void *recv_tok,
                         const int32_t *recv_idx, const int32_t *local_offsets, void *recv_x,
                         int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!recv_tok || !recv_idx || !local_offsets || !recv_x))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(recv_tok) || !aligned16(recv_x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t tok_rows = (int64_t)world * c->T;
    return cuda_status(launch_ep_fanout(recv_tok, recv_idx, local_offsets, c->E / world, tok_rows,
                                        tok_rows * c->K, c->d, recv_x, device_status,
                                        as_stream(stream)));
}

moe_status moe_ep_dispatch_dedup_fp8(const moe_config *c, int32_t world, const void *x,
                                     const int32_t *topk_idx, const int32_t *offsets,
                                     const int32_t *inv_perm, const int32_t *base,
                                     const int32_t *tok_slot, const int32_t *tok_base,
                                     void *const *recv_tq, void *const *recv_ts,
                                     int32_t *const *recv_idx, int32_t *device_status,
                                     void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world) || c->d % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!x || !topk_idx || !offsets || !inv_perm || !base || !tok_slot ||
                     !tok_base || !recv_tq || !recv_ts || !recv_idx))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t tok_rows = (int64_t)world * c->T;
    return cuda_status(launch_ep_dispatch_dedup_fp8(x, topk_idx, offsets, inv_perm, base,
                                                    tok_slot, tok_base, recv_tq, recv_ts,
                                                    recv_idx, tok_rows, tok_rows * c->K, c->T,
                                                    c->d, c->E, c->K, world, device_status,
                                                    as_stream(stream)));
}

moe_status moe_ep_fanout_fp8(const moe_config *c, int32_t world, const uint8_t *recv_tq,
                             const float *recv_ts, const int32_t *recv_idx,
                             const int32_t *local_offsets, uint8_t *recv_q, float *recv_scale,
                             int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world) || c->d % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!recv_tq || !recv_ts || !recv_idx || !local_offsets || !recv_q ||
                     !recv_scale))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(recv_tq) || !aligned16(recv_q)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t tok_rows = (int64_t)world * c->T;
    return cuda_status(launch_ep_fanout_fp8(recv_tq, recv_ts, recv_idx, local_offsets,
                                            c->E / world, tok_rows, tok_rows * c->K, c->d,
                                            recv_q, recv_scale, device_status,
                                            as_stream(stream)));
}

moe_status moe_ep_combine_plan(const moe_config *c, int32_t world, const int32_t *topk_idx,
                               const float *topk_w, const int32_t *offsets,
                               const int32_t *inv_perm, const int32_t *base,
                               const int32_t *tok_slot, const int32_t *tok_base,
                               int32_t *const *list, float *const *lw, int32_t *const *lcnt,
                               int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!topk_idx || !topk_w || !offsets || !inv_perm || !base || !tok_slot ||
                     !tok_base || !list || !lw || !lcnt))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t tok_rows = (int64_t)world * c->T;
    return cuda_status(launch_ep_combine_plan(topk_idx, topk_w, offsets, inv_perm, base, tok_slot,
                                              tok_base, list, lw, lcnt, tok_rows,
                                              tok_rows * c->K, c->T, c->E, c->K, world,
                                              device_status, as_stream(stream)));
}

moe_status moe_ep_precombine(const moe_config *c, int32_t world, const void *recv_y,
                             const int32_t *list, const float *lw, const int32_t *lcnt,
                             const int32_t *tok_base, void *partial, int32_t *device_status,
                             void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!recv_y || !list || !lw || !lcnt || !tok_base || !partial))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(recv_y) || !aligned16(partial)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t tok_rows = (int64_t)world * c->T;
    return cuda_status(launch_ep_precombine(recv_y, list, lw, lcnt, tok_base, world, tok_rows,
                                            tok_rows * c->K, c->d, c->K, partial, device_status,
                                            as_stream(stream)));
}

moe_status moe_ep_combine_dedup(const moe_config *c, int32_t world, const int32_t *topk_idx,
                                const int32_t *tok_slot, const int32_t *tok_base,
                                const void *const *partial, const void *y_shared, void *out,
                                int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!topk_idx || !tok_slot || !tok_base || !partial || !out))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_shared) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    return cuda_status(launch_ep_combine_dedup(topk_idx, tok_slot, tok_base, partial, y_shared,
                                               (int64_t)world * c->T, c->T, c->d, c->E, c->K,
                                               world, out, device_status, as_stream(stream)));
}

namespace {
// the expert FFN of one rank's experts over its receive buffer: bf16 rows
// (recv_x) or FP8 codes + scales (recv_q, recv_scale)
moe_status ep_expert_ffn(const moe_config *c, int32_t world, int32_t rank, bool fp8,
                         const void *recv_x,
                         const uint8_t *recv_q, const float *recv_scale,
                         const int32_t *local_offsets, const void *w_gate, const void *w_up,
                         const void *w_down, void *recv_y, const void *x, const void *ws_gate,
                         const void *ws_up, const void *ws_down, void *y_shared, void *ws,
                         size_t ws_bytes, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world) || rank < 0 || rank >= world) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (fp8 && c->d % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (c->T > 0) {
        if (fp8 ? (!recv_q || !recv_scale || !x) : !recv_x) return MOE_ERR_INVALID_ARG;
        if (!local_offsets || !w_gate || !w_up || !w_down || !recv_y) return MOE_ERR_INVALID_ARG;
        if (c->n_shared > 0 && (!x || !ws_gate || !ws_up || !ws_down || !y_shared))
            return MOE_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {recv_x, recv_q, recv_scale, w_gate, w_up, w_down, recv_y, x,
                          ws_gate, ws_up, ws_down, y_shared};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    const moe_config g = ep_global(c, world);
    const Layout L = layout(g);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    // the local experts over the received rows: world * T * K rows of capacity
    // (every copy of every rank could come here), this rank's T tokens for the
    // shared experts
    FfnArgs a{};
    a.T = c->T; a.d = c->d; a.E = c->E / world; a.K = c->K * world; a.d_ff = c->d_ff;
    a.n_shared = c->n_shared; a.d_ff_shared = c->d_ff_shared;
    a.x_perm = recv_x; a.perm_token = nullptr; a.offsets = local_offsets;
    a.x_perm_q = recv_q; a.x_scale = recv_scale;
    a.w_gate = w_gate; a.w_up = w_up; a.w_down = w_down;
    a.h = at<void>(ws, L.h); a.y_perm = recv_y;
    a.x = x; a.ws_gate = ws_gate; a.ws_up = ws_up; a.ws_down = ws_down;
    a.h_shared = at<void>(ws, L.h_sh); a.y_shared = y_shared;
    a.status = at<int32_t>(ws, L.status);
    a.timeout_ns = kWaitTimeoutNs;
    return cuda_status(launch_expert_ffn(a, as_stream(stream)));
}
}  // namespace

moe_status moe_ep_expert_ffn_fp8(const moe_config *c, int32_t world, int32_t rank,
                                 const uint8_t *recv_q, const float *recv_scale,
                                 const int32_t *local_offsets, const void *w_gate,
                                 const void *w_up, const void *w_down, void *recv_y, const void *x,
                                 const void *ws_gate, const void *ws_up, const void *ws_down,
                                 void *y_shared, void *ws, size_t ws_bytes, void *stream) {
    return ep_expert_ffn(c, world, rank, true, nullptr, recv_q, recv_scale, local_offsets, w_gate,
                         w_up, w_down, recv_y, x, ws_gate, ws_up, ws_down, y_shared, ws, ws_bytes,
                         stream);
}

moe_status moe_ep_expert_ffn(const moe_config *c, int32_t world, int32_t rank, const void *recv_x,
                             const int32_t *local_offsets, const void *w_gate, const void *w_up,
                             const void *w_down, void *recv_y, const void *x, const void *ws_gate,
                             const void *ws_up, const void *ws_down, void *y_shared, void *ws,
                             size_t ws_bytes, void *stream) {
    return ep_expert_ffn(c, world, rank, false, recv_x, nullptr, nullptr, local_offsets, w_gate,
                         w_up, w_down, recv_y, x, ws_gate, ws_up, ws_down, y_shared, ws, ws_bytes,
                         stream);
}

moe_status moe_ep_combine(const moe_config *c, int32_t world, const int32_t *topk_idx,
                          const float *topk_w, const int32_t *offsets, const int32_t *inv_perm,
                          const int32_t *base, const void *const *recv_y, const void *y_shared,
                          void *out, int32_t *device_status, void *stream) {
    moe_status st = moe_check_config(c);
    if (st) return st;
    if (!ep_args_ok(c, world)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (c->T > 0 && (!topk_idx || !topk_w || !offsets || !inv_perm || !base || !recv_y || !out))
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_shared) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if ((st = check_device())) return st;
    const int64_t cap = (int64_t)world * c->T * c->K;
    return cuda_status(launch_ep_combine(topk_idx, topk_w, offsets, inv_perm, base, recv_y, cap,
                                         y_shared, c->T, c->d, c->E, c->K, world, out,
                                         device_status, as_stream(stream)));
}

moe_status moe_ipc_get_handle(const void *dev_ptr, void *handle) {
    if (!dev_ptr || !handle) return MOE_ERR_INVALID_ARG;
    moe_status st = check_device();
    if (st) return st;
    // the handle names the whole allocation holding dev_ptr (a caching
    // allocator may place a buffer inside a larger one): send the offset too
    CUdeviceptr base = 0;
    size_t bytes = 0;
    if (!ipc_addr_range(dev_ptr, &base, &bytes)) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess)
        return MOE_ERR_CUDA;
    static_assert(sizeof(h) + sizeof(uint64_t) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
    const uint64_t off = reinterpret_cast<uintptr_t>(dev_ptr) - (uintptr_t)base;
    std::memcpy(handle, &h, sizeof(h));
    std::memcpy(static_cast<char *>(handle) + sizeof(h), &off, sizeof(off));
    return MOE_OK;
}

moe_status moe_ipc_open_handle(const void *handle, void **dev_ptr) {
    if (!handle || !dev_ptr) return MOE_ERR_INVALID_ARG;
    moe_status st = check_device();
    if (st) return st;
    cudaIpcMemHandle_t h;
    uint64_t off = 0;
    std::memcpy(&h, handle, sizeof(h));
    std::memcpy(&off, static_cast<const char *>(handle) + sizeof(h), sizeof(off));
    void *base = nullptr;
    if ((st = cuda_status(cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess))))
        return st;
    *dev_ptr = static_cast<char *>(base) + off;
    std::lock_guard<std::mutex> lock(ipc_mutex());
    auto it = ipc_opened().find(*dev_ptr);
    if (it == ipc_opened().end())
        ipc_opened().emplace(*dev_ptr, IpcOpened{base, 1});
    else
        ++it->second.opens;
    return MOE_OK;
}

moe_status moe_ipc_close_handle(void *dev_ptr) {
    if (!dev_ptr) return MOE_ERR_INVALID_ARG;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(ipc_mutex());
        auto it = ipc_opened().find(dev_ptr);
        if (it == ipc_opened().end()) return MOE_ERR_INVALID_ARG;  // not from open_handle
        base = it->second.base;
        if (--it->second.opens == 0) ipc_opened().erase(it);
    }
    moe_status st = check_device();
    if (st) return st;
    return cuda_status(cudaIpcCloseMemHandle(base));
}

moe_status moe_selftest_bounded_wait(int64_t timeout_ns, void *ws, void *stream) {
    if (!ws || timeout_ns < 1000 || timeout_ns > 10000000000LL) return MOE_ERR_INVALID_ARG;
    moe_status st = check_device();
    if (st) return st;
    return cuda_status(launch_bounded_wait_selftest(timeout_ns, static_cast<int32_t *>(ws),
                                                    as_stream(stream)));
}

}  // extern "C"
