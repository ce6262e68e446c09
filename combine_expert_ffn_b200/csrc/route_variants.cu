// route_variants.cu -- the two routing variants beside the learned router
// ("MoE + Expert-Parallel Overlap (Exp08)", Implemented: a hash router for
// early-layer emulation, and auxiliary-loss-free balancing through
// per-expert bias updates).
//
// Hash router.  The page gives no formula, so the rule is a reading that keeps
// the node limit of the learned router: a token takes M of the G groups and
// K/M experts in each, both drawn without replacement by a partial
// Fisher-Yates shuffle whose draws come from the lowbias32 integer hash
// (C. Wellons, hash-prospector) of the 64-bit token id; every gate is 1/K.
//   seed     s0  = h(lo32(id) ^ h(hi32(id) ^ 0x68E31DA4))
//   groups   draw i of [0, G): j_i = i + h(s0 ^ i*0x9E3779B9) mod (G - i)
//   group g  seed  h(s0 ^ (g+1)*0x85EBCA6B), the same draws over [0, E/G)
// Slots hold the groups in draw order, each group's K/M experts in draw order.
//
// Bias update (DeepSeek-V3's sign rule; the step size gamma is a parameter):
//   bias_i <- bias_i + gamma * sign(T*K/E - counts_i)
// with the mean compared exactly, counts_i * E against T * K in 64-bit
// integers, and one IEEE fp32 add.
#include "kernels.h"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t lowbias32(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7FEB352Du;
    x ^= x >> 15;
    x *= 0x846CA68Bu;
    x ^= x >> 16;
    return x;
}

// After the swaps (k, j[k]) for k < i of the array a[p] = p, the value at
// position p is found by undoing them from the last to the first.
__device__ __forceinline__ uint32_t value_after_swaps(uint32_t p, const uint32_t *j, int i) {
    for (int k = i - 1; k >= 0; --k) {
        if (p == (uint32_t)k) p = j[k];
        else if (p == j[k]) p = (uint32_t)k;
    }
    return p;
}

// The first m draws of the shuffle of [0, n) seeded by `seed` (m <= n).
template <int MAXM>
__device__ __forceinline__ void shuffle_draws(uint32_t n, int m, uint32_t seed, uint32_t *out) {
    uint32_t j[MAXM];
    for (int i = 0; i < m; ++i) {
        j[i] = (uint32_t)i + lowbias32(seed ^ ((uint32_t)i * 0x9E3779B9u)) % (n - (uint32_t)i);
        out[i] = value_after_swaps(j[i], j, i);
    }
}

// One thread per token.
__global__ void hash_route_kernel(const int64_t *__restrict__ token_ids, int T, int E, int G,
                                  int K, int M, int32_t *__restrict__ topk_idx,
                                  float *__restrict__ topk_w) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const uint64_t id = token_ids ? (uint64_t)token_ids[t] : (uint64_t)t;
    const uint32_t s0 = lowbias32((uint32_t)id ^ lowbias32((uint32_t)(id >> 32) ^ 0x68E31DA4u));
    const int gsz = E / G, kpg = K / M;
    const float w = 1.0f / (float)K;  // correctly rounded: K is a small integer
    uint32_t groups[64];
    shuffle_draws<64>((uint32_t)G, M, s0, groups);
    int32_t *idx = topk_idx + (size_t)t * K;
    float *wt = topk_w + (size_t)t * K;
    for (int gi = 0; gi < M; ++gi) {
        const uint32_t g = groups[gi];
        uint32_t local[32];
        shuffle_draws<32>((uint32_t)gsz, kpg, lowbias32(s0 ^ ((g + 1u) * 0x85EBCA6Bu)), local);
        for (int q = 0; q < kpg; ++q) {
            idx[gi * kpg + q] = (int32_t)(g * (uint32_t)gsz + local[q]);
            wt[gi * kpg + q] = w;
        }
    }
}

__global__ void bias_update_kernel(const int32_t *__restrict__ counts, int E, int64_t total,
                                   float gamma, float *__restrict__ bias) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= E) return;
    const int64_t c = (int64_t)counts[i] * E;
    const float step = c < total ? gamma : (c > total ? -gamma : 0.0f);
    bias[i] = __fadd_rn(bias[i], step);
}

}  // namespace

cudaError_t launch_hash_route(const int64_t *token_ids, int T, int E, int G, int K, int M,
                              int32_t *topk_idx, float *topk_w, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    hash_route_kernel<<<(T + 127) / 128, 128, 0, st>>>(token_ids, T, E, G, K, M, topk_idx, topk_w);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_bias_update(const int32_t *counts, int E, int T, int K, float gamma,
                               float *bias, cudaStream_t st) {
    bias_update_kernel<<<(E + 255) / 256, 256, 0, st>>>(counts, E, (int64_t)T * K, gamma, bias);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
