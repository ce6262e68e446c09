// route.cu -- node-limited top-K selection (the affinities s_i = f(x . e_i +
// o_i) come from the tensor-core router in router_tc.cu; top-k gating over
// expert affinities, "MoE + Expert-Parallel Overlap (Exp08)", Implemented; f is
// DeepSeek-V3's sigmoid or the V4 sqrt(softplus)).
// Selection: b_i = s_i + bias_i chooses, s_i weights; experts lie in at most M
// of the G contiguous groups ("moe-node-limited-routing", opening definition);
// a group scores the sum of its top-(K/M) b; ties go to the lower index.
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------- select
// One warp per token.  Keys order (b desc, index asc) as one unsigned 64-bit
// value: orderable(b) in the high word, ~index in the low word, so the
// maximum key is the best expert and "strictly below the previous pick"
// replaces any taken-mask.
namespace {
constexpr int SEL_WARPS = 8;
__device__ __forceinline__ uint64_t sel_key(float b, int i) {
    return ((uint64_t)orderable(b) << 32) | (uint32_t)(~(uint32_t)i);
}
__device__ __forceinline__ int pad_idx(int i) { return i + (i >> 5); }
}  // namespace

__global__ void __launch_bounds__(SEL_WARPS * 32)
route_select_kernel(const float *__restrict__ scores, const float *__restrict__ bias, int T,
                    int E, int G, int K, int M, int32_t *__restrict__ topk_idx,
                    float *__restrict__ topk_w) {
    extern __shared__ float sel_smem[];  // per warp: E + E/32 biased affinities
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int t = blockIdx.x * SEL_WARPS + warp;
    if (t >= T) return;
    const int stride = E + (E >> 5) + 1;
    float *b = sel_smem + warp * stride;
    const float *s = scores + (size_t)t * E;
    const int gsz = E / G, kpg = K / M;

    // step 2: biased affinity (one fp32 add, never fused)
    for (int i = lane; i < E; i += 32) b[pad_idx(i)] = __fadd_rn(s[i], bias ? bias[i] : 0.0f);
    __syncwarp();

    // step 3a: lane g scores group g = sum of its kpg best b, added in pick order
    uint64_t gkey[2] = {0, 0};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int g = lane + 32 * h;
        if (g >= G) continue;
        uint64_t prev = ~0ull;
        float sum = 0.f;
        for (int r = 0; r < kpg; ++r) {
            uint64_t best = 0;
            float bb = 0.f;
            for (int i = g * gsz; i < (g + 1) * gsz; ++i) {
                const float v = b[pad_idx(i)];
                const uint64_t k = sel_key(v, i);
                if (k < prev && k > best) { best = k; bb = v; }
            }
            prev = best;
            sum = (r == 0) ? bb : __fadd_rn(sum, bb);
        }
        gkey[h] = sel_key(sum, g);
    }

    // step 3b: the M best groups by warp arg-max, ties to the lower group index
    uint64_t keep = 0;  // bit g set: group g kept
    {
        uint64_t prev = ~0ull;
        for (int r = 0; r < M; ++r) {
            uint64_t cand = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                if (gkey[h] < prev && gkey[h] > cand) cand = gkey[h];
            const uint64_t best = warp_max_u64(cand);
            keep |= 1ull << (~(uint32_t)best);  // low word holds ~g
            prev = best;
        }
    }

    // step 4: top-K experts of the kept groups, in pick order
    int my_idx = 0;
    float my_s = 0.f;
    {
        uint64_t prev = ~0ull;
        for (int j = 0; j < K; ++j) {
            uint64_t cand = 0;
            for (int i = lane; i < E; i += 32) {
                if (!((keep >> (i / gsz)) & 1ull)) continue;
                const uint64_t k = sel_key(b[pad_idx(i)], i);
                if (k < prev && k > cand) cand = k;
            }
            const uint64_t best = warp_max_u64(cand);
            prev = best;
            if (lane == j) my_idx = (int)(~(uint32_t)best);
        }
    }
    // gate weights over the chosen unbiased affinities, fp32, slot order
    if (lane < K) my_s = s[my_idx];
    float denom = 0.f;
    for (int j = 0; j < K; ++j) denom = __fadd_rn(denom, __shfl_sync(0xFFFFFFFFu, my_s, j));
    if (lane < K) {
        topk_idx[(size_t)t * K + lane] = my_idx;
        topk_w[(size_t)t * K + lane] = __fdiv_rn(my_s, denom);
    }
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_route_select(const float *scores, const float *bias, int T, int E, int G,
                                int K, int M, int32_t *topk_idx, float *topk_w, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const size_t smem = sizeof(float) * SEL_WARPS * (E + (E >> 5) + 1);
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(route_select_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    route_select_kernel<<<(T + SEL_WARPS - 1) / SEL_WARPS, SEL_WARPS * 32, smem, st>>>(
        scores, bias, T, E, G, K, M, topk_idx, topk_w);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
