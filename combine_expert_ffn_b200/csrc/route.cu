// route.cu -- router affinity and node-limited top-K selection.
//
// Affinity: s_i = sigmoid(x . e_i + o_i) with bf16 x, fp32 e, fp32
// accumulation (top-k gating over expert affinities, "MoE + Expert-Parallel
// Overlap (Exp08)", Implemented; the sigmoid form is DeepSeek-V3's).
// Selection: b_i = s_i + bias_i chooses, s_i weights; experts lie in at most M
// of the G contiguous groups ("moe-node-limited-routing", opening definition);
// a group scores the sum of its top-(K/M) b; ties go to the lower index.
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------- logits
// L[t, i] = sum_k x[t, k] * e[i, k] in fp32 on the CUDA cores (the tile is
// 128 tokens x 64 experts, each thread owns an 8 x 8 block of outputs), then
// s = 1 / (1 + expf(-(L + o_i))).
namespace {
constexpr int RL_BM = 128, RL_BN = 64, RL_BK = 32, RL_THREADS = 128;
constexpr int RL_XS = RL_BM + 4;  // padded row (floats) of the transposed x tile
constexpr int RL_ES = RL_BN + 4;
}  // namespace

__global__ void __launch_bounds__(RL_THREADS)
router_logits_kernel(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ e,
                     const float *__restrict__ off, int T, int d, int E,
                     float *__restrict__ scores) {
    __shared__ __align__(16) float xs[RL_BK][RL_XS];
    __shared__ __align__(16) float es[RL_BK][RL_ES];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.x * RL_BM, n0 = blockIdx.y * RL_BN;
    const int tx = tid % 8, ty = tid / 8;  // 8 expert columns x 16 token rows of threads

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += RL_BK) {
        // x tile: 128 rows x 32 k of bf16 = 512 chunks of 8; 4 per thread.
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int c = tid + p * RL_THREADS;
            const int m = c / 4, kc = (c % 4) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m0 + m < T) v = *reinterpret_cast<const uint4 *>(x + (size_t)(m0 + m) * d + k0 + kc);
            xs[kc + 0][m] = bf16_lo(v.x);
            xs[kc + 1][m] = bf16_hi(v.x);
            xs[kc + 2][m] = bf16_lo(v.y);
            xs[kc + 3][m] = bf16_hi(v.y);
            xs[kc + 4][m] = bf16_lo(v.z);
            xs[kc + 5][m] = bf16_hi(v.z);
            xs[kc + 6][m] = bf16_lo(v.w);
            xs[kc + 7][m] = bf16_hi(v.w);
        }
        // e tile: 64 experts x 32 k fp32 = 512 float4; 4 per thread.
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int c = tid + p * RL_THREADS;
            const int n = c / 8, kc = (c % 8) * 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n0 + n < E) v = *reinterpret_cast<const float4 *>(e + (size_t)(n0 + n) * d + k0 + kc);
            es[kc + 0][n] = v.x;
            es[kc + 1][n] = v.y;
            es[kc + 2][n] = v.z;
            es[kc + 3][n] = v.w;
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < RL_BK; ++k) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&xs[k][ty * 8]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&xs[k][ty * 8 + 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&es[k][tx * 8]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&es[k][tx * 8 + 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = m0 + ty * 8 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int n = n0 + tx * 8 + j;
            if (n >= E) continue;
            float L = acc[i][j];
            if (off) L += off[n];
            scores[(size_t)t * E + n] = 1.0f / (1.0f + expf(-L));
        }
    }
}

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
cudaError_t launch_router_logits(const void *x, const float *e, const float *off, int T, int d,
                                 int E, float *scores, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    dim3 grid((T + RL_BM - 1) / RL_BM, (E + RL_BN - 1) / RL_BN);
    router_logits_kernel<<<grid, RL_THREADS, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), e,
                                                      off, T, d, E, scores);
    count_launch();
    return cudaGetLastError();
}

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
