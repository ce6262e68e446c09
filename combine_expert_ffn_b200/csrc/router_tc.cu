// router_tc.cu -- router affinities on the tensor cores.
//
//   s_i = f(x . e_i + o_i)      x bf16 [T, d], e fp32 [E, d]
// (top-k gating over expert affinities, "MoE + Expert-Parallel Overlap
// (Exp08)", Implemented; f is DeepSeek-V3's sigmoid, or the V4 form
// sqrt(softplus(L)) named there; o_i is the optional per-expert logit offset
// of the skewed-load workload.)
//
// The fp32 weights are split into three bf16 parts, e = hi + mid + lo to
// about 2^-27 relative (each subtraction exact in fp32), so every product
// x_k * part_k is exact on the tensor cores.  The tensor core's fp32
// accumulator loses low-order bits over long chains of MMAs, so it is used for
// one 64-wide k block at a time: the 12 MMAs of a block (lo, mid, hi parts x 4
// k-steps) land in a fresh TMEM buffer, and the epilogue warps add that
// partial sum into IEEE fp32 registers.  Affinities then agree with the
// double-precision definition to a few 1e-7 at V3 scale.
//
// Small batches leave most SMs idle (a decode batch of 128 tokens and 256
// experts is 2 tiles), so the reduction over d is split into `splits` ranges
// of k blocks (router_splits): each work item writes its partial logits, and
// router_finish_kernel adds them in split order and applies the affinity.
//
// Persistent kernel, one CTA per SM, tile = 128 tokens x 128 experts:
//   warp 0      TMA: x tile (128 x 64) + the three weight parts (3 x 128 x 64)
//               per stage, 3 stages of 64 KB
//   warp 1      TMEM owner (4 buffers x 128 columns), single-thread MMA issuer
//   warps 2..5  epilogue: per k block, TMEM -> registers (+=); per tile,
//               f -> fp32 scores
#include "kernels.h"

#include <algorithm>

namespace moe {
namespace router {

constexpr int BM = 128, BN = 128, BK = 64;
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + 3 * B_BYTES;  // 64 KB
constexpr int NUM_THREADS = 192;
constexpr int NBUF = 4;                             // TMEM chunk buffers
constexpr int TMEM_COLS = NBUF * BN;                // 512
constexpr int SMEM_DYN = STAGES * STAGE_BYTES + 1024;

struct Maps {
    CUtensorMap x;       // [T, d]        box 64 x 128
    CUtensorMap parts;   // [3, E, d]     box 64 x 128 x 1
};

struct Params {
    int T, E, d;
    int affinity;  // 0: sigmoid, 1: sqrt(softplus)
    int splits;    // k ranges per tile; > 1: partial logits go to `partial`
    float *partial;  // [splits, T, E] fp32 (splits > 1)
    const float *off;
    float *scores;
    int32_t *status;
    int64_t timeout_ns;
};

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, int64_t timeout_ns,
                                           int32_t *status) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if ((int64_t)(globaltimer_ns() - t0) > timeout_ns) {
            record_status(status, MOE_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
    return true;
}

// softplus(L) = log(1 + e^L), evaluated without overflow on either side
__device__ __forceinline__ float sqrt_softplus(float L) {
    const float sp = L > 0.f ? L + log1pf(expf(-L)) : log1pf(expf(L));
    return sqrtf(sp);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
router_tc_kernel(const __grid_constant__ Maps maps, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[STAGES];
    __shared__ __align__(8) uint64_t empty_bar[STAGES];
    __shared__ __align__(8) uint64_t cfull_bar[NBUF];
    __shared__ __align__(8) uint64_t cempty_bar[NBUF];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t smem0 = smem_u32(smem);
    volatile int *abort_flag = &abort_s;

    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&maps.x);
        tma_prefetch_desc(&maps.parts);
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(smem_u32(&full_bar[s]), 1);
                mbar_init(smem_u32(&empty_bar[s]), 1);
            }
            for (int b = 0; b < NBUF; ++b) {
                mbar_init(smem_u32(&cfull_bar[b]), 1);
                mbar_init(smem_u32(&cempty_bar[b]), 128);
            }
            mbar_init(smem_u32(&done_bar), 1);
            abort_s = 0;
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc<TMEM_COLS>(smem_u32(&tmem_base_s));
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    const int mt = (p.T + BM - 1) / BM, nt = (p.E + BN - 1) / BN;
    const int total = mt * nt * p.splits;     // work items: (tile, split), split fastest
    const int kblocks = p.d / BK;
    const int kper = (kblocks + p.splits - 1) / p.splits;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, n_issued = 0;
            bool ok = true;
            for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
                const int tile = idx / p.splits, sp = idx - tile * p.splits;
                const int m0 = (tile / nt) * BM, n0 = (tile % nt) * BN;
                const int kb1 = min(kblocks, (sp + 1) * kper);
                for (int kb = sp * kper; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag,
                                           p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t dst = smem0 + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(dst, &maps.x, fb, kb * BK, m0);
#pragma unroll
                    for (int part = 0; part < 3; ++part)
                        tma_load_3d(dst + A_BYTES + part * B_BYTES, &maps.parts, fb, kb * BK, n0, part);
                    ++n_issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            for (int s = 0; s < STAGES; ++s)
                if (n_issued > (uint32_t)s)
                    drain_wait(smem_u32(&full_bar[s]), (((n_issued - 1 - s) / STAGES)) & 1u,
                               p.timeout_ns, p.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            constexpr uint32_t idesc = idesc_bf16_f32<BM, BN>();
            bool ok = true;
            for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
                const int sp = idx % p.splits;
                const int kb1 = min(kblocks, (sp + 1) * kper);
                for (int kb = sp * kper; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&cempty_bar[buf]), bphase ^ 1u, abort_flag,
                                           p.status, p.timeout_ns) ||
                        !mbar_wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, p.status,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t base = smem0 + stage * STAGE_BYTES;
                    const uint64_t a_desc = smem_desc_sw128(base);
                    const uint32_t d_tmem = tmem_base + buf * BN;
                    // smallest part first: the fresh accumulator is smallest
                    // while the smallest products are added
#pragma unroll
                    for (int part = 2; part >= 0; --part) {
                        const uint64_t b_desc = smem_desc_sw128(base + A_BYTES + part * B_BYTES);
#pragma unroll
                        for (int ks = 0; ks < BK / 16; ++ks)
                            tc_mma_bf16(d_tmem, a_desc + 2 * ks, b_desc + 2 * ks, idesc,
                                        (part == 2 && ks == 0) ? 0u : 1u);
                    }
                    tc_commit(smem_u32(&empty_bar[stage]));
                    tc_commit(smem_u32(&cfull_bar[buf]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if (++buf == NBUF) { buf = 0; bphase ^= 1u; }
                }
            }
            tc_commit(smem_u32(&done_bar));
            drain_wait(smem_u32(&done_bar), 0, p.timeout_ns, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int row = q * 32 + lane;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
            const int tile = idx / p.splits, sp = idx - tile * p.splits;
            const int m0 = (tile / nt) * BM, n0 = (tile % nt) * BN;
            const int kb1 = min(kblocks, (sp + 1) * kper);
            float acc[BN];
#pragma unroll
            for (int c = 0; c < BN; ++c) acc[c] = 0.f;
            for (int kb = sp * kper; kb < kb1; ++kb) {
                if (!mbar_wait_bounded(smem_u32(&cfull_bar[buf]), bphase, abort_flag, p.status,
                                       p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
#pragma unroll
                for (int c = 0; c < BN; c += 32) {
                    uint32_t v[32];
                    tmem_ld32(taddr + c, v);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[c + j] = __fadd_rn(acc[c + j], __uint_as_float(v[j]));
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&cempty_bar[buf]));
                if (++buf == NBUF) { buf = 0; bphase ^= 1u; }
            }
            if (!ok) break;
            const int t = m0 + row;
            if (t < p.T && p.splits > 1) {  // partial logits of this k range
                float *out = p.partial + ((size_t)sp * p.T + t) * p.E;
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (n0 + c < p.E) out[n0 + c] = acc[c];
            } else if (t < p.T) {
                float *out = p.scores + (size_t)t * p.E;
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const int col = n0 + c;
                    if (col < p.E) {
                        float L = acc[c];
                        if (p.off) L += p.off[col];
                        out[col] = p.affinity == 1 ? sqrt_softplus(L) : 1.0f / (1.0f + expf(-L));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

// parts[p][i][k] = part p of e[i][k]: hi = bf16(e), mid = bf16(e - hi),
// lo = bf16(e - hi - mid); each subtraction is exact in fp32.
__global__ void router_split_kernel(const float *__restrict__ e, int64_t n,
                                    __nv_bfloat16 *__restrict__ parts) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = e[i];
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const float r1 = __fsub_rn(v, __bfloat162float(hi));
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = __fsub_rn(r1, __bfloat162float(mid));
        parts[i] = hi;
        parts[n + i] = mid;
        parts[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

// scores[t][e] = f(sum over splits, in split order, of partial[s][t][e] + off[e])
__global__ void router_finish_kernel(const float *__restrict__ partial, int splits, int T, int E,
                                     const float *__restrict__ off, int affinity,
                                     float *__restrict__ scores) {
    const int64_t n = (int64_t)T * E;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        float L = partial[i];
        for (int s = 1; s < splits; ++s) L = __fadd_rn(L, partial[(size_t)s * n + i]);
        if (off) L += off[i % E];
        scores[i] = affinity == 1 ? sqrt_softplus(L) : 1.0f / (1.0f + expf(-L));
    }
}

}  // namespace router

cudaError_t launch_router_split(const float *e, int E, int d, void *e_split, cudaStream_t st) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t n = (int64_t)E * d;
    router::router_split_kernel<<<(int)std::min<int64_t>((n + 255) / 256, (int64_t)sms * 8), 256,
                                  0, st>>>(e, n, static_cast<__nv_bfloat16 *>(e_split));
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_router_logits_tc(const void *x, const float *e, const float *off, int T, int d,
                                    int E, int affinity, void *e_split, float *partial,
                                    float *scores, int32_t *status, int64_t timeout_ns,
                                    cudaStream_t st) {
    using namespace router;
    if (T == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t err = launch_router_split(e, E, d, e_split, st);
    if (err != cudaSuccess) return err;
    Maps m;
    if (!tensor_map_2d_bf16(&m.x, x, T, d, BK, BM) ||
        !tensor_map_3d_bf16(&m.parts, e_split, 3, E, d, BK, BN))
        return cudaErrorInvalidValue;
    const int splits = router_splits(T, E, d);
    if (splits > 1 && !partial) return cudaErrorInvalidValue;
    Params p{T, E, d, affinity, splits, partial, off, scores, status, timeout_ns};
    err = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
    if (err != cudaSuccess) return err;
    const int items = ((T + BM - 1) / BM) * ((E + BN - 1) / BN) * splits;
    router_tc_kernel<<<std::min(items, sms), NUM_THREADS, SMEM_DYN, st>>>(m, p);
    count_launch();
    if ((err = cudaGetLastError()) != cudaSuccess || splits == 1) return err;
    const int64_t n_out = (int64_t)T * E;
    router_finish_kernel<<<(int)std::min<int64_t>((n_out + 255) / 256, (int64_t)sms * 8), 256, 0,
                           st>>>(partial, splits, T, E, off, affinity, scores);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
