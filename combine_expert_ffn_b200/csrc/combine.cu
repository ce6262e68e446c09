// combine.cu -- gate-weighted un-permute and reduce back to token order.
//
// The combine all-to-all ("moe-node-limited-routing", "Why all to all
// dominates MoE step time": outputs return to the token's origin) is a
// gather-reduce on one GPU:
//   out[t] = y_shared[t] + sum_j w[t, j] * y_perm[inv_perm[t, j]]
// in fp32, rounded once to bf16.  HBM-bound: per token K + 1 rows read, one
// written; every thread moves 16-byte chunks and keeps K + 1 loads in flight.
#include "kernels.h"

namespace moe {

namespace {
constexpr int CB_THREADS = 256;

__device__ __forceinline__ void acc_row(float (&acc)[8], float wj, const uint4 &v) {
    acc[0] = fmaf(wj, bf16_lo(v.x), acc[0]); acc[1] = fmaf(wj, bf16_hi(v.x), acc[1]);
    acc[2] = fmaf(wj, bf16_lo(v.y), acc[2]); acc[3] = fmaf(wj, bf16_hi(v.y), acc[3]);
    acc[4] = fmaf(wj, bf16_lo(v.z), acc[4]); acc[5] = fmaf(wj, bf16_hi(v.z), acc[5]);
    acc[6] = fmaf(wj, bf16_lo(v.w), acc[6]); acc[7] = fmaf(wj, bf16_hi(v.w), acc[7]);
}
}  // namespace

// KB = slots loaded per batch (all K at once when K <= 8, so that every row
// load of a chunk is in flight together); slots are accumulated in slot order.
template <int KB>
__global__ void __launch_bounds__(CB_THREADS)
combine_kernel(const uint4 *__restrict__ y_perm, const int32_t *__restrict__ inv_perm,
               const float *__restrict__ topk_w, const uint4 *__restrict__ y_shared, int T,
               int chunks, int K, int64_t n_rows, uint4 *__restrict__ out) {
    const int64_t total = (int64_t)T * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        float acc[8];
        if (y_shared) {
            const uint4 v = __ldg(y_shared + i);
            acc[0] = bf16_lo(v.x); acc[1] = bf16_hi(v.x);
            acc[2] = bf16_lo(v.y); acc[3] = bf16_hi(v.y);
            acc[4] = bf16_lo(v.z); acc[5] = bf16_hi(v.z);
            acc[6] = bf16_lo(v.w); acc[7] = bf16_hi(v.w);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        }
        for (int j0 = 0; j0 < K; j0 += KB) {
            uint4 rows[KB];
            float w[KB];
#pragma unroll
            for (int q = 0; q < KB; ++q) {
                const int j = j0 + q;
                rows[q] = make_uint4(0, 0, 0, 0);
                w[q] = 0.f;
                if (j < K) {
                    const int r = __ldg(inv_perm + t * K + j);
                    w[q] = __ldg(topk_w + t * K + j);
                    if (r >= 0 && r < n_rows) rows[q] = __ldg(y_perm + (int64_t)r * chunks + c);
                }
            }
#pragma unroll
            for (int q = 0; q < KB; ++q)
                if (j0 + q < K) acc_row(acc, w[q], rows[q]);
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        out[i] = o;
    }
}

cudaError_t launch_combine(const void *y_perm, const int32_t *inv_perm, const float *topk_w,
                           const void *y_shared, int T, int d, int K, int64_t n_rows, void *out,
                           cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int chunks = d / 8;
    const int64_t total = (int64_t)T * chunks;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (total + CB_THREADS - 1) / CB_THREADS;
    const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    const uint4 *yp = static_cast<const uint4 *>(y_perm);
    const uint4 *ys = static_cast<const uint4 *>(y_shared);
    uint4 *o = static_cast<uint4 *>(out);
    if (K <= 4)
        combine_kernel<4><<<grid, CB_THREADS, 0, st>>>(yp, inv_perm, topk_w, ys, T, chunks, K, n_rows, o);
    else
        combine_kernel<8><<<grid, CB_THREADS, 0, st>>>(yp, inv_perm, topk_w, ys, T, chunks, K, n_rows, o);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
