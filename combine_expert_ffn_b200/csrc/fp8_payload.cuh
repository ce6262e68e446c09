// fp8_payload.cuh -- the FP8 E4M3 dispatch payload of one 16-byte chunk.
//
// "DeepSeek 8.7 -- communication", section 4 (compression trades bytes for a
// quantize/dequantize step and its error): one fp32 scale per token and
// 128-channel block, s = amax / 448 (fp32 division), q = E4M3(x / s) with
// round-to-nearest-even and saturation to +-448; an all-zero block gives s = 0
// and q = 0.  The single-GPU FP8 gather and the expert-parallel FP8 dispatch
// both quantize through this one function, so their codes are identical.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// Called by all 32 lanes of a warp.  Lanes 16g .. 16g+15 hold the 16 chunks
// (8 bf16 channels each) of one 128-channel block; lanes without data pass
// zeros.  Returns this lane's 8 codes; *scale = the block's s.
__device__ __forceinline__ uint2 e4m3_quantize_chunk(const uint4 v, float *scale) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        f[2 * j] = bf16_lo(w[j]);
        f[2 * j + 1] = bf16_hi(w[j]);
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float sc = __fdiv_rn(amax, 448.0f);
    uint32_t q[2] = {0u, 0u};
    if (amax > 0.f) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(
                make_float2(__fdiv_rn(f[2 * j], sc), __fdiv_rn(f[2 * j + 1], sc)),
                __NV_SATFINITE, __NV_E4M3);
            q[j >> 1] |= (uint32_t)b << (16 * (j & 1));
        }
    }
    *scale = sc;
    return make_uint2(q[0], q[1]);
}

}  // namespace moe
