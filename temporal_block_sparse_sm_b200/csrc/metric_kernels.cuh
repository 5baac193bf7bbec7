// metric_kernels.cuh -- error of an attention output against a reference
// output, for calibrating thresholds against per-step error budgets
// ("LiteAttention: Temporal Sparse Attention for Diffusion Transformers",
// Architecture Overview: Accumulated-Error Calibration).  Not part of a step.
#pragma once

#include <cstdint>

#include "liteattn_internal.cuh"

namespace lite {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// n8 groups of 8 bf16 (16 bytes) of each tensor; grid-stride, fp64 sums per
// thread, warp reduction, three atomics per warp.  Memory-bound: 4 bytes read
// per element pair.
__global__ void output_error_kernel(const uint4 *o, const uint4 *ref, int64_t n8, ErrAcc *acc) {
    double sd = 0.0, sr = 0.0;
    float mx = 0.0f;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const uint4 a = __ldg(o + i), b = __ldg(ref + i);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
        float fd = 0.0f, fr = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float d0 = fabsf(bf16_lo(aw[k]) - bf16_lo(bw[k])), d1 = fabsf(bf16_hi(aw[k]) - bf16_hi(bw[k]));
            fd += d0 + d1;   // the 8 differences of one group summed in fp32, then added in fp64
            fr += fabsf(bf16_lo(bw[k])) + fabsf(bf16_hi(bw[k]));
            mx = fmaxf(mx, fmaxf(d0, d1));
        }
        sd += static_cast<double>(fd);
        sr += static_cast<double>(fr);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        sd += __shfl_down_sync(0xFFFFFFFFu, sd, off);
        sr += __shfl_down_sync(0xFFFFFFFFu, sr, off);
        mx = fmaxf(mx, __shfl_down_sync(0xFFFFFFFFu, mx, off));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&acc->sum_diff, sd);
        atomicAdd(&acc->sum_ref, sr);
        atomicMax(&acc->max_bits, __float_as_uint(mx));
    }
}

}  // namespace lite
