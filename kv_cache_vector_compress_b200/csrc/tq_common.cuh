// tq_common.cuh -- small device helpers shared by the kernels of libtq.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace tq {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ uint16_t f32_to_f16_bits(float v) {
    return __half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

// Code of y against an ascending boundary list: #{k : b[k] < y} (ties to the lower cell).
__device__ __forceinline__ int bucketize(const float *b, int nb, float y) {
    int c = 0;
    for (int k = 0; k < nb; ++k) c += (b[k] < y) ? 1 : 0;
    return c;
}

}  // namespace tq
