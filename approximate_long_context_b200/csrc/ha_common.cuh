// ha_common.cuh -- small device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ha {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// Load element i of a row of type T (0 = bf16, 1 = fp32) as float.
__device__ __forceinline__ float load_elem(const void *base, int64_t i, int dtype) {
    if (dtype == 0) return bf16_bits_to_float(static_cast<const uint16_t *>(base)[i]);
    return static_cast<const float *>(base)[i];
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem_src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void store_out(void *O, int64_t i, float v, int out_dtype) {
    if (out_dtype == 0) static_cast<__nv_bfloat16 *>(O)[i] = __float2bfloat16_rn(v);
    else static_cast<float *>(O)[i] = v;
}

}  // namespace ha
