// common.cuh -- small device helpers shared by the kernels of libgqa.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gqa.h"

namespace gqa {

// ---------------------------------------------------------------------------
// bf16 <-> fp32 (bit-level; bf16 is the upper half of a binary32)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> packed bf16x2 with round-to-nearest-even (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ void report(int32_t *status, int32_t bits) {
    if (status) atomicOr(status, bits);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 2^x on the special-function unit (the hardware instruction, flush-to-zero).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace gqa

// ---------------------------------------------------------------------------
// host-side helpers
// ---------------------------------------------------------------------------
namespace gqa_host {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool head_dim_ok(int D) { return D == 64 || D == 96 || D == 128; }

inline gqa_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace gqa_host
