// efla_common.cuh - shared device helpers of the EFLA CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace efla {

// Sticky device error word: a kernel whose bounded wait gives up ORs a
// reason bit in here and returns; efla_last_error() reads and clears it.
// The library is one translation unit (efla_api.cu includes every kernel
// header), so the definition lives here.
__device__ unsigned int g_error_word = 0u;

enum : unsigned int { kErrTimeout = 1u };

__device__ __forceinline__ void raise_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

// Exact-flow gate of "Exact Flow Linear Attention" (papernotes.org summary,
// 关键设计 2): alpha = (1 - e^{-beta*lambda}) / lambda, evaluated as
// -expm1(-beta*lc)/lc with lc = max(lambda, 1e-12) (section 损失函数 /
// 训练策略).  The comparison form keeps a NaN lambda mapped to the clamp,
// exactly as the fp64 oracle does.  `euler` selects alpha = beta
// (DeltaNet, 关键设计 1).
__device__ __forceinline__ float gate_alpha(float beta, float lambda, bool euler) {
    if (euler) return beta;
    const float lc = lambda > 1e-12f ? lambda : 1e-12f;
    return -expm1f(-beta * lc) / lc;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load 4 consecutive elements (16-byte aligned for fp32, 8-byte for bf16)
// widened to fp32.
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}

__device__ __forceinline__ float warp_sum(float x, unsigned mask = 0xffffffffu) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(mask, x, o);
    return x;
}

// Opt a kernel into more than 48 KB of dynamic shared memory once per
// device.  Later calls (including ones made while a stream is being
// captured into a CUDA graph) skip the runtime call.
template <auto Kernel>
inline bool ensure_smem(size_t bytes) {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return true;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return true;
}

}  // namespace efla
