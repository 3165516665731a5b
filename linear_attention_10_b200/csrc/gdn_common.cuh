// gdn_common.cuh -- shared device helpers of the gated-delta-rule kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Chunk size of the chunkwise WY/UT form (Ferrite project page, Design section 03: 32 rows).
constexpr int kChunk = 32;

// Rows per step of the bf16 path: two chunks.  Its operator for the 64 rows is the 2 x 2 block
// combination of the two chunks' 32 x 32 WY/UT inverses, so that [K; Q] and [T''; P T''] fill the
// 128 rows of one M = 128 tensor-core tile and the state advances once per pair of chunks.
constexpr int kPair = 64;

// Operator record of one (pair, head) on the bf16 path: [T''; P T''] (128 x 64) as three bf16 parts
// of 16 KB in the 128-byte-swizzled K-major layout, then Gamma_i and delta_i (64 floats each).
constexpr uint32_t kPairPart = 16384;
constexpr uint32_t kPairGate = 3 * kPairPart;
constexpr uint32_t kPairRecordBytes = kPairGate + 2 * 64 * 4;

// The per-device status word lives in gdn_api.cu; kernels receive its address.
__device__ __forceinline__ void report(int* status, int code)
{
    // keep the first error: only a zero word is replaced
    atomicCAS(status, 0, code);
}

// Element access for the two storage types.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static __device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
    static __device__ __forceinline__ void st(float* p, float x) { *p = x; }
    // four consecutive elements (16-byte aligned for fp32)
    static __device__ __forceinline__ float4 ld4(const float* p)
    {
        return __ldg(reinterpret_cast<const float4*>(p));
    }
    static __device__ __forceinline__ void st4(float* p, float4 x) { *reinterpret_cast<float4*>(p) = x; }
};

template <>
struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p)
    {
        return __bfloat162float(__ldg(p));
    }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
    // four consecutive elements (8-byte aligned)
    static __device__ __forceinline__ float4 ld4(const __nv_bfloat16* p)
    {
        uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        return make_float4(fa.x, fa.y, fb.x, fb.y);
    }
    static __device__ __forceinline__ void st4(__nv_bfloat16* p, float4 x)
    {
        __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
        uint2 raw;
        raw.x = *reinterpret_cast<uint32_t*>(&a);
        raw.y = *reinterpret_cast<uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = raw;
    }
};

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace gdn
