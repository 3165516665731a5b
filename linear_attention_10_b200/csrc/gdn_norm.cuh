// gdn_norm.cuh -- L2 normalisation of raw q and k inside the library (sm_100a).
//
// The method takes L2-normalised q_t and k_t per (token, head).  With the GDN_QK_L2NORM flag the
// caller passes them raw and the library normalises: x / max(||x||_2, 1e-12), taken as
// x * rsqrt(max(sum x^2, 1e-24)) with the sum in fp32 (one reciprocal square root per vector instead
// of a square root and a divide), and the result rounded to the storage dtype -- the same steps, in
// the same order, in the prefill's pre-pass and inside the decode and verify kernels, so that every
// path sees the same normalised values.  A row of DK elements is held by DK/4 lanes as four consecutive elements each
// and its sum of squares is reduced over those lanes with xor shuffles, as row_dot does.
#pragma once

#include <type_traits>

#include "gdn_common.cuh"

namespace gdn {

__device__ __forceinline__ float l2_inv_norm(float sum_sq) { return rsqrtf(fmaxf(sum_sq, 1e-24f)); }

// x -> x * inv, rounded to T and widened back (the value the tensor cores or the decode step use)
template <typename T>
__device__ __forceinline__ float4 scale_round(float4 x, float inv)
{
    x.x *= inv;
    x.y *= inv;
    x.z *= inv;
    x.w *= inv;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        x.x = __bfloat162float(__float2bfloat16_rn(x.x));
        x.y = __bfloat162float(__float2bfloat16_rn(x.y));
        x.z = __bfloat162float(__float2bfloat16_rn(x.z));
        x.w = __bfloat162float(__float2bfloat16_rn(x.w));
    }
    return x;
}

// Pre-pass of the prefill: qn, kn = normalised q, k ([nvec, DK] each, nvec = T * H).  LPR lanes per
// vector; a warp loads U groups of 32 / LPR vectors (q and k) before reducing, to keep enough
// bytes in flight.
constexpr int kNormU = 4;

template <typename T, int DK>
__global__ void __launch_bounds__(256) gdn_l2norm_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                     T* __restrict__ qn, T* __restrict__ kn, int64_t nvec)
{
    constexpr int LPR = DK / 4;
    constexpr int VPW = 32 / LPR;             // vectors per warp group
    constexpr int U = kNormU;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 8 + warp;
    const int sub = lane / LPR;
    const int col = (lane % LPR) * 4;
    float4 x[2][U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t v = (gw * U + u) * VPW + sub;
        const bool live = v < nvec;
        x[0][u] = live ? Elem<T>::ld4(q + v * DK + col) : make_float4(0.f, 0.f, 0.f, 0.f);
        x[1][u] = live ? Elem<T>::ld4(k + v * DK + col) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int which = 0; which < 2; ++which) {
        T* dst = which ? kn : qn;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t v = (gw * U + u) * VPW + sub;
            const float4 a = x[which][u];
            float ss = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            // the store rounds to T once (scale_round's round-and-widen would only repeat it)
            const float inv = l2_inv_norm(ss);
            const float4 y = make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
            if (v < nvec) Elem<T>::st4(dst + v * DK + col, y);
        }
    }
}

}  // namespace gdn
