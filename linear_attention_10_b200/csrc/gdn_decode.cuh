// gdn_decode.cuh -- recurrent single-token step of the gated delta rule (sm_100a).
//
// The consumer of the state that the chunked prefill writes back (Ferrite project page, Design
// section 03).  For one token of sequence b and head h, with S the dv x dk fp32 state:
//
//     S_t = alpha S (I - beta k k^T) + beta v k^T = alpha S + u k^T,   u = beta (v - alpha S k)
//     o   = S_t q / sqrt(dk) = (alpha S q + u (k . q)) / sqrt(dk)
//
// Every row r of S evolves on its own (right multiplication), so one pass over the rows suffices:
// a row is loaded once, its two dot products S_r.k and S_r.q are reduced across the lanes that
// hold it, and the updated row is stored once.  The kernel is bound by HBM bandwidth: per (b, h)
// it moves 2 * dv * dk * 4 bytes of state and a few hundred bytes of q, k, v, o.
//
// Mapping: one CTA (8 warps) per (b, h).  A row of dk fp32 is held by dk/4 lanes as float4s
// (a full warp for dk = 128, half a warp for dk = 64).  Each warp owns dv/8 consecutive rows and
// loads UNROLL row-groups before reducing, to keep enough bytes in flight.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256) gdn_decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, const float* __restrict__ g,
                                                          const float* __restrict__ beta, float* state,
                                                          T* __restrict__ out, int H)
{
    constexpr int LPR = DK / 4;               // lanes per row
    constexpr int RPW = 32 / LPR;             // rows handled by one warp at once
    constexpr int ROWS_PER_WARP = DV / 8;
    constexpr int UNROLL = 4;
    static_assert(ROWS_PER_WARP % (RPW * UNROLL) == 0 || ROWS_PER_WARP < RPW * UNROLL, "row split");
    constexpr int STEP = (ROWS_PER_WARP < RPW * UNROLL) ? ROWS_PER_WARP : RPW * UNROLL;
    constexpr int U = STEP / RPW;             // row groups per iteration

    const int bh = blockIdx.x;                // b * H + h
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR;               // which of the RPW rows this lane serves
    const int col = (lane % LPR) * 4;

    const float4 k4 = Elem<T>::ld4(k + (size_t)bh * DK + col);
    const float4 q4 = Elem<T>::ld4(q + (size_t)bh * DK + col);
    const float alpha = expf(__ldg(g + bh));
    const float b = __ldg(beta + bh);
    const float scale = rsqrtf((float)DK);

    // k . q over the row's lanes
    float kq = k4.x * q4.x + k4.y * q4.y + k4.z * q4.z + k4.w * q4.w;
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);

    float* S = state + (size_t)bh * DV * DK;
    const int row0 = warp * ROWS_PER_WARP;
#pragma unroll
    for (int base = 0; base < ROWS_PER_WARP; base += STEP) {
        float4 s[U];
        float vr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = row0 + base + u * RPW + sub;
            s[u] = *reinterpret_cast<const float4*>(S + (size_t)r * DK + col);
            vr[u] = Elem<T>::ld(v + (size_t)bh * DV + r);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float sk = s[u].x * k4.x + s[u].y * k4.y + s[u].z * k4.z + s[u].w * k4.w;
            float sq = s[u].x * q4.x + s[u].y * q4.y + s[u].z * q4.z + s[u].w * q4.w;
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
            }
            const float uu = b * (vr[u] - alpha * sk);
            float4 n;
            n.x = fmaf(alpha, s[u].x, uu * k4.x);
            n.y = fmaf(alpha, s[u].y, uu * k4.y);
            n.z = fmaf(alpha, s[u].z, uu * k4.z);
            n.w = fmaf(alpha, s[u].w, uu * k4.w);
            const int r = row0 + base + u * RPW + sub;
            *reinterpret_cast<float4*>(S + (size_t)r * DK + col) = n;
            if (out != nullptr && (lane % LPR) == 0)
                Elem<T>::st(out + (size_t)bh * DV + r, scale * fmaf(alpha, sq, uu * kq));
        }
    }
}

}  // namespace gdn
