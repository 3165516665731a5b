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
// Mapping: the state of one (b, h) is split into row blocks of 32 rows, one CTA (8 warps) per block;
// a row of dk fp32 is held by dk/4 lanes as float4s (a full warp for dk = 128, half a warp for
// dk = 64).  Each warp owns 4 consecutive rows and loads them all before reducing.  Small CTAs keep
// the last wave short (2048 (b, h) pairs would leave a 0.3-full third wave at 256-row granularity).
#pragma once

#include "gdn_common.cuh"
#include "gdn_norm.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

// One row r of S for one token: the two dot products S_r.k and S_r.q are reduced over the LPR
// lanes that hold the row (float4 each), then S_r <- alpha S_r + u k with u = beta (v_r - alpha S_r.k),
// and o_r = scale (alpha S_r.q + u (k.q)).  Shared by the single-step and the multi-token kernels so
// that both perform the same operations in the same order.
template <int LPR>
__device__ __forceinline__ float4 decode_row_step(const float4 s, const float4 k4, const float4 q4, float alpha,
                                                  float b, float vr, float kq, float scale, float& o)
{
    float sk = s.x * k4.x + s.y * k4.y + s.z * k4.z + s.w * k4.w;
    float sq = s.x * q4.x + s.y * q4.y + s.z * q4.z + s.w * q4.w;
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
    }
    const float uu = b * (vr - alpha * sk);
    float4 n;
    n.x = fmaf(alpha, s.x, uu * k4.x);
    n.y = fmaf(alpha, s.y, uu * k4.y);
    n.z = fmaf(alpha, s.z, uu * k4.z);
    n.w = fmaf(alpha, s.w, uu * k4.w);
    o = scale * fmaf(alpha, sq, uu * kq);
    return n;
}

template <int LPR>
__device__ __forceinline__ float row_dot(const float4 a, const float4 b)
{
    float d = a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    return d;
}

// Rows of one (sequence, head) state per CTA and threads per CTA of the decode step (rows evolve
// independently, so a state may be split across CTAs; smaller CTAs leave a smaller last wave).
#ifndef GDN_DECODE_RB
#define GDN_DECODE_RB 32
#endif
#ifndef GDN_DECODE_NT
#define GDN_DECODE_NT 256
#endif

template <typename T, int DK, int DV, bool NORM>
__global__ void __launch_bounds__(GDN_DECODE_NT) gdn_decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, const float* __restrict__ g,
                                                          const float* __restrict__ beta, float* state,
                                                          T* __restrict__ out, int H)
{
    constexpr int LPR = DK / 4;               // lanes per row
    constexpr int RPW = 32 / LPR;             // rows handled by one warp at once
    constexpr int RB = (GDN_DECODE_RB < DV) ? GDN_DECODE_RB : DV;   // rows of the state per CTA
    constexpr int NW = GDN_DECODE_NT / 32;
    constexpr int ROWS_PER_WARP = RB / NW;
    constexpr int UNROLL = 4;
    static_assert(ROWS_PER_WARP >= RPW && ROWS_PER_WARP % RPW == 0, "row split");
    static_assert(ROWS_PER_WARP % (RPW * UNROLL) == 0 || ROWS_PER_WARP < RPW * UNROLL, "row split");
    constexpr int STEP = (ROWS_PER_WARP < RPW * UNROLL) ? ROWS_PER_WARP : RPW * UNROLL;
    constexpr int U = STEP / RPW;             // row groups per iteration

    // launched as a programmatic dependent: the previous kernel in the stream (typically the last
    // decode step, which wrote this state) has completed before anything is read here
    sm100::grid_dep_wait();
    sm100::grid_dep_launch();

    const int bh = blockIdx.x / (DV / RB);    // b * H + h
    const int rblk = blockIdx.x % (DV / RB);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR;               // which of the RPW rows this lane serves
    const int col = (lane % LPR) * 4;

    float4 k4 = Elem<T>::ld4(k + (size_t)bh * DK + col);
    float4 q4 = Elem<T>::ld4(q + (size_t)bh * DK + col);
    if constexpr (NORM) {
        // raw q and k: normalised here exactly as the prefill's pre-pass does
        k4 = scale_round<T>(k4, l2_inv_norm(row_dot<LPR>(k4, k4)));
        q4 = scale_round<T>(q4, l2_inv_norm(row_dot<LPR>(q4, q4)));
    }
    const float alpha = expf(__ldg(g + bh));
    const float b = __ldg(beta + bh);
    const float scale = rsqrtf((float)DK);

    const float kq = row_dot<LPR>(k4, q4);      // k . q over the row's lanes

    float* S = state + (size_t)bh * DV * DK;
    const int row0 = rblk * RB + warp * ROWS_PER_WARP;
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
            float o;
            const float4 n = decode_row_step<LPR>(s[u], k4, q4, alpha, b, vr[u], kq, scale, o);
            const int r = row0 + base + u * RPW + sub;
            *reinterpret_cast<float4*>(S + (size_t)r * DK + col) = n;
            if (out != nullptr && (lane % LPR) == 0) Elem<T>::st(out + (size_t)bh * DV + r, o);
        }
    }
}

// Multi-token recurrent verify: Tk draft tokens of one sequence run through the recurrence, starting
// from the committed state, which is only read (Ferrite project page, Design section 04: drafts are
// verified in one pass, as best-first trees).  Without TREE the tokens form a linear chain; with
// TREE token t continues from the state after token parents[b, t] (< t), or from the committed state
// when that is -1.  (The chain is its own instantiation, so its code is not burdened by the tree's.)  The state after every token is written to states_out, so that
// the caller keeps the one after the last accepted token and drops the rest.
//
// Mapping: one CTA (8 warps) per block of GDN_DECODE_RB rows of one (b, h) state; the block lives in
// registers for the Tk tokens (each lane holds NR float4s of its rows), is read from HBM once and
// written Tk times.
template <typename T, int DK, int DV, bool NORM, bool TREE>
__global__ void __launch_bounds__(256) gdn_decode_verify_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                            const T* __restrict__ v, const float* __restrict__ g,
                                                            const float* __restrict__ beta,
                                                            const float* __restrict__ state_in,
                                                            float* __restrict__ states_out, T* __restrict__ out,
                                                            const int32_t* __restrict__ parents, int* status,
                                                            int H, int Tk)
{
    constexpr int LPR = DK / 4;               // lanes per row
    constexpr int RPW = 32 / LPR;             // rows handled by one warp at once
    constexpr int RB = (GDN_DECODE_RB < DV) ? GDN_DECODE_RB : DV;   // rows of the state per CTA
    constexpr int ROWS_PER_WARP = RB / 8;
    constexpr int NR = ROWS_PER_WARP / RPW;   // rows held by one lane
    static_assert(ROWS_PER_WARP >= RPW && ROWS_PER_WARP % RPW == 0, "row split");

    // launched as a programmatic dependent, as the decode step is
    sm100::grid_dep_wait();
    sm100::grid_dep_launch();

    const int bh = blockIdx.x / (DV / RB);    // b * H + h
    const int rblk = blockIdx.x % (DV / RB);
    const int b = bh / H, h = bh - b * H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR;
    const int col = (lane % LPR) * 4;
    const int row0 = rblk * RB + warp * ROWS_PER_WARP + sub;
    const float scale = rsqrtf((float)DK);

    float4 s[NR];
    const float* S0 = state_in + (size_t)bh * DV * DK;
#pragma unroll
    for (int u = 0; u < NR; ++u) s[u] = *reinterpret_cast<const float4*>(S0 + (size_t)(row0 + u * RPW) * DK + col);

    for (int t = 0; t < Tk; ++t) {
        const size_t tok = ((size_t)b * Tk + t) * H + h;      // index into [B, Tk, H]
        if constexpr (TREE) {
            int p = __ldg(parents + (size_t)b * Tk + t);
            if (p < -1 || p >= t) {
                // not -1 or an earlier node: reported, and the node starts from the committed state
                if (threadIdx.x == 0) report(status, GDN_ERR_BAD_PARENTS);
                p = -1;
            }
            if (p != t - 1) {
                // the parent's state: the committed one, or the rows this thread wrote for node p
                // (read back through L2, never the read-only path: this kernel wrote them)
                if (p < 0) {
#pragma unroll
                    for (int u = 0; u < NR; ++u)
                        s[u] = *reinterpret_cast<const float4*>(S0 + (size_t)(row0 + u * RPW) * DK + col);
                } else {
                    const float* Sp = states_out + (((size_t)b * Tk + p) * H + h) * DV * DK;
#pragma unroll
                    for (int u = 0; u < NR; ++u)
                        s[u] = __ldcg(reinterpret_cast<const float4*>(Sp + (size_t)(row0 + u * RPW) * DK + col));
                }
            }
        }
        float4 k4 = Elem<T>::ld4(k + tok * DK + col);
        float4 q4 = Elem<T>::ld4(q + tok * DK + col);
        if constexpr (NORM) {
            k4 = scale_round<T>(k4, l2_inv_norm(row_dot<LPR>(k4, k4)));
            q4 = scale_round<T>(q4, l2_inv_norm(row_dot<LPR>(q4, q4)));
        }
        const float alpha = expf(__ldg(g + tok));
        const float bb = __ldg(beta + tok);
        const float kq = row_dot<LPR>(k4, q4);
        float vr[NR];
#pragma unroll
        for (int u = 0; u < NR; ++u) vr[u] = Elem<T>::ld(v + tok * DV + row0 + u * RPW);
        float* St = states_out ? states_out + tok * DV * DK : nullptr;
#pragma unroll
        for (int u = 0; u < NR; ++u) {
            const int r = row0 + u * RPW;
            float o;
            s[u] = decode_row_step<LPR>(s[u], k4, q4, alpha, bb, vr[u], kq, scale, o);
            if (St) *reinterpret_cast<float4*>(St + (size_t)r * DK + col) = s[u];
            if (out != nullptr && (lane % LPR) == 0) Elem<T>::st(out + tok * DV + r, o);
        }
    }
}

}  // namespace gdn
