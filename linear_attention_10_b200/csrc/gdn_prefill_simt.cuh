// gdn_prefill_simt.cuh -- chunkwise WY/UT prefill of the gated delta rule, fp32 CUDA-core kernels.
//
// Ferrite project page, Design section 03 "Chunked Gated DeltaNet": prompt rows go through the
// recurrent state in chunks of 32 using the chunkwise WY/UT form of the delta rule, and the final
// state is written back.  Notation inside one chunk of L <= 32 rows (rows L..31 are padding with
// q = k = v = 0, g = 0, beta = 0), S = the state entering the chunk (dv x dk):
//
//   gamma_i = g_0 + ... + g_i (chunk-local),  Gamma_i = exp(gamma_i),  delta_i = exp(gamma_31 - gamma_i)
//   A       = strictly-lower(diag(beta) (D o K K^T)),  D_ij = exp(gamma_i - gamma_j)
//   T       = (I + A)^-1                               (unit lower triangular, forward substitution)
//   T''     = T diag(beta),  W = T diag(beta Gamma) K,  P = lower-incl-diagonal(D o Q K^T)
//
// The chunk's effective writes U and its outputs O are both affine in [V ; S^T]:
//
//   U      = T'' V - W S^T                       (from (I + A) U = diag(beta)(V - diag(Gamma) K S^T))
//   O / s  = diag(Gamma) Q S^T + P U = (P T'') V + (diag(Gamma) Q - P W) S^T
//
// so one operator per (chunk, head), independent of the state,
//
//   M = [[ diag(delta) T'' , -diag(delta) W         ]     (rows 0..31:  U~ = diag(delta) U)
//        [ P T''           ,  diag(Gamma) Q - P W   ]]    (rows 32..63: O / s)
//
// of shape 64 x (32 + dk), turns the state-dependent part into one product [U~ ; O/s] = M [V ; S^T]
// followed by the carry S' = Gamma_31 S + U~^T K.  The first kernel below builds M for every
// (chunk, head) in parallel; the second walks the chunks of each sequence in order.
#pragma once

#include "gdn_common.cuh"
#include "gdn_plan.cuh"

namespace gdn {

// ------------------------------------------------------------------------------------------------
// Kernel 1: per (chunk, head) operator M and exp(gamma_31).  grid (nc_max, H), 256 threads.
// ------------------------------------------------------------------------------------------------
template <typename T, int DK>
__global__ void __launch_bounds__(256) gdn_prep_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const float* __restrict__ g,
                                                        const float* __restrict__ beta,
                                                        const int* __restrict__ meta,
                                                        const int4* __restrict__ chunk_tab,
                                                        float* __restrict__ op, float* __restrict__ aux,
                                                        int H)
{
    constexpr int C = kChunk;
    constexpr int KP = DK + 1;              // padded row stride
    constexpr int MW = C + DK;              // operator row length
    extern __shared__ float sm[];
    float* Ks = sm;                         // [C][KP]
    float* Qs = Ks + C * KP;                // [C][KP]
    float* Ws = Qs + C * KP;                // [C][KP]
    float* Am = Ws + C * KP;                // [C][C+1]  A, later reused
    float* Pm = Am + C * (C + 1);           // [C][C+1]
    float* Tm = Pm + C * (C + 1);           // [C][C+1]  T, then T''
    float* gam = Tm + C * (C + 1);          // [C]
    float* bet = gam + C;                   // [C]

    const int gc = blockIdx.x, h = blockIdx.y;
    if (gc >= meta[0]) return;
    const int4 ct = chunk_tab[gc];
    const int64_t t0 = ct.y;
    const int L = ct.z;
    const int tid = threadIdx.x;

    for (int idx = tid; idx < C * DK; idx += 256) {
        const int i = idx / DK, c = idx % DK;
        float kv = 0.f, qv = 0.f;
        if (i < L) {
            const size_t o = ((size_t)(t0 + i) * H + h) * DK + c;
            kv = Elem<T>::ld(k + o);
            qv = Elem<T>::ld(q + o);
        }
        Ks[i * KP + c] = kv;
        Qs[i * KP + c] = qv;
    }
    if (tid < 32) {
        const bool ok = tid < L;
        float gv = ok ? __ldg(g + (size_t)(t0 + tid) * H + h) : 0.f;
        bet[tid] = ok ? __ldg(beta + (size_t)(t0 + tid) * H + h) : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float y = __shfl_up_sync(0xffffffffu, gv, o);
            if (tid >= o) gv += y;
        }
        gam[tid] = gv;
    }
    __syncthreads();

    // Gram matrices K K^T and Q K^T with the gate and beta weights
    for (int idx = tid; idx < C * C; idx += 256) {
        const int i = idx / C, j = idx % C;
        float kk = 0.f, qk = 0.f;
        if (j <= i) {
            for (int c = 0; c < DK; ++c) {
                const float kj = Ks[j * KP + c];
                kk = fmaf(Ks[i * KP + c], kj, kk);
                qk = fmaf(Qs[i * KP + c], kj, qk);
            }
        }
        const float d = (j <= i) ? expf(gam[i] - gam[j]) : 0.f;
        Am[i * (C + 1) + j] = (j < i) ? bet[i] * d * kk : 0.f;
        Pm[i * (C + 1) + j] = d * qk;
    }
    __syncthreads();

    // T = (I + A)^-1: one lane per column j, rows in order
    if (tid < 32) {
        const int j = tid;
        for (int i = 0; i < C; ++i) {
            float t;
            if (i < j) t = 0.f;
            else if (i == j) t = 1.f;
            else {
                float acc = 0.f;
                for (int m = j; m < i; ++m) acc = fmaf(Am[i * (C + 1) + m], Tm[m * (C + 1) + j], acc);
                t = -acc;
            }
            Tm[i * (C + 1) + j] = t;
        }
    }
    __syncthreads();
    // T'' = T diag(beta) (in place), W = T'' diag(Gamma) K
    for (int idx = tid; idx < C * C; idx += 256) {
        const int i = idx / C, j = idx % C;
        Tm[i * (C + 1) + j] *= bet[j];
    }
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += 256) {
        const int i = idx / DK, c = idx % DK;
        float acc = 0.f;
        for (int j = 0; j <= i; ++j) acc = fmaf(Tm[i * (C + 1) + j] * expf(gam[j]), Ks[j * KP + c], acc);
        Ws[i * KP + c] = acc;
    }
    __syncthreads();

    // operator rows
    float* M = op + ((size_t)gc * H + h) * 64 * MW;
    const float glast = gam[C - 1];
    for (int idx = tid; idx < C * MW; idx += 256) {
        const int i = idx / MW, c = idx % MW;
        const float dl = expf(glast - gam[i]);
        // top block: diag(delta) [T'', -W]
        float top = (c < C) ? dl * Tm[i * (C + 1) + c] : -dl * Ws[i * KP + (c - C)];
        // bottom block: [P T'', diag(Gamma) Q - P W]
        float bot;
        if (c < C) {
            float acc = 0.f;
            for (int m = c; m <= i; ++m) acc = fmaf(Pm[i * (C + 1) + m], Tm[m * (C + 1) + c], acc);
            bot = acc;
        } else {
            const int cc = c - C;
            float acc = 0.f;
            for (int m = 0; m <= i; ++m) acc = fmaf(Pm[i * (C + 1) + m], Ws[m * KP + cc], acc);
            bot = expf(gam[i]) * Qs[i * KP + cc] - acc;
        }
        M[(size_t)i * MW + c] = top;
        M[(size_t)(C + i) * MW + c] = bot;
    }
    if (tid == 0) aux[((size_t)gc * H + h) * 4] = expf(glast);
}

// ------------------------------------------------------------------------------------------------
// Kernel 2: chunk-sequential state carry and outputs.  grid (N, H, dv / 16), 256 threads.
// Each CTA owns 16 rows of one head's state (rows of S evolve independently).
// ------------------------------------------------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256) gdn_scan_simt_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                        const int* __restrict__ meta,
                                                        const int* __restrict__ chunk_off,
                                                        const int4* __restrict__ chunk_tab,
                                                        const float* __restrict__ op,
                                                        const float* __restrict__ aux,
                                                        const float* state_in, T* __restrict__ out,
                                                        float* state_out, int H)
{
    constexpr int C = kChunk;
    constexpr int MR = 16;                  // state rows per CTA
    constexpr int MW = C + DK;
    constexpr int MP = MW + 1;
    constexpr int KP = DK + 1;
    extern __shared__ float sm[];
    float* Ms = sm;                         // [64][MP]
    float* Ks = Ms + 64 * MP;               // [C][KP]
    float* Ss = Ks + C * KP;                // [MR][KP]
    float* Vs = Ss + MR * KP;               // [C][MR]
    float* Us = Vs + C * MR;                // [C][MR]

    if (meta[1]) return;                    // bad cu_seqlens: nothing is written
    const int n = blockIdx.x, h = blockIdx.y, r0 = blockIdx.z * MR;
    const int tid = threadIdx.x;
    const float scale = rsqrtf((float)DK);

    for (int idx = tid; idx < MR * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        Ss[r * KP + c] = state_in ? state_in[(((size_t)n * H + h) * DV + r0 + r) * DK + c] : 0.f;
    }
    const int c_begin = chunk_off[n], c_end = chunk_off[n + 1];
    for (int gc = c_begin; gc < c_end; ++gc) {
        const int4 ct = chunk_tab[gc];
        const int64_t t0 = ct.y;
        const int L = ct.z;
        __syncthreads();                    // previous chunk finished with Ms/Ks/Vs/Us
        const float* M = op + ((size_t)gc * H + h) * 64 * MW;
        for (int idx = tid; idx < 64 * MW; idx += 256) Ms[(idx / MW) * MP + idx % MW] = M[idx];
        for (int idx = tid; idx < C * DK; idx += 256) {
            const int j = idx / DK, c = idx % DK;
            Ks[j * KP + c] = (j < L) ? Elem<T>::ld(k + ((size_t)(t0 + j) * H + h) * DK + c) : 0.f;
        }
        for (int idx = tid; idx < C * MR; idx += 256) {
            const int j = idx / MR, r = idx % MR;
            Vs[j * MR + r] = (j < L) ? Elem<T>::ld(v + ((size_t)(t0 + j) * H + h) * DV + r0 + r) : 0.f;
        }
        const float gl = aux[((size_t)gc * H + h) * 4];
        __syncthreads();

        // [U~ ; O/s] = M [V ; S^T]: 64 x MR outputs, 4 per thread
        {
            const int i = tid >> 2;
            const int rb = (tid & 3) * 4;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < C; ++j) {
                const float mij = Ms[i * MP + j];
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u] = fmaf(mij, Vs[j * MR + rb + u], acc[u]);
            }
            for (int c = 0; c < DK; ++c) {
                const float mic = Ms[i * MP + C + c];
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u] = fmaf(mic, Ss[(rb + u) * KP + c], acc[u]);
            }
            if (i < C) {
#pragma unroll
                for (int u = 0; u < 4; ++u) Us[i * MR + rb + u] = acc[u];
            } else if (i - C < L) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    Elem<T>::st(out + ((size_t)(t0 + i - C) * H + h) * DV + r0 + rb + u, scale * acc[u]);
            }
        }
        __syncthreads();
        // S' = Gamma_31 S + U~^T K
        for (int idx = tid; idx < MR * DK; idx += 256) {
            const int r = idx / DK, c = idx % DK;
            float acc = gl * Ss[r * KP + c];
            for (int j = 0; j < C; ++j) acc = fmaf(Us[j * MR + r], Ks[j * KP + c], acc);
            Ss[r * KP + c] = acc;
        }
    }
    __syncthreads();
    if (state_out) {
        for (int idx = tid; idx < MR * DK; idx += 256) {
            const int r = idx / DK, c = idx % DK;
            state_out[(((size_t)n * H + h) * DV + r0 + r) * DK + c] = Ss[r * KP + c];
        }
    }
}

}  // namespace gdn
