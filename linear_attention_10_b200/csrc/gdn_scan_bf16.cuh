// gdn_scan_bf16.cuh -- chunk-sequential scan of the chunked prefill for bf16 q/k/v (sm_100a).
//
// Same algebra as gdn_scan_tc_kernel (see gdn_prefill_tc.cuh): per chunk
//
//   MMA_a  [X ; Z]     = [K ; Q] S^T            M=64,  N=3MS, K=dk   kind::f16 (bf16)
//   MMA_b  [U ; P U]   = [T'' ; P T''] Y        M=64,  N=2MS, K=32   kind::tf32 (3xTF32)
//   MMA_c  (dS)^T      = K^T (diag(delta) U)    M=dk,  N=3MS, K=32   kind::f16 (bf16)
//
// What is specific to bf16 inputs:
//   * q and k are exact bf16 values, so [K; Q] is used as stored: the tensor-memory-access engine
//     copies the chunk's rows straight from global memory into the 128-byte-swizzled operand layout,
//     and K^T for MMA_c is the same bytes read through an M-major descriptor.
//   * The fp32 operand on the other side (S, U~) is split into three bf16 parts that carry its 24
//     significant bits, stacked along N; one bf16 MMA (K=16) forms all three partial products, and
//     the epilogue adds the three column blocks.  The result is fp32-accurate like the 3xTF32 split
//     and needs half as many MMA instructions (bf16 takes 16 K-elements per instruction, TF32 8).
//   * One producer thread stages each chunk with bulk copies (K/Q/V tiles by tensor map, the
//     [T''; P T''] image and gates from the workspace) tracked by one transaction barrier; no thread
//     converts or stores staged operands.
//   * Rows of the last chunk of a sequence that lie beyond its end may hold the next sequence's
//     tokens (or zeros past the tensor); the epilogues zero Y for them, the operator [T''; P T'']
//     has zero columns for them, and their outputs are not stored, so they never contribute.
#pragma once

#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

template <int DK, int MS, int STAGES>
struct ScanBf16Smem {
    static constexpr int NP = DK / 64;                                // 64-element panels of dk
    // one stage
    static constexpr uint32_t oAKQ = 0;                               // [K;Q] bf16: NP panels x 64 rows x 128 B
    static constexpr uint32_t oOp = oAKQ + NP * 8192;                 // operator image + gates
    static constexpr uint32_t oV = oOp + ((kOpBCopyBytes + 1023) & ~1023u);  // V tile: 32 rows x MS bf16
    static constexpr uint32_t kStage = ((oV + 32 * MS * 2) + 1023) & ~1023u;
    static constexpr uint32_t kStageTx = NP * 2 * 4096 + kOpBCopyBytes + 32 * MS * 2;
    // shared by all stages
    // B operands of the bf16 products are stored N-major (N = 3 parts x MS, two 64-wide N-blocks)
    static constexpr uint32_t kLboS = DK * 128;                       // N-block stride of S parts
    static constexpr uint32_t kLboU = 32 * 128;                       // N-block stride of U~ parts
    static constexpr uint32_t oBS = STAGES * kStage;                  // S parts, N-major: 2 x DK rows x 128 B
    static constexpr uint32_t oBY = oBS + 2 * kLboS;                  // Y parts, N-major: 2 x 32 rows x 128 B
    static constexpr uint32_t oBU = oBY + 2 * kLboU;                  // U~ parts, N-major: 2 x 32 rows x 128 B
    static constexpr uint32_t oBar = oBU + 2 * kLboU;
    static constexpr uint32_t oTmem = oBar + 8 * (2 * STAGES + 4);
    static constexpr uint32_t oAbort = oTmem + 4;
    static constexpr uint32_t kTotal = oAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;
};

template <int DK, int DV, int MS, int STAGES>
__global__ void __launch_bounds__(288, 1) gdn_scan_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_k,
                                                               const __grid_constant__ CUtensorMap tm_v,
                                                               const int* __restrict__ meta,
                                                               const int* __restrict__ chunk_off,
                                                               const int4* __restrict__ chunk_tab,
                                                               const uint8_t* __restrict__ op,
                                                               const float* state_in,
                                                               __nv_bfloat16* __restrict__ out,
                                                               float* state_out, int H, int* status)
{
    using namespace sm100;
    using L = ScanBf16Smem<DK, MS, STAGES>;
    static_assert(MS == 32, "bf16 scan: 32 state rows per CTA");
    static_assert(DK == 64 || DK == 128, "DK");
    static_assert(DV % MS == 0, "DV");
    constexpr int NP = L::NP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::oBar);
    uint64_t* empty = full + STAGES;
    uint64_t* bar_a = empty + STAGES;
    uint64_t* bar_b = bar_a + 1;
    uint64_t* bar_c = bar_a + 2;
    uint64_t* bar_drain = bar_a + 3;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::oTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::oAbort);

    if (meta[1]) return;   // bad cu_seqlens: nothing is written
    const int n = blockIdx.x, h = blockIdx.y, r0 = blockIdx.z * MS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c_begin = chunk_off[n], c_end = chunk_off[n + 1];
    const int nch = c_end - c_begin;
    int64_t seq_t0 = 0, seq_end = 0;
    if (nch > 0) {
        const int4 first = chunk_tab[c_begin], last = chunk_tab[c_end - 1];
        seq_t0 = first.y;
        seq_end = (int64_t)last.y + last.z;
    }

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(bar_a, 1);
        mbar_init(bar_b, 1);
        mbar_init(bar_c, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    // accumulators: D1 [X;Z], D2 [U;PU], D3 dS^T, 3MS columns each (one block per bf16 part)
    const uint32_t tD1 = tmem, tD2 = tmem + 128, tD3 = tmem + 256;

    if (warp == 8) {
        // ------------------------------------------------------------------ producer (one thread)
        if (lane == 0) {
            for (int cl = 0; cl < nch; ++cl) {
                const int s = cl % STAGES;
                if (cl >= STAGES &&
                    !mbar_wait(&empty[s], (uint32_t)((cl / STAGES) - 1) & 1u, abort_flag)) {
                    tc_abort(status, abort_flag);
                    break;
                }
                const uint32_t st = sbase + s * L::kStage;
                const int t0 = (int)(seq_t0 + (int64_t)cl * kChunk);
                const int gc = c_begin + cl;
                GDN_SCAN_TRACE(cl, 11);
                mbar_arrive_expect_tx(&full[s], L::kStageTx);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    tma_load_2d(st + L::oAKQ + p * 8192, &tm_k, h * DK + p * 64, t0, &full[s]);
                    tma_load_2d(st + L::oAKQ + p * 8192 + 4096, &tm_q, h * DK + p * 64, t0, &full[s]);
                }
                bulk_load(st + L::oOp, op + ((size_t)gc * H + h) * kOpBytes, kOpBCopyBytes, &full[s]);
                tma_load_2d(st + L::oV, &tm_v, h * DV + r0, t0, &full[s]);
            }
        }
    } else {
        // ------------------------------------------------------------------ consumers (8 warps)
        // Every product is issued with M = 128 (same cost as M = 64), so an accumulator row r sits
        // in TMEM lane r: warp w reads lane quarter q4 = w % 4, and the two warps of a quarter
        // (w and w + 4) split the columns: this thread handles the MH columns [hf*MH, hf*MH + MH)
        // of each column block.
        constexpr int MH = MS / 2;
        const int q4 = warp & 3, hf = warp >> 2;
        // state: this thread holds S[hf*MH + ii][c_own], ii < MH (column c_own = TMEM lane of dS^T)
        const int c_own = q4 * 32 + lane;
        const bool owns = c_own < DK;
        float S[MH];
#pragma unroll
        for (int ii = 0; ii < MH; ++ii)
            S[ii] = (state_in && owns) ? state_in[(((size_t)n * H + h) * DV + r0 + hf * MH + ii) * DK + c_own] : 0.f;

        const float scale = rsqrtf((float)DK);
        constexpr uint32_t idA = idesc_bf16(128, 3 * MS, false, true);
        constexpr uint32_t idB3 = idesc_bf16(128, 3 * MS, false, true), idB2 = idesc_bf16(128, 2 * MS, false, true),
                           idB1 = idesc_bf16(128, MS, false, true);
        constexpr uint32_t idC = idesc_bf16(128, 3 * MS, true, true);
        const uint32_t lane_q = (uint32_t)(q4 * 32) << 16;
        bool aborted = false;

        // Writes this thread's MH consecutive N-values (N = part * MS + hf * MH + i) of K-row `k` of an
        // N-major B tile as three bf16 parts: two 16-byte stores per part.
        auto put_parts = [&](uint32_t tile, uint32_t lbo, int k, const float (&x)[MH]) {
            uint32_t w[3][MH / 2];
#pragma unroll
            for (int i = 0; i < MH; i += 2) bf16x2_split3(x[i], x[i + 1], w[0][i / 2], w[1][i / 2], w[2][i / 2]);
#pragma unroll
            for (int p = 0; p < 3; ++p) {
#pragma unroll
                for (int g = 0; g < MH / 8; ++g) {
                    const int n0 = p * MS + hf * MH + g * 8;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tile + sw128_off_nmaj(n0, k, lbo)),
                                 "r"(w[p][g * 4]), "r"(w[p][g * 4 + 1]), "r"(w[p][g * 4 + 2]), "r"(w[p][g * 4 + 3]));
                }
            }
        };

        for (int cl = 0; cl <= nch; ++cl) {
            GDN_SCAN_TRACE(cl, 0);
            // S -> three bf16 parts, N-major B operand of MMA_a (N = part * MS + row, K = dk column)
            if (owns) put_parts(sbase + L::oBS, L::kLboS, c_own, S);
            if (cl == nch) break;
            GDN_SCAN_TRACE(cl, 10);
            fence_async_smem();
            GDN_SCAN_TRACE(cl, 12);
            tc_fence_before();
            named_bar(2, 256);      // every column of S written before MMA_a reads it
            GDN_SCAN_TRACE(cl, 1);
            const int s = cl % STAGES;
            const uint32_t st = sbase + s * L::kStage;
            const uint8_t* stp = sm + s * L::kStage;

            // ---- MMA_a: [X; Z] = [K; Q] S^T  (column blocks: the three parts of S)
            if (tid == 0) {
                if (!mbar_wait(&full[s], (uint32_t)(cl / STAGES) & 1u, abort_flag)) {
                    tc_abort(status, abort_flag);
                } else {
                    GDN_SCAN_TRACE(cl, 2);
                    tc_fence_after();
                    const uint64_t a = sw128_desc(st + L::oAKQ, 0, 64);
                    const uint64_t b = sw128_desc_mn(sbase + L::oBS, L::kLboS, 1024);
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks)
                        mma_bf16(tD1, a + sw128_ks_off(ks, 64), b + (uint64_t)(ks * 128), idA, ks > 0);
                    mma_commit(bar_a);
                    GDN_SCAN_TRACE(cl, 3);
                    if (!mbar_wait(bar_a, (uint32_t)cl & 1u, abort_flag)) tc_abort(status, abort_flag);
                    GDN_SCAN_TRACE(cl, 4);
                }
            }
            named_bar(2, 256);
            GDN_SCAN_TRACE(cl, 13);
            if (*abort_flag) { aborted = true; break; }
            tc_fence_after();
            const int64_t t0 = seq_t0 + (int64_t)cl * kChunk;
            const int Lr = (int)((seq_end - t0) < kChunk ? (seq_end - t0) : kChunk);
            const float* gate = reinterpret_cast<const float*>(stp + L::oOp + kOpBGate);
            const float Gam = gate[lane];           // token `lane` (quarters 0 and 1)
            const float del = gate[32 + lane];
            const float GamC = gate[64];
            float za[MH];
            if (q4 < 2) {
                // quarter 0: X rows (token = lane), quarter 1: Z rows (token = lane)
                float x1[MH], x2[MH], x3[MH];
                tmem_ld<MH>(tD1 + lane_q + hf * MH, x1);
                tmem_ld<MH>(tD1 + lane_q + MS + hf * MH, x2);
                tmem_ld<MH>(tD1 + lane_q + 2 * MS + hf * MH, x3);
                tmem_ld_wait();
                GDN_SCAN_TRACE(cl, 14);
#pragma unroll
                for (int i = 0; i < MH; ++i) za[i] = (x1[i] + x2[i]) + x3[i];
            }
            if (q4 == 0) {
                // Y = V - diag(Gamma) X (zero past the sequence end) -> tf32 hi/lo rows of MMA_b's B
                float vt[MH];
                const uint4* vrow = reinterpret_cast<const uint4*>(stp + L::oV + lane * MS * 2 + hf * MH * 2);
#pragma unroll
                for (int q8 = 0; q8 < MH / 8; ++q8) {
                    const uint4 u = vrow[q8];
                    const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(hv[e]);
                        vt[q8 * 8 + 2 * e] = f.x;
                        vt[q8 * 8 + 2 * e + 1] = f.y;
                    }
                }
                const bool live = lane < Lr;
#pragma unroll
                for (int i = 0; i < MH; ++i) vt[i] = live ? vt[i] - Gam * za[i] : 0.f;
                put_parts(sbase + L::oBY, L::kLboU, lane, vt);     // N = part * MS + i, K = token
                GDN_SCAN_TRACE(cl, 15);
                fence_async_smem();
            }
            tc_fence_before();
            named_bar(2, 256);
            // ---- MMA_b: [U; PU] = [T''; PT''] Y  (bf16 parts: a1 x [y1|y2|y3] + a2 x [y1|y2] + a3 x y1)
            if (tid == 0) {
                GDN_SCAN_TRACE(cl, 5);
                tc_fence_after();
                const uint64_t b = sw128_desc_mn(sbase + L::oBY, L::kLboU, 1024);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const uint64_t ob = (uint64_t)(ks * 128), oa = (uint64_t)(ks * 2);
                    mma_bf16(tD2, sw64_desc(st + L::oOp) + oa, b + ob, idB3, ks > 0);
                    mma_bf16(tD2, sw64_desc(st + L::oOp + kOpBPart) + oa, b + ob, idB2, 1);
                    mma_bf16(tD2, sw64_desc(st + L::oOp + 2 * kOpBPart) + oa, b + ob, idB1, 1);
                }
                mma_commit(bar_b);
                if (!mbar_wait(bar_b, (uint32_t)cl & 1u, abort_flag)) tc_abort(status, abort_flag);
                GDN_SCAN_TRACE(cl, 6);
            }
            named_bar(2, 256);
            if (*abort_flag) { aborted = true; break; }
            tc_fence_after();
            if (q4 < 2) {
                float u[MH], u2[MH], u3[MH];
                tmem_ld<MH>(tD2 + lane_q + hf * MH, u);
                tmem_ld<MH>(tD2 + lane_q + MS + hf * MH, u2);
                tmem_ld<MH>(tD2 + lane_q + 2 * MS + hf * MH, u3);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MH; ++i) u[i] = (u[i] + u2[i]) + u3[i];
                if (q4 == 0) {
                    // U~ = diag(delta) U -> three bf16 parts, N-major B operand of MMA_c
                    // (N = part * MS + i, K = token = lane)
#pragma unroll
                    for (int i = 0; i < MH; ++i) u[i] *= del;
                    put_parts(sbase + L::oBU, L::kLboU, lane, u);
                    fence_async_smem();
                } else if (lane < Lr) {
                    // O = s (diag(Gamma) Z + P U) for token `lane`, this thread's MH columns
                    float o[MH];
#pragma unroll
                    for (int i = 0; i < MH; ++i) o[i] = scale * fmaf(Gam, za[i], u[i]);
                    store_row<MH>(out + ((size_t)(t0 + lane) * H + h) * DV + r0 + hf * MH, o);
                }
            }
            tc_fence_before();
            named_bar(2, 256);
            // ---- MMA_c: dS^T = K^T U~  (K^T read M-major from the K rows; frees the stage)
            if (tid == 0) {
                GDN_SCAN_TRACE(cl, 7);
                tc_fence_after();
                const uint64_t a = sw128_desc_mn(st + L::oAKQ, 8192, 1024);
                const uint64_t b = sw128_desc_mn(sbase + L::oBU, L::kLboU, 1024);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    mma_bf16(tD3, a + (uint64_t)(ks * 128), b + (uint64_t)(ks * 128), idC, ks > 0);
                mma_commit(bar_c);
                mma_commit(&empty[s]);
                if (!mbar_wait(bar_c, (uint32_t)cl & 1u, abort_flag)) tc_abort(status, abort_flag);
                GDN_SCAN_TRACE(cl, 8);
            }
            named_bar(2, 256);
            if (*abort_flag) { aborted = true; break; }
            tc_fence_after();
            {
                // S' = Gamma_31 S + dS  (row c_own of dS^T, this thread's half of the S rows)
                float d1[MH], d2[MH], d3[MH];
                tmem_ld<MH>(tD3 + lane_q + hf * MH, d1);
                tmem_ld<MH>(tD3 + lane_q + MS + hf * MH, d2);
                tmem_ld<MH>(tD3 + lane_q + 2 * MS + hf * MH, d3);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MH; ++i) S[i] = fmaf(GamC, S[i], (d1[i] + d2[i]) + d3[i]);
            }
            GDN_SCAN_TRACE(cl, 9);
            tc_fence_before();
        }
        if (state_out && owns && !aborted) {
#pragma unroll
            for (int ii = 0; ii < MH; ++ii)
                state_out[(((size_t)n * H + h) * DV + r0 + hf * MH + ii) * DK + c_own] = S[ii];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        // after a timeout, give copies and MMAs still in flight a bounded time to finish
        mma_commit(bar_drain);
        volatile int never = 0;
        mbar_wait(bar_drain, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace gdn
