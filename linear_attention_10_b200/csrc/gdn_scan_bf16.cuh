// gdn_scan_bf16.cuh -- chunk-sequential scan of the chunked prefill for bf16 q/k/v (sm_100a).
//
// Same algebra as gdn_scan_tc_kernel (see gdn_prefill_tc.cuh).  With S_c the state after chunk c
// (S_-1 the initial state), chunk c needs X_c = K_c S_{c-1}^T and Z_c = Q_c S_{c-1}^T.  Because
//
//   S_{c-1} = Gamma_{c-1} S_{c-2} + U~_{c-1}^T K_{c-1}          (Gamma_{c-1}: total decay of c-1)
//
// the same products also read
//
//   [X_c; Z_c] = Gamma_{c-1} W_c + G'_c U~_{c-1},   W_c = [K_c; Q_c] S_{c-2}^T,
//                                                   G'_c = [K_c; Q_c] K_{c-1}^T  (from the prep kernel)
//
// so the big product W_c can run one chunk early, off the dependent chain, and the chain of one
// chunk shrinks to four steps:
//
//   MMA_x  D1 = G'_c U~_{c-1}              M=64, N=3MS, K=32  (three bf16 parts each side)
//   epilogue  Y = V - diag(Gamma)(Gamma_{c-1} W_c + D1)
//   MMA_b  [U; P U] = [T''; P T''] Y       M=64, N=3MS, K=32
//   epilogue  U~ = diag(delta) U -> MMA_x of the next chunk;  O = s (diag(Gamma) Z + P U)
//
// Two thread groups share the work:
//   * chain warps (0, 1, 4, 5): the two epilogues above; thread 0 issues MMA_b, MMA_x and
//     MMA_c = K^T U~ (the state increment);
//   * state warps (2, 3, 6, 7, 8, 9, 12, 13): S_c = Gamma_c S_{c-1} + (MMA_c result), the state's
//     three bf16 parts as an operand, and W_{c+2} = [K; Q]_{c+2} S_c^T (issued by one of them);
// and one producer thread (warp 10) stages each chunk's K/Q/V tiles and operator record with bulk
// copies.  Every product is issued with M = 128 (the same cost as M = 64), so an accumulator row r
// sits in tensor-memory lane r.
//
// What is specific to bf16 inputs:
//   * q and k are exact bf16 values, so [K; Q] is used as stored: the tensor-memory-access engine
//     copies the chunk's rows straight into the 128-byte-swizzled operand layout, and K^T for MMA_c
//     is the same bytes read through an M-major descriptor.
//   * The fp32 operands (S, Y, U~, the operator [T''; P T''] and G') are split into three bf16
//     parts that carry their 24 significant bits; the parts of one side are stacked along N, and
//     a1 x [b1|b2|b3] + a2 x [b1|b2] + a3 x b1 keeps every partial product above 2^-24 relative,
//     so the results are fp32-accurate like the 3xTF32 split.
//   * Rows of the last chunk of a sequence that lie beyond its end may hold the next sequence's
//     tokens (or zeros past the tensor); the epilogue zeroes Y for them, the operator has zero
//     columns for them, and their outputs are not stored, so they never contribute.
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
    static constexpr uint32_t oOp = oAKQ + NP * 8192;                 // operator record: parts, G' parts, gates
    static constexpr uint32_t oCt = oOp + ((kOpBCopyBytes + 15) & ~15u);    // the chunk's table entry (int4)
    // V tile: 32 rows x MS bf16 (64-byte rows, 64-byte swizzle: 16-byte chunk j of row r at j ^ ((r / 2) % 4))
    static constexpr uint32_t oV = oOp + ((kOpBCopyBytes + 16 + 1023) & ~1023u);
    static constexpr uint32_t kStage = ((oV + 32 * MS * 2) + 1023) & ~1023u;
    static constexpr uint32_t kStageTx = NP * 2 * 4096 + kOpBCopyBytes + 32 * MS * 2;
    // shared by all stages
    // B operands of the bf16 products are stored N-major (N = 3 parts x MS, two 64-wide N-blocks)
    static constexpr uint32_t kLboS = DK * 128;                       // N-block stride of S parts
    static constexpr uint32_t kLboU = 32 * 128;                       // N-block stride of Y / U~ parts
    static constexpr uint32_t oBS = STAGES * kStage;                  // S parts, N-major: 2 x DK rows x 128 B
    static constexpr uint32_t oBY = oBS + 2 * kLboS;                  // Y parts, N-major: 2 x 32 rows x 128 B
    static constexpr uint32_t oBU = oBY + 2 * kLboU;                  // U~ parts, N-major: 2 x 32 rows x 128 B
    static constexpr uint32_t oBar = oBU + 2 * kLboU;
    // full[STAGES], empty[STAGES], bar_x, bar_b, bar_c, bar_w[2], s_done, drain[2]
    static constexpr int kBars = 2 * STAGES + 8;
    static constexpr uint32_t oTmem = oBar + 8 * kBars;
    static constexpr uint32_t oAbort = oTmem + 4;
    static constexpr uint32_t kTotal = oAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;
};

constexpr int kScanBf16Threads = 448;

// Writes the MH consecutive N-values (N = part * MS + hf * MH + i) of K-row `k` of an N-major
// B tile as three bf16 parts: MH/8 16-byte stores per part.
template <int MS, int MH>
__device__ __forceinline__ void put_parts(uint32_t tile, uint32_t lbo, int k, int hf, const float (&x)[MH])
{
    using namespace sm100;
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
}

// CUTS: the call has cut points (segments, snapshots); without them chunk c of a sequence starts at
// its token 32 c and only chunk 0 starts a segment.
template <int DK, int DV, int MS, int STAGES, bool CUTS>
__global__ void __launch_bounds__(kScanBf16Threads, 1)
    gdn_scan_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const int* __restrict__ meta,
                         const int* __restrict__ order, const int* __restrict__ chunk_off, const int4* __restrict__ chunk_tab,
                         const uint8_t* __restrict__ op, const float* state_in, __nv_bfloat16* __restrict__ out,
                         float* state_out, float* __restrict__ snaps, int H, int* status)
{
    using namespace sm100;
    using L = ScanBf16Smem<DK, MS, STAGES>;
    // launched as a dependent of the prep kernel: its records (and the plan's table) are read below
    grid_dep_wait();
    static_assert(MS == 32, "bf16 scan: 32 state rows per CTA");
    static_assert(DK == 64 || DK == 128, "DK");
    static_assert(DV % MS == 0, "DV");
    static_assert(STAGES >= 3, "W of chunk c + 2 is issued while chunks c and c + 1 are resident");
    constexpr int NP = L::NP;
    constexpr int MH = MS / 2;                // columns of a column block handled by one thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::oBar);
    uint64_t* empty = full + STAGES;
    uint64_t* bar_x = empty + STAGES;         // MMA_c(c) and MMA_x(c + 1) done
    uint64_t* bar_b = bar_x + 1;              // MMA_b done
    uint64_t* bar_c = bar_x + 2;              // MMA_c done
    uint64_t* bar_w = bar_x + 3;              // [2]: W of even / odd chunks done
    uint64_t* s_done = bar_x + 5;             // the state warps have read the MMA_c result
    uint64_t* drain = bar_x + 6;              // [2]
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::oTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::oAbort);

    if (meta[1]) return;   // bad cu_seqlens: nothing is written
    // CTA = (slice of MS state rows, head, sequence rank): the longest sequences' CTAs come first
    constexpr int NSL = DV / MS;
    const int r0 = (int)(blockIdx.x % NSL) * MS;
    const int h = (int)((blockIdx.x / NSL) % (unsigned)H);
    const int n = order[blockIdx.x / NSL / (unsigned)H];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c_begin = chunk_off[n], c_end = chunk_off[n + 1];
    const int nch = c_end - c_begin;
    int64_t seq_t0 = 0, seq_end = 0;
    if (!CUTS && nch > 0) {
        const int4 first = chunk_tab[c_begin], last = chunk_tab[c_end - 1];
        seq_t0 = first.y;
        seq_end = (int64_t)last.y + last.z;
    }

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 8; ++i) mbar_init(bar_x + i, 1);
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
    // accumulators, 3MS columns each (one block per bf16 part of the B operand):
    // D1 G'U~, D2 [U;PU], D3 (dS)^T, DW[2] W of even / odd chunks
    static_assert(15 * MS <= 512, "tensor memory");
    const uint32_t tD1 = tmem, tD2 = tmem + 3 * MS, tD3 = tmem + 6 * MS;
    const uint32_t tDW0 = tmem + 9 * MS, tDW1 = tmem + 12 * MS;

    constexpr uint32_t idW = idesc_bf16(128, 3 * MS, false, true);
    constexpr uint32_t idB3 = idesc_bf16(128, 3 * MS, false, true), idB2 = idesc_bf16(128, 2 * MS, false, true),
                       idB1 = idesc_bf16(128, MS, false, true);
    constexpr uint32_t idC = idesc_bf16(128, 3 * MS, true, true);

    // chunk-local index -> stage and the parity of its fill
    auto stage_of = [](int c) { return c % STAGES; };
    auto phase_of = [](int c) { return (uint32_t)(c / STAGES) & 1u; };

    // a chunk that starts a segment (its sequence's first, or the first after a cut point) takes its
    // [X; Z] from the exact state before it, as a call resumed at the cut would
    auto seg_first = [&](int c) { return c == 0 || (CUTS && chunk_tab[c_begin + c - 1].w >= 0); };

    // Operand descriptors of stage 0 and of the shared operand tiles, formed once: the copy in stage s
    // is kStage * s bytes further, which adds kStage * s / 16 to the 14-bit start-address field (no
    // carry: every address is below 256 KB).  The issuing threads then only add constants.
    static_assert(L::kStage % 16 == 0 && kOpBPart % 16 == 0, "descriptor offsets");
    constexpr uint64_t kStageD = L::kStage >> 4, kPartD = kOpBPart >> 4;
    const uint64_t dOp0 = sw64_desc(sbase + L::oOp);                 // [T''; PT''] part 1, stage 0
    const uint64_t dCr0 = sw64_desc(sbase + L::oOp + kOpBCross);     // G' part 1, stage 0
    const uint64_t dKt0 = sw128_desc_mn(sbase + L::oAKQ, 8192, 1024); // K^T, stage 0
    const uint64_t dKQ0 = sw128_desc(sbase + L::oAKQ, 0, 64);        // [K; Q], stage 0
    const uint64_t dY = sw128_desc_mn(sbase + L::oBY, L::kLboU, 1024);
    const uint64_t dU = sw128_desc_mn(sbase + L::oBU, L::kLboU, 1024);
    const uint64_t dS = sw128_desc_mn(sbase + L::oBS, L::kLboS, 1024);

    const bool chain = warp < 8 && (warp & 3) < 2;
    const bool sgrp = (warp < 8) ? ((warp & 3) >= 2) : (warp == 8 || warp == 9 || warp == 12 || warp == 13);

    if (warp == 10) {
        // ------------------------------------------------------------------ producer (one thread)
        if (lane == 0) {
            int issued = 0;
            for (int cl = 0; cl < nch; ++cl) {
                const int s = stage_of(cl);
                if (cl >= STAGES && !mbar_wait(&empty[s], (uint32_t)((cl / STAGES) - 1) & 1u, abort_flag)) {
                    tc_abort(status, abort_flag);
                    break;
                }
                const uint32_t st = sbase + s * L::kStage;
                int t0 = (int)(seq_t0 + (int64_t)cl * kChunk);
                if constexpr (CUTS) {
                    const int4 ct = chunk_tab[c_begin + cl];
                    t0 = ct.y;
                    // the entry travels with the stage (published by the arrive below)
                    *reinterpret_cast<int4*>(sm + s * L::kStage + L::oCt) = ct;
                }
                const int gc = c_begin + cl;
                mbar_arrive_expect_tx(&full[s], L::kStageTx);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    tma_load_2d(st + L::oAKQ + p * 8192, &tm_k, h * DK + p * 64, t0, &full[s]);
                    tma_load_2d(st + L::oAKQ + p * 8192 + 4096, &tm_q, h * DK + p * 64, t0, &full[s]);
                }
                bulk_load(st + L::oOp, op + ((size_t)gc * H + h) * kOpBytesB, kOpBCopyBytes, &full[s]);
                tma_load_2d(st + L::oV, &tm_v, h * DV + r0, t0, &full[s]);
                issued = cl + 1;
            }
            // after an abort, copies still in flight land before the CTA exits (bounded)
            volatile int never = 0;
            for (int cl = (issued > STAGES ? issued - STAGES : 0); cl < issued; ++cl)
                mbar_wait(&full[stage_of(cl)], phase_of(cl), &never, 100000000ull);
        }
    } else if (chain) {
        // ------------------------------------------------------------------ chain warps
        // quarter q4 = 0: X / Y / U~ rows (token = lane), q4 = 1: Z / O rows; hf: column half
        const int q4 = warp & 3, hf = warp >> 2;
        const uint32_t lane_q = (uint32_t)(q4 * 32) << 16;
        const float scale = rsqrtf((float)DK);
        float GamPrev = 1.f;
        int nx = 0;                           // MMA_x products waited for so far
        // chunk-table entries travel in registers, the next one loaded a chunk ahead
        int prev_w = -1;
        for (int c = 0; c < nch; ++c) {
            const bool first = (c == 0) || (CUTS && prev_w >= 0);
            const int s = stage_of(c);
            const uint32_t st = sbase + s * L::kStage;
            const uint8_t* stp = sm + s * L::kStage;
            GDN_SCAN_TRACE(c, 0);
            bool ok = mbar_wait(&full[s], phase_of(c), abort_flag) &&
                      mbar_wait(&bar_w[c & 1], (uint32_t)(c >> 1) & 1u, abort_flag);
            GDN_SCAN_TRACE(c, 1);
            // W_c is ready well before MMA_x: read and sum its three parts while MMA_x still runs
            tc_fence_after();
            float wsum[MH];
            {
                float w1[MH], w2[MH], w3[MH];
                const uint32_t tw = ((c & 1) ? tDW1 : tDW0) + lane_q + hf * MH;
                tmem_ld<MH>(tw, w1);
                tmem_ld<MH>(tw + MS, w2);
                tmem_ld<MH>(tw + 2 * MS, w3);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MH; ++i) wsum[i] = (w1[i] + w2[i]) + w3[i];
            }
            // MMA_x of this chunk (which also covers MMA_c of the last one) or, at a segment start,
            // MMA_c of the last chunk alone
            if constexpr (CUTS) {
                if (ok && c > 0) ok = first ? mbar_wait(bar_c, (uint32_t)(c - 1) & 1u, abort_flag)
                                            : mbar_wait(bar_x, (uint32_t)nx & 1u, abort_flag);
                if (c > 0 && !first) ++nx;
            } else {
                if (ok && c > 0) ok = mbar_wait(bar_x, (uint32_t)(c - 1) & 1u, abort_flag);
            }
            if (!ok) tc_abort(status, abort_flag);
            GDN_SCAN_TRACE(c, 2);
            tc_fence_after();
            int64_t t0;
            int Lr, ctab_w = -1;
            if constexpr (CUTS) {
                const int4 ctab = *reinterpret_cast<const int4*>(stp + L::oCt);
                t0 = ctab.y;
                Lr = ctab.z;
                ctab_w = ctab.w;
            } else {
                t0 = seq_t0 + (int64_t)c * kChunk;
                Lr = (int)((seq_end - t0) < kChunk ? (seq_end - t0) : kChunk);
            }
            const float* gate = reinterpret_cast<const float*>(stp + L::oOp + kOpBGate);
            const float Gam = gate[lane];
            const float del = gate[32 + lane];
            const float GamC = gate[64];
            // [X; Z] rows: Gamma_{c-1} W_c + G'_c U~_{c-1}  (chunk 0: W_0 = [K; Q] S_-1^T alone)
            float za[MH];
            if (!first) {
                float x1[MH], x2[MH], x3[MH];
                const uint32_t tx = tD1 + lane_q + hf * MH;
                tmem_ld<MH>(tx, x1);
                tmem_ld<MH>(tx + MS, x2);
                tmem_ld<MH>(tx + 2 * MS, x3);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MH; ++i) za[i] = fmaf(GamPrev, wsum[i], (x1[i] + x2[i]) + x3[i]);
            } else {
#pragma unroll
                for (int i = 0; i < MH; ++i) za[i] = wsum[i];
            }
            GDN_SCAN_TRACE(c, 3);
            if (q4 == 0) {
                // Y = V - diag(Gamma) X (zero past the sequence end) -> bf16 parts of MMA_b's B
                float vt[MH];
                const uint8_t* vrow = stp + L::oV + lane * MS * 2;
#pragma unroll
                for (int q8 = 0; q8 < MH / 8; ++q8) {
                    // the swizzled position of 16-byte chunk (hf * MH / 8 + q8) of row `lane`: the 32
                    // lanes of a warp then read distinct banks
                    const int j = (hf * (MH / 8) + q8) ^ ((lane >> 1) & 3);
                    const uint4 u = *reinterpret_cast<const uint4*>(vrow + j * 16);
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
                put_parts<MS, MH>(sbase + L::oBY, L::kLboU, lane, hf, vt);   // N = part * MS + i, K = token
                fence_async_smem();
            }
            tc_fence_before();
            if (named_bar_any(2, 128, *abort_flag)) break;
            GDN_SCAN_TRACE(c, 4);
            // ---- MMA_b: [U; PU] = [T''; PT''] Y
            if (tid == 0) {
                tc_fence_after();
                const uint64_t a1 = dOp0 + (uint64_t)s * kStageD;
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const uint64_t ob = (uint64_t)(ks * 128), oa = (uint64_t)(ks * 2);
                    mma_bf16(tD2, a1 + oa, dY + ob, idB3, ks > 0);
                    mma_bf16(tD2, a1 + kPartD + oa, dY + ob, idB2, 1);
                    mma_bf16(tD2, a1 + 2 * kPartD + oa, dY + ob, idB1, 1);
                }
                mma_commit(bar_b);
            }
            if (!mbar_wait(bar_b, (uint32_t)c & 1u, abort_flag)) tc_abort(status, abort_flag);
            GDN_SCAN_TRACE(c, 5);
            tc_fence_after();
            {
                float u[MH], u2[MH], u3[MH];
                const uint32_t tu = tD2 + lane_q + hf * MH;
                tmem_ld<MH>(tu, u);
                tmem_ld<MH>(tu + MS, u2);
                tmem_ld<MH>(tu + 2 * MS, u3);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MH; ++i) u[i] = (u[i] + u2[i]) + u3[i];
                if (q4 == 0) {
                    // U~ = diag(delta) U -> bf16 parts, N-major B operand of MMA_c and MMA_x
#pragma unroll
                    for (int i = 0; i < MH; ++i) u[i] *= del;
                    put_parts<MS, MH>(sbase + L::oBU, L::kLboU, lane, hf, u);
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
            if (named_bar_any(2, 128, *abort_flag)) break;
            GDN_SCAN_TRACE(c, 6);
            if (tid == 0) {
                tc_fence_after();
                // ---- MMA_c: (dS)^T = K^T U~, once the state warps have read the previous one
                bool ok2 = (c == 0) || mbar_wait(s_done, (uint32_t)(c - 1) & 1u, abort_flag);
                GDN_SCAN_TRACE(c, 8);
                if (ok2) {
                    const uint64_t a = dKt0 + (uint64_t)s * kStageD;
                    const uint64_t b = dU;
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                        mma_bf16(tD3, a + (uint64_t)(ks * 128), b + (uint64_t)(ks * 128), idC, ks > 0);
                    mma_commit(bar_c);
                    GDN_SCAN_TRACE(c, 9);
                    // ---- MMA_x of the next chunk: D1 = G'_{c+1} U~_c
                    if (c + 1 < nch && (!CUTS || ctab_w < 0)) {
                        const int s1 = stage_of(c + 1);
                        const uint64_t g1 = dCr0 + (uint64_t)s1 * kStageD;
                        ok2 = mbar_wait(&full[s1], phase_of(c + 1), abort_flag);
                        GDN_SCAN_TRACE(c, 10);
                        if (ok2) {
                            tc_fence_after();
#pragma unroll
                            for (int ks = 0; ks < 2; ++ks) {
                                const uint64_t ob = (uint64_t)(ks * 128), oa = (uint64_t)(ks * 2);
                                mma_bf16(tD1, g1 + oa, b + ob, idB3, ks > 0);
                                mma_bf16(tD1, g1 + kPartD + oa, b + ob, idB2, 1);
                                mma_bf16(tD1, g1 + 2 * kPartD + oa, b + ob, idB1, 1);
                            }
                            mma_commit(bar_x);
                        }
                    }
                }
                if (!ok2) tc_abort(status, abort_flag);
                GDN_SCAN_TRACE(c, 7);
            }
            GamPrev = GamC;
            prev_w = ctab_w;
        }
    } else if (sgrp) {
        // ------------------------------------------------------------------ state warps
        // this thread holds S[hf*MH + ii][c_own], ii < MH (column c_own = TMEM lane of (dS)^T)
        const int q4 = warp & 3, hf = (warp >> 2) & 1;
        const int c_own = q4 * 32 + lane;
        const bool owns = c_own < DK;
        const uint32_t lane_q = (uint32_t)(q4 * 32) << 16;
        const bool lead = (warp == 8 && lane == 0);
        float S[MH];
#pragma unroll
        for (int ii = 0; ii < MH; ++ii)
            S[ii] = (state_in && owns) ? state_in[(((size_t)n * H + h) * DV + r0 + hf * MH + ii) * DK + c_own] : 0.f;

        // W_k = [K; Q]_k S^T into DW[k & 1], where the S parts hold the state entering chunk k - 1
        auto issue_w = [&](int k) -> bool {
            const int sk = stage_of(k);
            const uint64_t a = dKQ0 + (uint64_t)sk * kStageD;
            const uint64_t b = dS;
            if (!mbar_wait(&full[sk], phase_of(k), abort_flag)) return false;
            tc_fence_after();
            const uint32_t d = (k & 1) ? tDW1 : tDW0;
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks)
                mma_bf16(d, a + sw128_ks_off(ks, 64), b + (uint64_t)(ks * 128), idW, ks > 0);
            mma_commit(&bar_w[k & 1]);
            return true;
        };

        int last_w = 0;                       // the last W issued (it reads the state's parts)
        bool aborted = false;
        if (nch > 0) {
            // the initial state serves W_0 and (unless a cut follows chunk 0) W_1
            if (owns) put_parts<MS, MH>(sbase + L::oBS, L::kLboS, c_own, hf, S);
            fence_async_smem();
            tc_fence_before();
            named_bar(3, 256);
            if (lead) {
                tc_fence_after();
                if (!issue_w(0) || (nch > 1 && !seg_first(1) && !issue_w(1))) tc_abort(status, abort_flag);
            }
            last_w = (nch > 1 && !seg_first(1)) ? 1 : 0;
        }
        for (int j = 0; j < nch; ++j) {
            const int s = stage_of(j);
            // snapshot indices of chunks j and j + 1 (a segment ends after a chunk with one), from
            // the chunk-table entries that travel with the stages
            int w_cur = -1, w_next = -1;
            if constexpr (CUTS) {
                const bool okw = mbar_wait(&full[s], phase_of(j), abort_flag) &&
                                 (j + 1 >= nch || mbar_wait(&full[stage_of(j + 1)], phase_of(j + 1), abort_flag));
                if (!okw || !mbar_wait(bar_c, (uint32_t)j & 1u, abort_flag)) tc_abort(status, abort_flag);
                w_cur = reinterpret_cast<const int4*>(sm + s * L::kStage + L::oCt)->w;
                if (j + 1 < nch) w_next = reinterpret_cast<const int4*>(sm + stage_of(j + 1) * L::kStage + L::oCt)->w;
            } else {
                if (!mbar_wait(&full[s], phase_of(j), abort_flag) || !mbar_wait(bar_c, (uint32_t)j & 1u, abort_flag))
                    tc_abort(status, abort_flag);
            }
            if (lead) GDN_SCAN_TRACE(j, 12);
            tc_fence_after();
            {
                // S_j = Gamma_j S_{j-1} + dS_j  (row c_own of (dS)^T, this thread's half of the S rows)
                const float GamC = reinterpret_cast<const float*>(sm + s * L::kStage + L::oOp + kOpBGate)[64];
                float d1[MH], d2[MH], d3[MH];
                const uint32_t td = tD3 + lane_q + hf * MH;
                tmem_ld<MH>(td, d1);
                tmem_ld<MH>(td + MS, d2);
                tmem_ld<MH>(td + 2 * MS, d3);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MH; ++i) S[i] = fmaf(GamC, S[i], (d1[i] + d2[i]) + d3[i]);
                // the state at a cut point the caller asked a snapshot of
                const int snap = w_cur;
                if (CUTS && snap >= 0 && snaps != nullptr && owns) {
#pragma unroll
                    for (int ii = 0; ii < MH; ++ii)
                        snaps[(((size_t)snap * H + h) * DV + r0 + hf * MH + ii) * DK + c_own] = S[ii];
                }
            }
            tc_fence_before();
            if (named_bar_any(3, 256, *abort_flag)) { aborted = true; break; }
            if (lead) {
                // (dS)^T is read and stage j has no reader left
                mbar_arrive(s_done);
                mbar_arrive(&empty[s]);
                GDN_SCAN_TRACE(j, 13);
            }
            if constexpr (CUTS) {
                // W_{j+1} when chunk j+1 starts a segment (from the exact state S_j), and W_{j+2} one
                // chunk ahead unless chunk j+2 starts a segment (then it waits for S_{j+1})
                const bool wa = (j + 1 < nch) && w_cur >= 0;
                const bool wb = (j + 2 < nch) && w_next < 0;
                if (wa || wb) {
                    // once the last W issued has finished reading the previous state's parts
                    if (!mbar_wait(&bar_w[last_w & 1], (uint32_t)(last_w >> 1) & 1u, abort_flag))
                        tc_abort(status, abort_flag);
                    if (owns) put_parts<MS, MH>(sbase + L::oBS, L::kLboS, c_own, hf, S);
                    fence_async_smem();
                    tc_fence_before();
                    if (named_bar_any(3, 256, *abort_flag)) { aborted = true; break; }
                    if (lead) {
                        tc_fence_after();
                        if ((wa && !issue_w(j + 1)) || (wb && !issue_w(j + 2))) tc_abort(status, abort_flag);
                    }
                    last_w = wb ? j + 2 : j + 1;
                }
            } else if (j + 2 < nch) {
                // once W_{j+1} has finished reading the previous state's parts
                if (!mbar_wait(&bar_w[(j + 1) & 1], (uint32_t)((j + 1) >> 1) & 1u, abort_flag))
                    tc_abort(status, abort_flag);
                if (owns) put_parts<MS, MH>(sbase + L::oBS, L::kLboS, c_own, hf, S);
                fence_async_smem();
                tc_fence_before();
                if (named_bar_any(3, 256, *abort_flag)) { aborted = true; break; }
                if (lead) {
                    GDN_SCAN_TRACE(j, 14);
                    tc_fence_after();
                    if (!issue_w(j + 2)) tc_abort(status, abort_flag);
                    GDN_SCAN_TRACE(j, 15);
                }
            }
        }
        if (state_out && owns && !aborted) {
#pragma unroll
            for (int ii = 0; ii < MH; ++ii)
                state_out[(((size_t)n * H + h) * DV + r0 + hf * MH + ii) * DK + c_own] = S[ii];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && (tid == 0 || tid == 256)) {
        // after a timeout, give the products this thread issued a bounded time to finish
        uint64_t* d = drain + (tid == 0 ? 0 : 1);
        mma_commit(d);
        volatile int never = 0;
        mbar_wait(d, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace gdn
