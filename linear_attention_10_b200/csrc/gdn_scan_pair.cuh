// gdn_scan_pair.cuh -- chunk-sequential scan of the chunked prefill for bf16 q/k/v (sm_100a), two
// 32-row chunks per step.
//
// The chunkwise WY/UT form (Ferrite project page, Design section 03) carries the state S from one
// chunk to the next.  This scan carries it across a pair of chunks at a time: with S_{j-1} the state
// before pair j and the pair's operator [T''; P T''], Gamma_i, delta_i (64 rows; built by the prep
// kernel from the two chunks' 32 x 32 inverses), one step is
//
//   MMA_a  [X; Z] = [K; Q] S_{j-1}^T                     M = 128, N = 3 MS, K = dk
//          Y = V - diag(Gamma) X          (zero past the sequence end)
//   MMA_b  [U; P U] = [T''; P T''] Y                     M = 128, N = 3 MS, K = 64
//          U~ = diag(delta) U,  O = s (diag(Gamma) Z + P U)
//   MMA_c  (dS)^T = K^T U~                               M = dk,  N = 3 MS, K = 64
//          S_j = Gamma_C S_{j-1} + dS
//
// With 64 rows, [K; Q] and [T''; P T''] fill the 128 rows of the tensor core's M = 128 tile, and a
// step costs about what one 32-row chunk cost when half of those rows were idle; the dependent chain
// of a sequence is half as long.
//
// One CTA owns MS = 32 rows of one head's state (rows of S evolve independently).  Warps 0..4 NQ - 1
// run the chain; thread (q4 = warp % 4, hq = warp / 4, lane) reads tensor-memory lane 32 q4 + lane (a
// lane quarter is only visible to the warps with that warp index mod 4) and the hq-th group of
// MH = 32 / NQ columns:
//   * as state owner: S[hq * MH + i][32 q4 + lane], i < MH, in registers for the whole sequence;
//   * q4 = 0, 1: token 32 q4 + lane of the pair: X -> Y and U -> U~ (B operands of MMA_b, MMA_c);
//   * q4 = 2, 3: token 32 (q4 - 2) + lane: Z, then the output row O.
// Thread 0 issues the products; warp 4 NQ (one thread) stages each pair's K/Q/V tiles with tensor
// maps and its operator record with a bulk copy, two stages deep.
//
// Precision: q and k are exact bf16 values and enter the products as stored.  The fp32 operands
// (S, Y, U~ and the operator) are split into three bf16 parts stacked along N;
// a1 x [b1|b2|b3] + a2 x [b1|b2] + a3 x b1 keeps every partial product above 2^-24 relative, so the
// products are fp32-accurate.  Rows of the last pair of a sequence that lie beyond its end may hold
// the next sequence's tokens (or zeros past the tensor): Y is zeroed for them, the operator has
// zero columns for them, and their outputs are not stored.
#pragma once

#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

template <int DK>
struct ScanPairSmem {
    static constexpr int NP = DK / 64;                               // 64-wide panels of dk
    static constexpr uint32_t kPanel = 128 * 128;                    // [K; Q] panel: 128 rows x 128 B
    // one stage: [K; Q] (NP panels), the operator record, V (64 rows x 64 B, 64-byte swizzle)
    static constexpr uint32_t oKQ = 0;
    static constexpr uint32_t oOp = NP * kPanel;
    static constexpr uint32_t oV = (oOp + kPairRecordBytes + 1023) & ~1023u;
    static constexpr uint32_t kStage = oV + 64 * 64;
    static constexpr uint32_t kStageTx = NP * kPanel + kPairRecordBytes + 64 * 64;
    // shared by both stages: B operands, N-major (N = 3 parts x 32, two 64-wide N-blocks)
    static constexpr uint32_t kLboS = DK * 128;                      // N-block stride of the S parts
    static constexpr uint32_t kLboY = 64 * 128;                      // N-block stride of the Y / U~ parts
    static constexpr uint32_t oBS = 2 * kStage;
    static constexpr uint32_t oBY = oBS + 2 * kLboS;                 // Y, then U~ of the same pair
    static constexpr uint32_t oCt = oBY + 2 * kLboY;                 // int4[2]: table entries of the staged pairs
    static constexpr uint32_t oBar = oCt + 32;                       // full[2], empty[2], a, b, c, drain
    static constexpr uint32_t oTmem = oBar + 8 * 8;
    static constexpr uint32_t oAbort = oTmem + 4;
    static constexpr uint32_t kTotal = oAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;
    static_assert(kStage % 1024 == 0 && oOp % 1024 == 0, "operand tiles on 1024-byte boundaries");
};

// threads of the scan with NQ column groups per lane quarter: 4 NQ chain warps and one producer warp
constexpr int scan_pair_threads(int nq) { return 32 * (4 * nq + 1); }

// Writes the MH consecutive N-values (N = part * MS + hq * MH + i) of K-row `k` of an N-major
// B tile as three bf16 parts: MH/8 16-byte stores per part.
template <int MS, int MH>
__device__ __forceinline__ void put_parts(uint32_t tile, uint32_t lbo, int k, int hq, const float (&x)[MH])
{
    using namespace sm100;
    uint32_t w[3][MH / 2];
#pragma unroll
    for (int i = 0; i < MH; i += 2) bf16x2_split3(x[i], x[i + 1], w[0][i / 2], w[1][i / 2], w[2][i / 2]);
#pragma unroll
    for (int p = 0; p < 3; ++p) {
#pragma unroll
        for (int g = 0; g < MH / 8; ++g) {
            const int n0 = p * MS + hq * MH + g * 8;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tile + sw128_off_nmaj(n0, k, lbo)),
                         "r"(w[p][g * 4]), "r"(w[p][g * 4 + 1]), "r"(w[p][g * 4 + 2]), "r"(w[p][g * 4 + 3]));
        }
    }
}

// Sum of the three part columns (c, c + MS, c + 2 MS) of MH consecutive accumulator columns.
template <int MS, int MH>
__device__ __forceinline__ void tmem_sum3(uint32_t taddr, float (&r)[MH])
{
    using namespace sm100;
    float a[MH], b[MH], c[MH];
    tmem_ld<MH>(taddr, a);
    tmem_ld<MH>(taddr + MS, b);
    tmem_ld<MH>(taddr + 2 * MS, c);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < MH; ++i) r[i] = (a[i] + b[i]) + c[i];
}

// CUTS: the call has cut points (segments, snapshots); without them pair j of a sequence starts at
// its token 64 j.  chunk_off / chunk_tab describe pairs (the plan kernel's table with 64-row entries).
template <int DK, int DV, bool CUTS, int NQ>
__global__ void __launch_bounds__(scan_pair_threads(NQ), 1)
    gdn_scan_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const int* __restrict__ meta,
                         const int* __restrict__ order, const int* __restrict__ chunk_off,
                         const int4* __restrict__ chunk_tab, const uint8_t* __restrict__ op,
                         const float* state_in, __nv_bfloat16* __restrict__ out, float* state_out,
                         float* __restrict__ snaps, int H, int* status)
{
    using namespace sm100;
    using L = ScanPairSmem<DK>;
    // launched as a dependent of the prep kernel: its records (and the plan's table) are read below
    grid_dep_wait();
    constexpr int MS = 32;                    // state rows per CTA
    constexpr int MH = MS / NQ;               // of which one thread handles
    constexpr int NCW = 4 * NQ;               // chain warps
    static_assert(NQ == 2 || NQ == 4, "column groups per lane quarter");
    constexpr int NP = L::NP;
    static_assert(DK == 64 || DK == 128, "DK");
    static_assert(DV % MS == 0, "DV");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::oBar);
    uint64_t* empty = full + 2;
    uint64_t* bar_a = full + 4;               // MMA_a done
    uint64_t* bar_b = full + 5;               // MMA_b done
    uint64_t* bar_c = full + 6;               // MMA_c done
    uint64_t* drain = full + 7;
    int4* ctab_s = reinterpret_cast<int4*>(sm + L::oCt);
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
    const int npair = c_end - c_begin;
    int64_t seq_t0 = 0, seq_end = 0;
    if (!CUTS && npair > 0) {
        const int4 first = chunk_tab[c_begin], last = chunk_tab[c_end - 1];
        seq_t0 = first.y;
        seq_end = (int64_t)last.y + last.z;
    }

    if (tid == 0) {
        for (int i = 0; i < 8; ++i) mbar_init(full + i, 1);
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
    // accumulators, 3 MS columns each (one block per bf16 part of the B operand)
    const uint32_t tD1 = tmem, tD2 = tmem + 128, tD3 = tmem + 256;

    constexpr uint32_t idA = idesc_bf16(128, 3 * MS, false, true);
    constexpr uint32_t idB3 = idesc_bf16(128, 3 * MS, false, true), idB2 = idesc_bf16(128, 2 * MS, false, true),
                       idB1 = idesc_bf16(128, MS, false, true);
    constexpr uint32_t idC = idesc_bf16(128, 3 * MS, true, true);

    // Operand descriptors of stage 0 and of the shared B tiles, formed once: the copy in stage s is
    // kStage * s bytes further, which adds kStage * s / 16 to the 14-bit start-address field (no
    // carry: every address is below 256 KB).  The issuing thread then only adds constants.
    constexpr uint64_t kStageD = L::kStage >> 4, kPartD = kPairPart >> 4;
    const uint64_t dKQ0 = sw128_desc(sbase + L::oKQ, 0, 128);                 // [K; Q], K-major
    const uint64_t dKt0 = sw128_desc_mn(sbase + L::oKQ, L::kPanel, 1024);     // K^T, M-major
    const uint64_t dOp0 = sw128_desc(sbase + L::oOp, 0, 128);                 // [T''; P T''] part 1
    const uint64_t dS = sw128_desc_mn(sbase + L::oBS, L::kLboS, 1024);
    const uint64_t dY = sw128_desc_mn(sbase + L::oBY, L::kLboY, 1024);

    if (warp == NCW) {
        // ------------------------------------------------------------------ producer (one thread)
        if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < npair; ++j) {
                const int s = j & 1;
                if (j >= 2 && !mbar_wait(&empty[s], (uint32_t)((j >> 1) - 1) & 1u, abort_flag)) {
                    tc_abort(status, abort_flag);
                    break;
                }
                int64_t t0 = seq_t0 + (int64_t)j * kPair;
                if constexpr (CUTS) {
                    const int4 ct = chunk_tab[c_begin + j];
                    t0 = ct.y;
                    // the entry travels with the stage (published by the arrive below)
                    ctab_s[s] = ct;
                }
                // rows at or past the end of the tensor read as zeros; the second box never
                // starts beyond INT32_MAX
                const int y0 = (int)t0, y1 = (int)(t0 + 32 < INT32_MAX ? t0 + 32 : INT32_MAX);
                const uint32_t st = sbase + s * L::kStage;
                mbar_arrive_expect_tx(&full[s], L::kStageTx);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    const uint32_t pan = st + L::oKQ + p * L::kPanel;
                    tma_load_2d(pan, &tm_k, h * DK + p * 64, y0, &full[s]);
                    tma_load_2d(pan + 4096, &tm_k, h * DK + p * 64, y1, &full[s]);
                    tma_load_2d(pan + 8192, &tm_q, h * DK + p * 64, y0, &full[s]);
                    tma_load_2d(pan + 12288, &tm_q, h * DK + p * 64, y1, &full[s]);
                }
                bulk_load(st + L::oOp, op + ((size_t)(c_begin + j) * H + h) * kPairRecordBytes, kPairRecordBytes,
                          &full[s]);
                tma_load_2d(st + L::oV, &tm_v, h * DV + r0, y0, &full[s]);
                tma_load_2d(st + L::oV + 2048, &tm_v, h * DV + r0, y1, &full[s]);
                issued = j + 1;
            }
            // copies still in flight land before the CTA exits (bounded)
            volatile int never = 0;
            for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
                mbar_wait(&full[j & 1], (uint32_t)(j >> 1) & 1u, &never, 100000000ull);
        }
    } else {
        // ------------------------------------------------------------------ chain warps
        const int q4 = warp & 3, hq = warp >> 2;   // lane quarter, column group
        const uint32_t lane_q = (uint32_t)(q4 * 32) << 16;
        const int c_own = q4 * 32 + lane;     // dk column of the state this thread holds
        const bool owns = c_own < DK;
        const bool warp_owns = q4 * 32 < DK;
        const bool xrow = q4 < 2;             // X / Y / U~ rows; else Z / O rows
        const int tok = xrow ? q4 * 32 + lane : (q4 - 2) * 32 + lane;
        const float scale = rsqrtf((float)DK);
        float S[MH];
#pragma unroll
        for (int i = 0; i < MH; ++i)
            S[i] = (state_in && owns) ? state_in[(((size_t)n * H + h) * DV + r0 + hq * MH + i) * DK + c_own] : 0.f;
        bool aborted = false;
        if (npair > 0) {
            // S_-1 -> three bf16 parts, the B operand of the first MMA_a
            if (owns) put_parts<MS, MH>(sbase + L::oBS, L::kLboS, c_own, hq, S);
            fence_async_smem();
            tc_fence_before();
            named_bar(1, 32 * NCW);
        }
        for (int j = 0; j < npair; ++j) {
            const int s = j & 1;
            const uint32_t ph = (uint32_t)(j >> 1) & 1u;
            const uint8_t* stp = sm + s * L::kStage;
            GDN_SCAN_TRACE(j, 0);
            // ---- MMA_a: [X; Z] = [K; Q] S^T   (N = 3 MS: one column block per part of S)
            if (tid == 0) {
                if (mbar_wait(&full[s], ph, abort_flag)) {
                    tc_fence_after();
                    const uint64_t a0 = dKQ0 + (uint64_t)s * kStageD;
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks)
                        mma_bf16(tD1, a0 + sw128_ks_off(ks, 128), dS + (uint64_t)(ks * 128), idA, ks > 0);
                    mma_commit(bar_a);
                } else {
                    tc_abort(status, abort_flag);
                }
            }
            bool ok = mbar_wait(&full[s], ph, abort_flag) && mbar_wait(bar_a, (uint32_t)j & 1u, abort_flag);
            if (!ok) tc_abort(status, abort_flag);
            GDN_SCAN_TRACE(j, 1);
            tc_fence_after();
            int64_t t0;
            int Lr, snap = -1;
            if constexpr (CUTS) {
                const int4 ct = ctab_s[s];
                t0 = ct.y;
                Lr = ct.z;
                snap = ct.w;
            } else {
                t0 = seq_t0 + (int64_t)j * kPair;
                Lr = (int)((seq_end - t0) < kPair ? (seq_end - t0) : kPair);
            }
            const float* gate = reinterpret_cast<const float*>(stp + L::oOp + kPairGate);
            const float Gam = gate[tok];
            float za[MH];
            tmem_sum3<MS, MH>(tD1 + lane_q + hq * MH, za);
            if (xrow) {
                // Y = V - diag(Gamma) X (zero past the sequence end) -> bf16 parts of MMA_b's B
                float y[MH];
                const uint8_t* vrow = stp + L::oV + tok * 64;
#pragma unroll
                for (int q8 = 0; q8 < MH / 8; ++q8) {
                    // 16-byte chunk (hq * MH / 8 + q8) of row `tok` at its 64-byte-swizzled place
                    const int jc = (hq * (MH / 8) + q8) ^ ((tok >> 1) & 3);
                    const uint4 u = *reinterpret_cast<const uint4*>(vrow + jc * 16);
                    const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(hv[e]);
                        y[q8 * 8 + 2 * e] = f.x;
                        y[q8 * 8 + 2 * e + 1] = f.y;
                    }
                }
                const bool live = tok < Lr;
#pragma unroll
                for (int i = 0; i < MH; ++i) y[i] = live ? fmaf(-Gam, za[i], y[i]) : 0.f;
                put_parts<MS, MH>(sbase + L::oBY, L::kLboY, tok, hq, y);   // N = part * MS + i, K = token
                fence_async_smem();
            }
            tc_fence_before();
            // MMA_b reads only the Y parts: the warps of the Z rows do not hold its issue back (the
            // loop's abort decision is taken at the state barrier below)
            if (xrow) named_bar(3, 16 * NCW);
            GDN_SCAN_TRACE(j, 2);
            // ---- MMA_b: [U; P U] = [T''; P T''] Y
            if (tid == 0) {
                tc_fence_after();
                const uint64_t a1 = dOp0 + (uint64_t)s * kStageD;
#pragma unroll
                for (int ks = 0; ks < kPair / 16; ++ks) {
                    const uint64_t ob = (uint64_t)(ks * 128), oa = (uint64_t)(ks * 2);
                    mma_bf16(tD2, a1 + oa, dY + ob, idB3, ks > 0);
                    mma_bf16(tD2, a1 + kPartD + oa, dY + ob, idB2, 1);
                    mma_bf16(tD2, a1 + 2 * kPartD + oa, dY + ob, idB1, 1);
                }
                mma_commit(bar_b);
            }
            ok = mbar_wait(bar_b, (uint32_t)j & 1u, abort_flag);
            if (!ok) tc_abort(status, abort_flag);
            GDN_SCAN_TRACE(j, 3);
            tc_fence_after();
            {
                float u[MH];
                tmem_sum3<MS, MH>(tD2 + lane_q + hq * MH, u);
                if (xrow) {
                    // U~ = diag(delta) U -> bf16 parts, B operand of MMA_c (Y has been read)
                    const float del = gate[64 + tok];
#pragma unroll
                    for (int i = 0; i < MH; ++i) u[i] *= del;
                    put_parts<MS, MH>(sbase + L::oBY, L::kLboY, tok, hq, u);
                    fence_async_smem();
                    tc_fence_before();
                    named_bar(2, 16 * NCW);
                    GDN_SCAN_TRACE(j, 4);
                    // ---- MMA_c: (dS)^T = K^T U~
                    if (tid == 0 && !*abort_flag) {
                        tc_fence_after();
                        const uint64_t a = dKt0 + (uint64_t)s * kStageD;
#pragma unroll
                        for (int ks = 0; ks < kPair / 16; ++ks)
                            mma_bf16(tD3, a + (uint64_t)(ks * 128), dY + (uint64_t)(ks * 128), idC, ks > 0);
                        mma_commit(bar_c);
                    }
                } else if (ok && tok < Lr) {
                    // O = s (diag(Gamma) Z + P U) for token `tok`, this thread's MH columns
                    float o[MH];
#pragma unroll
                    for (int i = 0; i < MH; ++i) o[i] = scale * fmaf(Gam, za[i], u[i]);
                    store_row<MH>(out + ((size_t)(t0 + tok) * H + h) * DV + r0 + hq * MH, o);
                }
            }
            // ---- state: S_j = Gamma_C S_{j-1} + dS  (row c_own of (dS)^T, this thread's MH rows)
            ok = mbar_wait(bar_c, (uint32_t)j & 1u, abort_flag);
            if (!ok) tc_abort(status, abort_flag);
            GDN_SCAN_TRACE(j, 5);
            tc_fence_after();
            if (warp_owns) {
                float d[MH];
                tmem_sum3<MS, MH>(tD3 + lane_q + hq * MH, d);
                const float GamC = gate[kPair - 1];
#pragma unroll
                for (int i = 0; i < MH; ++i) S[i] = fmaf(GamC, S[i], d[i]);
                // the state at a cut point the caller asked a snapshot of
                if (CUTS && ok && snap >= 0 && snaps != nullptr && owns) {
#pragma unroll
                    for (int i = 0; i < MH; ++i)
                        snaps[(((size_t)snap * H + h) * DV + r0 + hq * MH + i) * DK + c_own] = S[i];
                }
            }
            if (j + 1 == npair) {
                aborted = *abort_flag != 0;
                break;
            }
            if (owns) put_parts<MS, MH>(sbase + L::oBS, L::kLboS, c_own, hq, S);
            fence_async_smem();
            tc_fence_before();
            if (named_bar_any(1, 32 * NCW, *abort_flag)) { aborted = true; break; }
            // stage s has no reader left: its products are complete and its tiles read
            if (tid == 0) mbar_arrive(&empty[s]);
            GDN_SCAN_TRACE(j, 6);
        }
        if (state_out && owns && !aborted) {
#pragma unroll
            for (int i = 0; i < MH; ++i)
                state_out[(((size_t)n * H + h) * DV + r0 + hq * MH + i) * DK + c_own] = S[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // after a timeout, give the products this thread issued a bounded time to finish
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace gdn
