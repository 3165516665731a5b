// gdn_scan_bf16.cuh -- chunk-sequential scan of the chunked prefill for bf16 q/k/v (sm_100a).
//
// Same algebra as gdn_scan_tc_kernel (see gdn_prefill_tc.cuh), rearranged so that the dependent
// chain from one chunk to the next is one small product on the CUDA cores.  With S_c the state
// after chunk c (S_-1 the initial state), U~_c = diag(delta) U_c the chunk's writes as they enter
// the state (S_c = Gamma_C S_{c-1} + U~_c^T K_c) and, from the prep kernel,
//
//   M_c = diag(delta) T'' diag(Gamma) K_c K_{c-1}^T,   R_c = diag(Gamma) Q_c K_{c-1}^T - P T'' diag(Gamma) K_c K_{c-1}^T,
//
// the identity S_{c-1} = Gamma_{c-1} S_{c-2} + U~_{c-1}^T K_{c-1} turns one chunk into
//
//   W_c  = [Q; K]_c S_{c-2}^T                                   (tensor cores, a chunk ahead)
//   E_c  = V_c - Gamma_{c-1} diag(Gamma) W_K                     (epilogue)
//   [T'' E; P T'' E] = [T''; P T'']_c E_c                       (tensor cores)
//   U~_c = diag(delta) T'' E_c - M_c U~_{c-1}                    (the chain: CUDA cores, fp32)
//   O_c  = s (Gamma_{c-1} diag(Gamma) W_Q + P T'' E_c + R_c U~_{c-1})   (R_c U~_{c-1}: tensor cores)
//   (dS_c)^T = K_c^T U~_c,  S_c = Gamma_C S_{c-1} + dS_c         (tensor cores + state warps)
//
// so only U~_c = D_c - M_c U~_{c-1} (32 x 32 times 32 x 32 per CTA) is on the critical path; every
// tensor-core product depends on it through at least one chunk of slack.  A chunk that starts its
// segment (its sequence's first, or the first after a cut point) takes Gamma_{c-1} = 1, U~_{c-1} = 0
// and W_c from the exact state before it, as a call resumed there would.
//
// One CTA per (sequence, head, 32 state rows); rows of S evolve independently.  Thread roles:
//   * chain warps 0-3 (one per SM sub-partition): U~_c; lane = (token 8 w + lane / 4, columns
//     8 (lane % 4) .. + 7), M_c rows in registers;
//   * state warps 4-7: S (a dk column per thread, the CTA's 32 rows) in registers, S_c from the
//     (dS)^T rows of their lane quarter, and the three bf16 parts of S for W;
//   * warp 8: D_c = diag(delta) T'' E_c (tensor-memory lanes 0..31) -> shared memory for the chain;
//   * warp 9: O_c (lanes 32..63 of W, [T''E; PT''E] and R U~);
//   * warp 10: E_c (lanes 64..95 of W) -> three bf16 parts, the B operand of [T''; P T''] E;
//   * warp 11: the tensor-core issuer: one thread issues every product as soon as its operands are
//     ready, loop-critical products (K^T U~, W, [T''; P T''] E) before R U~;
//   * warp 12: the producer thread: TMA copies of each chunk's [Q; K] rows and the tensor-core part
//     of its operator record, STAGES chunks ahead.
// Every product has M = 128 (the same cost as M = 64), with the A operand's start placed so that the
// rows each epilogue needs fall in the tensor-memory lanes of its own sub-partition.  The fp32
// operands of the products are split into three bf16 parts stacked along N:
// a1 x [b1|b2|b3] + a2 x [b1|b2] + a3 x b1 keeps every partial product above 2^-24 relative, so
// results are fp32-accurate like the 3xTF32 split; q and k are exact bf16 values and are used as
// stored.  Rows of the last chunk of a sequence beyond its end: E is zeroed there, T'' and M have
// zero rows and columns for them, and their outputs are not stored.
#pragma once

#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

template <int DK, int STAGES>
struct ScanBf16Smem {
    static constexpr int NP = DK / 64;                    // 64-element panels of dk
    // 32-row B tiles (E, U~ parts), N-major with the 128-byte swizzle: N = 3 parts x 32 columns in
    // two 64-wide N-blocks
    static constexpr uint32_t kLboT = 32 * 128;
    // Shared buffers come first: the W product's A descriptor starts 32 rows (4 KB) before a
    // stage's tile, and the tensor cores read 128 rows of every A operand.
    static constexpr uint32_t oE = 0;                     // E parts
    static constexpr uint32_t oUp = oE + 2 * kLboT;       // [2] U~ parts
    static constexpr uint32_t oD = oUp + 4 * kLboT;       // [2] D fp32, 32 rows x 128 B (swizzled)
    static constexpr uint32_t oUf = oD + 2 * 4096;        // [2] U~ fp32, 32 rows x 128 B (swizzled)
    static constexpr uint32_t oStage = oUf + 2 * 4096;
    // one stage: [Q; K] (NP panels of 64 rows x 128 B; rows 0..31 Q, 32..63 K), then the record's
    // tensor-core operands ([T''; P T''] parts, R parts)
    static constexpr uint32_t sOp = NP * 8192;
    static constexpr uint32_t kStage = ((sOp + kOpBTcBytes) + 1023) & ~1023u;
    static constexpr uint32_t kStageTx = NP * 8192 + kOpBTcBytes;
    // S parts, N-major: two 64-wide N-blocks of DK rows x 128 B (after the stages: R's A rows read
    // up to 4 KB past the last stage)
    static constexpr uint32_t kLboS = DK * 128;
    static constexpr uint32_t oS = oStage + STAGES * kStage;
    static constexpr uint32_t oBar = oS + 2 * kLboS;
    static constexpr int kBars = 2 * STAGES + 24;
    static constexpr uint32_t oTmem = oBar + 8 * kBars;
    static constexpr uint32_t oAbort = oTmem + 4;
    static constexpr uint32_t kTotal = oAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;
    static_assert(oStage % 1024 == 0 && kStage % 1024 == 0 && oS % 1024 == 0, "swizzle atoms");
    static_assert(oStage >= 4096, "W reads 4 KB before the first stage");
    static_assert(2 * kLboS >= 4096, "R reads 4 KB past the last stage");
};

constexpr int kScanBf16Threads = 13 * 32;

// D_c and U~_c in fp32: row r at r * 128 bytes, its 16-byte chunk j at position j ^ (r % 8), so that
// a warp reading one chunk of eight rows, or one row's chunks, meets no bank conflict.
__device__ __forceinline__ uint32_t rowsw_off(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

// Three bf16 parts of 8 consecutive values of K-row `k` of an N-major 128-byte-swizzled B tile
// (N = part * 32 + n0 .. + 7; one 16-byte store per part).
__device__ __forceinline__ void put_parts8(uint32_t tile, uint32_t lbo, int k, int n0, const float (&x)[8])
{
    using namespace sm100;
    uint32_t w[3][4];
#pragma unroll
    for (int i = 0; i < 8; i += 2) bf16x2_split3(x[i], x[i + 1], w[0][i / 2], w[1][i / 2], w[2][i / 2]);
#pragma unroll
    for (int p = 0; p < 3; ++p)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tile + sw128_off_nmaj(p * 32 + n0, k, lbo)),
                     "r"(w[p][0]), "r"(w[p][1]), "r"(w[p][2]), "r"(w[p][3]));
}

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(sm100::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Sums the three column blocks (one per bf16 part of the B operand) of 32 accumulator columns
// starting at `t` into x (two 16-column halves, to bound the registers in flight).
__device__ __forceinline__ void tmem_sum3_32(uint32_t t, float (&x)[32])
{
    using namespace sm100;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float a[16], b[16], c[16];
        tmem_ld16(t + hf * 16, a);
        tmem_ld16(t + 32 + hf * 16, b);
        tmem_ld16(t + 64 + hf * 16, c);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) x[hf * 16 + i] = (a[i] + b[i]) + c[i];
    }
}

// x += the same three-block sum (in 8-column pieces: few registers in flight).
__device__ __forceinline__ void tmem_acc3_32(uint32_t t, float (&x)[32])
{
    using namespace sm100;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float a[8], b[8], c[8];
        tmem_ld8(t + q * 8, a);
        tmem_ld8(t + 32 + q * 8, b);
        tmem_ld8(t + 64 + q * 8, c);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) x[q * 8 + i] += (a[i] + b[i]) + c[i];
    }
}

// CUTS: the call has cut points (segments, snapshots); without them chunk c of a sequence starts at
// its token 32 c and only chunk 0 starts a segment.
template <int DK, int DV, int STAGES, bool CUTS>
__global__ void __launch_bounds__(kScanBf16Threads, 1)
    gdn_scan_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __nv_bfloat16* __restrict__ v, const int* __restrict__ meta,
                         const int* __restrict__ chunk_off, const int4* __restrict__ chunk_tab,
                         const uint8_t* __restrict__ op, const float* state_in, __nv_bfloat16* __restrict__ out,
                         float* state_out, float* __restrict__ snaps, int H, int* status)
{
    using namespace sm100;
    using L = ScanBf16Smem<DK, STAGES>;
    constexpr int MS = 32;
    static_assert(DK == 64 || DK == 128, "DK");
    static_assert(DV % MS == 0, "DV");
    static_assert(STAGES >= 3, "W of chunk c + 2 is issued while chunks c and c + 1 are resident");
    constexpr int NP = L::NP;
    // launched as a dependent of the prep kernel: its records (and the plan's table) are read below
    grid_dep_wait();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::oBar);
    uint64_t* empty = full + STAGES;
    uint64_t* bb = empty + STAGES;
    uint64_t* bW = bb + 0;            // [2] W_c done (per buffer)
    uint64_t* bPE = bb + 2;           // [T''; PT''] E_c done
    uint64_t* bRU = bb + 3;           // R_c U~_{c-1} done (a commit for every chunk)
    uint64_t* bP4 = bb + 4;           // K_c^T U~_c done
    uint64_t* sReady = bb + 5;        // a version of the S parts stored (4 state warps)
    uint64_t* eReady = bb + 6;        // E_c parts stored (E warp)
    uint64_t* uReady = bb + 7;        // [2] U~_c parts stored (4 chain warps)
    uint64_t* dReady = bb + 9;        // [2] D_c stored (D warp)
    uint64_t* dwFree = bb + 11;       // [2] W_c read (E and O warps)
    uint64_t* dpeFree = bb + 13;      // [T''E; PT''E]_c read (D and O warps)
    uint64_t* drFree = bb + 14;       // R U~ of chunk c read (O warp)
    uint64_t* d3Free = bb + 15;       // (dS_c)^T read (4 state warps)
    uint64_t* dFree = bb + 16;        // [2] D_c read (4 chain warps)
    uint64_t* uFree = bb + 18;        // [2] the products reading U~ parts buffer b done (issuer commit)
    uint64_t* drain = bb + 20;        // after an abort: the issuer's products
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::oTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::oAbort);

    if (meta[1]) return;   // bad cu_seqlens: nothing is written
    const int n = blockIdx.x, h = blockIdx.y, r0 = blockIdx.z * MS;
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
        const uint32_t cnt[21] = {1, 1, 1, 1, 1, 4, 1, 4, 4, 1, 1, 2, 2, 2, 1, 4, 4, 4, 1, 1, 1};
        for (int i = 0; i < 21; ++i) mbar_init(bb + i, cnt[i]);
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
    // accumulators, 96 columns each (one 32-column block per bf16 part of the B operand)
    const uint32_t tDW0 = tmem, tDPE = tmem + 192, tDR = tmem + 288, tD3 = tmem + 384;

    // chunk-local index -> stage and the parity of its fill
    auto stage_of = [](int c) { return c % STAGES; };
    auto phase_of = [](int c) { return (uint32_t)(c / STAGES) & 1u; };
    // a chunk that starts a segment (its sequence's first, or the first after a cut point)
    auto seg_first = [&](int c) { return c == 0 || (CUTS && chunk_tab[c_begin + c - 1].w >= 0); };
    // first token and valid rows of chunk c
    auto chunk_t0 = [&](int c) -> int64_t {
        if constexpr (CUTS) return chunk_tab[c_begin + c].y;
        else return seq_t0 + (int64_t)c * kChunk;
    };
    auto chunk_rows = [&](int c) -> int {
        if constexpr (CUTS) return chunk_tab[c_begin + c].z;
        else {
            const int64_t t0 = seq_t0 + (int64_t)c * kChunk;
            return (int)((seq_end - t0) < kChunk ? (seq_end - t0) : kChunk);
        }
    };
    auto record = [&](int c) { return op + ((size_t)(c_begin + c) * H + h) * kOpBytesB; };
    auto gates = [&](int c) { return reinterpret_cast<const float*>(record(c) + kOpBGate); };
    // The S parts are stored in versions: version 0 is the initial state, version v >= 1 the state
    // after chunk v - 1.  W_c reads version c - 1 (the state two chunks back) unless chunk c starts a
    // segment, when it reads version c (the exact state before it).  wset(v) = the W's of version v.
    auto w_a = [&](int v) { return (v == 0) ? 0 : ((v < nch && seg_first(v)) ? v : -1); };   // exact-state W
    auto w_b = [&](int v) { return (v + 1 < nch && !seg_first(v + 1)) ? v + 1 : -1; };       // lookahead W

    if (warp == 12) {
        // ------------------------------------------------------------------ producer (one thread)
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < nch; ++c) {
                const int s = stage_of(c);
                if (c >= STAGES && !mbar_wait(&empty[s], (uint32_t)((c / STAGES) - 1) & 1u, abort_flag)) {
                    tc_abort(status, abort_flag);
                    break;
                }
                const uint32_t st = sbase + L::oStage + s * L::kStage;
                const int t0 = (int)chunk_t0(c);
                mbar_arrive_expect_tx(&full[s], L::kStageTx);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    tma_load_2d(st + p * 8192, &tm_q, h * DK + p * 64, t0, &full[s]);
                    tma_load_2d(st + p * 8192 + 4096, &tm_k, h * DK + p * 64, t0, &full[s]);
                }
                bulk_load(st + L::sOp, record(c), kOpBTcBytes, &full[s]);
                issued = c + 1;
            }
            // after an abort, copies still in flight land before the CTA exits (bounded)
            volatile int never = 0;
            for (int c = (issued > STAGES ? issued - STAGES : 0); c < issued; ++c)
                mbar_wait(&full[stage_of(c)], phase_of(c), &never, 100000000ull);
        }
    } else if (warp == 11) {
        // ------------------------------------------------------------------ tensor-core issuer
        if (lane == 0 && nch > 0) {
            constexpr uint32_t idW = idesc_bf16(128, 96, false, true);
            constexpr uint32_t idB3 = idesc_bf16(128, 96, false, true), idB2 = idesc_bf16(128, 64, false, true),
                               idB1 = idesc_bf16(128, 32, false, true);
            constexpr uint32_t idC = idesc_bf16(128, 96, true, true);
            constexpr uint64_t kStageD = L::kStage >> 4, kPartD = kOpBPart >> 4, kRPartD = kOpBRPart >> 4;
            const uint32_t stage0 = sbase + L::oStage;
            // descriptors of stage 0 (stage s: + s * kStage / 16 in the start-address field)
            const uint64_t dWA0 = sw128_desc(stage0 - 4096, 0, 64);       // [Q; K] from 32 rows before
            const uint64_t dKt0 = sw128_desc_mn(stage0 + 4096, 8192, 1024); // K^T (M-major)
            const uint64_t dOp0 = sw64_desc(stage0 + L::sOp);                // [T''; PT''] part 1
            const uint64_t dR0 = sw64_desc(stage0 + L::sOp + kOpBR - kOpBRPart);   // R part 1, rows 32..63
            const uint64_t dE = sw128_desc_mn(sbase + L::oE, L::kLboT, 1024);
            const uint64_t dU0 = sw128_desc_mn(sbase + L::oUp, L::kLboT, 1024);
            constexpr uint64_t kUpD = (2 * L::kLboT) >> 4;
            const uint64_t dS = sw128_desc_mn(sbase + L::oS, L::kLboS, 1024);

            // three-part product D (+)= A x B over K = 32 (two K-steps), A parts kPart apart
            auto prod3 = [&](uint32_t d, uint64_t a1, uint64_t part, uint64_t b) {
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const uint64_t ob = (uint64_t)(ks * 128), oa = (uint64_t)(ks * 2);
                    mma_bf16(d, a1 + oa, b + ob, idB3, ks > 0);
                    mma_bf16(d, a1 + part + oa, b + ob, idB2, 1);
                    mma_bf16(d, a1 + 2 * part + oa, b + ob, idB1, 1);
                }
            };
            int nP4 = 0;     // next (dS_c)^T = K_c^T U~_c
            int nRU = 0;     // next c whose R_{c+1} U~_c is due (after K_c^T U~_c)
            int nPE = 0;     // next [T''; PT''] E_c
            int nV = 0;      // next S-parts version to consume
            int nSt = 0;     // versions stored so far (sReady phases consumed)
            int nWdone = 0;  // W's issued so far (they are issued in increasing chunk order)
            int pend[2] = {-1, -1};   // W's of the consumed version not yet issued
            // R_0 U~_-1 does not exist: chunk 0's phase of bRU completes at once
            mma_commit(bRU);
            uint64_t t_last = globaltimer_ns();
            bool ok = true;
            while (ok && (nP4 < nch || nRU < nch || nPE < nch || nWdone < nch)) {
                bool progress = false;
                // (1) U~_c ready: (dS_c)^T = K_c^T U~_c (the state update, on the loop to W_{c+2})
                if (nP4 < nch && mbar_test(&uReady[nP4 & 1], (uint32_t)(nP4 >> 1) & 1u) &&
                    (nP4 == 0 || mbar_test(d3Free, (uint32_t)(nP4 - 1) & 1u))) {
                    const int c = nP4;
                    tc_fence_after();
                    const uint64_t b = dU0 + (uint64_t)(c & 1) * kUpD;
                    const uint64_t a = dKt0 + (uint64_t)stage_of(c) * kStageD;
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                        mma_bf16(tD3, a + (uint64_t)(ks * 128), b + (uint64_t)(ks * 128), idC, ks > 0);
                    mma_commit(bP4);
                    ++nP4;
                    progress = true;
                }
                // (2) W's of the stored versions of the S parts, each once its stage is loaded and its
                // accumulator buffer has been read (never waiting: the stage may need event (4) first)
                if (!progress && nWdone < nch) {
                    if (pend[0] < 0 && pend[1] < 0) {
                        // skip versions that no W reads (the state warps store none for them)
                        while (nV <= nch && w_a(nV) < 0 && w_b(nV) < 0) ++nV;
                        if (nV <= nch && mbar_test(sReady, (uint32_t)nSt & 1u)) {
                            pend[0] = w_a(nV);
                            pend[1] = w_b(nV);
                            ++nV;
                            ++nSt;
                        }
                    }
                    const int w = (pend[0] >= 0) ? pend[0] : pend[1];
                    if (w >= 0 && mbar_test(&full[stage_of(w)], phase_of(w)) &&
                        (w < 2 || mbar_test(&dwFree[w & 1], (uint32_t)((w >> 1) - 1) & 1u))) {
                        tc_fence_after();
                        const uint64_t a = dWA0 + (uint64_t)stage_of(w) * kStageD;
                        const uint32_t d = tDW0 + (uint32_t)(w & 1) * 96;
#pragma unroll
                        for (int ks = 0; ks < DK / 16; ++ks)
                            mma_bf16(d, a + sw128_ks_off(ks, 64), dS + (uint64_t)(ks * 128), idW, ks > 0);
                        mma_commit(&bW[w & 1]);
                        ++nWdone;
                        if (pend[0] >= 0) pend[0] = -1;
                        else pend[1] = -1;
                        progress = true;
                    }
                }
                // (3) [T''; PT''] E_c
                if (!progress && nPE < nch && mbar_test(eReady, (uint32_t)nPE & 1u) &&
                    (nPE == 0 || mbar_test(dpeFree, (uint32_t)(nPE - 1) & 1u))) {
                    tc_fence_after();
                    prod3(tDPE, dOp0 + (uint64_t)stage_of(nPE) * kStageD, kPartD, dE);
                    mma_commit(bPE);
                    ++nPE;
                    progress = true;
                }
                // (4) R_{c+1} U~_c for the outputs of chunk c + 1 (off every loop), once K_c^T U~_c is
                // issued and the previous R U~ has been read; then U~ buffer c & 1 and stage c have
                // no product left to issue
                if (!progress && nRU < nP4 && mbar_test(drFree, (uint32_t)nRU & 1u) &&
                    (nRU + 1 >= nch || seg_first(nRU + 1) || mbar_test(&full[stage_of(nRU + 1)], phase_of(nRU + 1)))) {
                    const int c = nRU;
                    if (c + 1 < nch) {
                        if (!seg_first(c + 1)) {
                            tc_fence_after();
                            prod3(tDR, dR0 + (uint64_t)stage_of(c + 1) * kStageD, kRPartD,
                                  dU0 + (uint64_t)(c & 1) * kUpD);
                        }
                        mma_commit(bRU);
                    }
                    mma_commit(&uFree[c & 1]);
                    mma_commit(&empty[stage_of(c)]);   // every product reading stage c is issued
                    ++nRU;
                    progress = true;
                }
                if (progress) {
                    t_last = globaltimer_ns();
                } else if (*abort_flag || globaltimer_ns() - t_last > 2000000000ull) {
                    ok = false;
                }
            }
            if (!ok) tc_abort(status, abort_flag);
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------------ chain warps
        const int i = warp * 8 + (lane >> 2), jb = lane & 3;
        float Mr[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) Mr[k] = 0.f;      // chunk 0 starts its segment: no M_0
        for (int c = 0; c < nch; ++c) {
            const int b = c & 1;
            // next chunk's M row, a chunk ahead
            float Mn[32];
            if (c + 1 < nch) {
                const float4* mp = reinterpret_cast<const float4*>(record(c + 1) + kOpBM) + i * 8;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 x = __ldg(mp + q);
                    Mn[4 * q] = x.x; Mn[4 * q + 1] = x.y; Mn[4 * q + 2] = x.z; Mn[4 * q + 3] = x.w;
                }
            }
            bool ok = mbar_wait(&dReady[b], (uint32_t)(c >> 1) & 1u, abort_flag);
            float acc[8];
            {
                const float4 x0 = *reinterpret_cast<const float4*>(sm + L::oD + b * 4096 + rowsw_off(i, 2 * jb));
                const float4 x1 = *reinterpret_cast<const float4*>(sm + L::oD + b * 4096 + rowsw_off(i, 2 * jb + 1));
                acc[0] = x0.x; acc[1] = x0.y; acc[2] = x0.z; acc[3] = x0.w;
                acc[4] = x1.x; acc[5] = x1.y; acc[6] = x1.z; acc[7] = x1.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&dFree[b]);
            if (!seg_first(c)) {
                // U~_c = D_c - M_c U~_{c-1}
                const uint8_t* up = sm + L::oUf + (b ^ 1) * 4096;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float4 u0 = *reinterpret_cast<const float4*>(up + rowsw_off(k, 2 * jb));
                    const float4 u1 = *reinterpret_cast<const float4*>(up + rowsw_off(k, 2 * jb + 1));
                    const float m = Mr[k];
                    acc[0] = fmaf(-m, u0.x, acc[0]);
                    acc[1] = fmaf(-m, u0.y, acc[1]);
                    acc[2] = fmaf(-m, u0.z, acc[2]);
                    acc[3] = fmaf(-m, u0.w, acc[3]);
                    acc[4] = fmaf(-m, u1.x, acc[4]);
                    acc[5] = fmaf(-m, u1.y, acc[5]);
                    acc[6] = fmaf(-m, u1.z, acc[6]);
                    acc[7] = fmaf(-m, u1.w, acc[7]);
                }
            }
            // U~_c in fp32 for the next chunk's chain step
            *reinterpret_cast<float4*>(sm + L::oUf + b * 4096 + rowsw_off(i, 2 * jb)) =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
            *reinterpret_cast<float4*>(sm + L::oUf + b * 4096 + rowsw_off(i, 2 * jb + 1)) =
                make_float4(acc[4], acc[5], acc[6], acc[7]);
            // and as bf16 parts, the B operand of K^T U~ and R U~, once the products that read this
            // buffer two chunks ago are done
            if (ok && c >= 2) ok = mbar_wait(&uFree[b], (uint32_t)((c >> 1) - 1) & 1u, abort_flag);
            put_parts8(sbase + L::oUp + b * 2 * L::kLboT, L::kLboT, i, 8 * jb, acc);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&uReady[b]);
            if (!ok) tc_abort(status, abort_flag);
            if (named_bar_any(1, 128, *abort_flag)) break;
            if (c + 1 < nch) {
#pragma unroll
                for (int k = 0; k < 32; ++k) Mr[k] = Mn[k];
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------------ state warps
        // this thread holds S[r0 + j][c_own], j < 32 (column c_own = tensor-memory lane of (dS)^T)
        const int q4 = warp & 3;
        const int c_own = q4 * 32 + lane;
        const bool owns = c_own < DK;
        const uint32_t lane_q = (uint32_t)(q4 * 32) << 16;
        float S[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            S[j] = (state_in && owns) ? state_in[(((size_t)n * H + h) * DV + r0 + j) * DK + c_own] : 0.f;
        auto store_parts = [&]() {
            if (owns) {
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = S[g8 * 8 + e];
                    put_parts8(sbase + L::oS, L::kLboS, c_own, 8 * g8, x);
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(sReady);
        };
        int last_w = -1;      // the last W issued from the stored parts (it must finish reading them)
        bool ok = true;
        if (nch > 0) {
            store_parts();    // version 0: W_0, and W_1 unless chunk 1 starts a segment
            last_w = (w_b(0) >= 0) ? w_b(0) : 0;
        }
        for (int c = 0; c < nch && ok; ++c) {
            const float GamC = gates(c)[64];
            ok = mbar_wait(bP4, (uint32_t)c & 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            {
                float d[32];
                tmem_sum3_32(tD3 + lane_q, d);
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = fmaf(GamC, S[j], d[j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(d3Free);
            if (CUTS && snaps != nullptr && owns) {
                const int snap = chunk_tab[c_begin + c].w;
                if (snap >= 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) snaps[(((size_t)snap * H + h) * DV + r0 + j) * DK + c_own] = S[j];
                }
            }
            const int v = c + 1;
            const int wa = w_a(v), wbb = w_b(v);
            if (wa >= 0 || wbb >= 0) {
                // the previous version's last W must have finished reading the parts
                ok = mbar_wait(&bW[last_w & 1], (uint32_t)(last_w >> 1) & 1u, abort_flag);
                if (!ok) break;
                store_parts();
                last_w = (wbb >= 0) ? wbb : wa;
            }
        }
        if (!ok) tc_abort(status, abort_flag);
        if (state_out && owns && ok && !*abort_flag) {
#pragma unroll
            for (int j = 0; j < 32; ++j) state_out[(((size_t)n * H + h) * DV + r0 + j) * DK + c_own] = S[j];
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------------ D warp (lanes 0..31)
        bool ok = true;
        for (int c = 0; c < nch && ok; ++c) {
            const int b = c & 1;
            const float del = gates(c)[32 + lane];
            ok = mbar_wait(bPE, (uint32_t)c & 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            float d[32];
            tmem_sum3_32(tDPE, d);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dpeFree);
            if (c >= 2) ok = mbar_wait(&dFree[b], (uint32_t)((c >> 1) - 1) & 1u, abort_flag);
            if (!ok) break;
            uint8_t* drow = sm + L::oD + b * 4096;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(drow + rowsw_off(lane, q)) =
                    make_float4(del * d[4 * q], del * d[4 * q + 1], del * d[4 * q + 2], del * d[4 * q + 3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&dReady[b]);
        }
        if (!ok) tc_abort(status, abort_flag);
    } else if (warp == 9) {
        // ------------------------------------------------------------------ O warp (lanes 32..63)
        const uint32_t lq = 32u << 16;
        const float scale = rsqrtf((float)DK);
        float GamPrev = 1.f;
        bool ok = true;
        for (int c = 0; c < nch && ok; ++c) {
            const float* gt = gates(c);
            const float Gam = gt[lane], GamC = gt[64];
            const bool first = seg_first(c);
            const int64_t t0 = chunk_t0(c);
            const int Lr = chunk_rows(c);
            const float gp = first ? 1.f : GamPrev;
            float o[32];
            ok = mbar_wait(&bW[c & 1], (uint32_t)(c >> 1) & 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            tmem_sum3_32(tDW0 + (uint32_t)(c & 1) * 96 + lq, o);
            const float a = gp * Gam;
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] *= a;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dwFree[c & 1]);
            ok = mbar_wait(bPE, (uint32_t)c & 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            tmem_acc3_32(tDPE + lq, o);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dpeFree);
            ok = mbar_wait(bRU, (uint32_t)c & 1u, abort_flag);
            if (!ok) break;
            if (!first) {
                tc_fence_after();
                tmem_acc3_32(tDR + lq, o);
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(drFree);
            if (lane < Lr) {
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] *= scale;
                store_row<32>(out + ((size_t)(t0 + lane) * H + h) * DV + r0, o);
            }
            GamPrev = GamC;
        }
        if (!ok) tc_abort(status, abort_flag);
    } else if (warp == 10) {
        // ------------------------------------------------------------------ E warp (lanes 64..95)
        const uint32_t lq = 64u << 16;
        float GamPrev = 1.f;
        bool ok = true;
        for (int c = 0; c < nch && ok; ++c) {
            const float* gt = gates(c);
            const float Gam = gt[lane], GamC = gt[64];
            const bool first = seg_first(c);
            const int64_t t0 = chunk_t0(c);
            const int Lr = chunk_rows(c);
            const bool live = lane < Lr;
            // V row of this token, kept as bf16 pairs (zero past the chunk's rows)
            uint4 vpk[4];
            {
                const uint4* vp = reinterpret_cast<const uint4*>(v + ((size_t)(t0 + (live ? lane : 0)) * H + h) * DV + r0);
#pragma unroll
                for (int q = 0; q < 4; ++q) vpk[q] = live ? __ldg(vp + q) : make_uint4(0, 0, 0, 0);
            }
            const float a = (first ? 1.f : GamPrev) * Gam;
            ok = mbar_wait(&bW[c & 1], (uint32_t)(c >> 1) & 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            float w[32];
            tmem_sum3_32(tDW0 + (uint32_t)(c & 1) * 96 + lq, w);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dwFree[c & 1]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&vpk[q]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(hv[e]);
                    w[q * 8 + 2 * e] = live ? fmaf(-a, w[q * 8 + 2 * e], f.x) : 0.f;
                    w[q * 8 + 2 * e + 1] = live ? fmaf(-a, w[q * 8 + 2 * e + 1], f.y) : 0.f;
                }
            }
            // the E buffer is free once [T''; PT''] E of the previous chunk is done
            if (c >= 1) ok = mbar_wait(bPE, (uint32_t)(c - 1) & 1u, abort_flag);
            if (!ok) break;
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = w[g8 * 8 + e];
                put_parts8(sbase + L::oE, L::kLboT, lane, 8 * g8, x);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(eReady);
            GamPrev = GamC;
        }
        if (!ok) tc_abort(status, abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 11 * 32) {
        // after a timeout, give the products the issuer issued a bounded time to finish
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace gdn
