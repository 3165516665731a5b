// gdn_prep_bf16.cuh -- per-(chunk, head) WY/UT operator for bf16 q/k (sm_100a).
//
// Builds the operator record the bf16 scan reads, for one chunk of 32 rows of one head: [T''; P T'']
// and the cross-chunk Gram G' = [K; Q] K_prev^T, each as three bf16 parts in the 64-byte-swizzled
// K-major layout of a tensor-core A operand, and the gates Gamma_i, delta_i, Gamma_C, where
// (chunk-local cumulative log-gate gamma)
//
//   A = strictly-lower(diag(beta) (D o K K^T)),  P = lower-incl-diagonal(D o Q K^T),
//   D_ij = exp(gamma_i - gamma_j),  T = (I + A)^-1,  T'' = T diag(beta).
//
// What is specific to bf16 inputs: the chunk's [K; Q] rows are exact bf16 values, so the tensor-
// memory-access engine copies them straight into the 128-byte-swizzled operand layout (the next
// item's rows arrive while this one is gated, solved and written out, five CTAs per SM) and one
// bf16 tensor-core product (M = 128, N = 32, K = dk) forms both Gram
// matrices exactly in fp32.  The gates are applied while the Gram rows come out of tensor memory.
// The inverse uses the 2 x 2 block form with 16 x 16 blocks,
//
//   T11 = (I + A11)^-1,  T22 = (I + A22)^-1  (forward substitution, in parallel),
//   T21 = -T22 (A21 T11),
//
// which shortens the dependent chain of the substitution from 31 steps to 15.
//
// The cross-chunk Gram G' = [K; Q] K_prev^T (the scan's MMA_x operand) is issued by a second thread
// with the A descriptor started 64 rows before the tile, so its rows land in tensor-memory lanes
// 64..127: warps 2 and 3, which only those lanes are visible to, split and store it while warps 0
// and 1 gate the chunk's own Gram rows in lanes 0..63.
#pragma once

#include <cuda.h>

#include "gdn_common.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

template <int DK>
struct PrepBf16Smem {
    static constexpr int NP = DK / 64;
    // The tensor cores read 128 rows of an A operand.  The chunk's Gram reads the tile's 64 rows and
    // the 64 rows after them; G' reads 64 rows before the tile and the tile.  Each tile therefore has
    // at least 8 KB of this CTA's shared memory on both sides.
    static constexpr uint32_t kTile = NP * 8192;                      // [K;Q] bf16: NP panels x 64 rows x 128 B
    static constexpr uint32_t oPrev = 0;                              // previous chunk's K: NP x 32 rows x 128 B
    static constexpr uint32_t oTile = 8192;                           // one buffer, refilled once the item's
                                                                      // products have read it
    static constexpr int LD = 36;                                     // row pitch: 16-byte rows, no bank conflicts
    static constexpr uint32_t oG = oTile + kTile;                     // [32][LD] A
    static constexpr uint32_t oP = oG + 32 * LD * 4;                  // [32][LD] P
    static constexpr uint32_t oT = oP + 32 * LD * 4;                  // [32][LD] T
    static constexpr int LM = 16;                                     // pitch of M (2-way write conflicts)
    static constexpr uint32_t oM = oT + 32 * LD * 4;                  // [16][LM] A21 T11
    static constexpr uint32_t oGam = oM + 16 * LM * 4;
    static constexpr uint32_t oBet = oGam + 128;
    static constexpr uint32_t oAlph = oBet + 128;                     // per-token decays exp(g), one spare
    static constexpr uint32_t oBar = oAlph + 136;   // tile_full, (spare), mma, drain[2], prev_full, cross
    static constexpr uint32_t oTmem = oBar + 56;
    static constexpr uint32_t oAbort = oTmem + 4;
    static constexpr uint32_t kTotal = oAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;
    static_assert(NP * 4096 <= oTile, "previous-K buffer; 8 KB before the first tile");
    static_assert(kTotal >= oG + 8192, "rows read after the last tile's last panel");
    static_assert(5 * (kBytes + 1024) <= 233472, "five CTAs per SM (1 KB reserved per CTA)");
};

// CTAs resident per SM (shared memory and registers are sized for it; the launch sizes its grid so)
constexpr int kPrepBf16CtasPerSm = 5;

template <int DK>
__global__ void __launch_bounds__(128, kPrepBf16CtasPerSm) gdn_prep_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_k,
                                                               const float* __restrict__ g,
                                                               const float* __restrict__ beta,
                                                               const int* __restrict__ meta,
                                                               const int* __restrict__ chunk_off,
                                                               const int4* __restrict__ chunk_tab,
                                                               uint8_t* __restrict__ op, int H, int* status)
{
    using namespace sm100;
    using L = PrepBf16Smem<DK>;
    constexpr int NP = L::NP;
    constexpr int LD = L::LD;
    // launched as a dependent of the plan kernel: its chunk table is read below
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float* G = reinterpret_cast<float*>(sm + L::oG);
    float* P = reinterpret_cast<float*>(sm + L::oP);
    float* Tm = reinterpret_cast<float*>(sm + L::oT);
    float* M1 = reinterpret_cast<float*>(sm + L::oM);
    float* gam = reinterpret_cast<float*>(sm + L::oGam);
    float* bet = reinterpret_cast<float*>(sm + L::oBet);
    float* alph = reinterpret_cast<float*>(sm + L::oAlph);
    uint64_t* tile_full = reinterpret_cast<uint64_t*>(sm + L::oBar);
    uint64_t* mma_bar = tile_full + 2;        // the chunk's Gram product done
    uint64_t* drain = tile_full + 3;          // [2]: after an abort, the products of threads 0 / 96
    uint64_t* prev_full = tile_full + 5;
    uint64_t* cross_bar = tile_full + 6;      // the cross-chunk Gram product (thread 96's) done
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::oTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::oAbort);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nitems = meta[0] * H;
    if (tid == 0) {
        mbar_init(&tile_full[0], 1);
        mbar_init(&tile_full[1], 1);
        mbar_init(mma_bar, 1);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        mbar_init(prev_full, 1);
        mbar_init(cross_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 64);      // columns 0..31: Gram products, 32..63: cross-chunk Gram
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    // whether chunk gc has a previous chunk in its sequence (then the cross-chunk Gram is built)
    auto has_prev = [&](int gc) { return gc > chunk_off[chunk_tab[gc].x]; };
    // copies the [K; Q] rows of one item into the tile buffer (one thread per fill; issued once the
    // previous item's products have read the buffer)
    auto issue_tile = [&](int item) {
        const int gc = item / H, h = item % H;
        const int t0 = chunk_tab[gc].y;
        const uint32_t dst = sbase + L::oTile;
        mbar_arrive_expect_tx(tile_full, NP * 2 * 4096);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            tma_load_2d(dst + p * 8192, &tm_k, h * DK + p * 64, t0, tile_full);
            tma_load_2d(dst + p * 8192 + 4096, &tm_q, h * DK + p * 64, t0, tile_full);
        }
    };
    // copies the previous chunk's K rows of one item into the single previous-K buffer (one thread;
    // issued once the buffer's last reader has completed).  An item that starts its sequence
    // loads its own K rows instead, so that the buffer's barrier completes once per item.
    auto issue_prev = [&](int item) {
        const int gc = item / H, h = item % H;
        const int t0 = chunk_tab[gc].y;
        const int tp = has_prev(gc) ? chunk_tab[gc - 1].y : t0;    // the previous chunk may end at a cut
        mbar_arrive_expect_tx(prev_full, NP * 4096);
#pragma unroll
        for (int p = 0; p < NP; ++p) tma_load_2d(sbase + L::oPrev + p * 4096, &tm_k, h * DK + p * 64, tp, prev_full);
    };
    // gate inputs of one item (lanes of warp 2; zero past the chunk's rows)
    auto load_gates = [&](int item, float& gv, float& bv) {
        const int gc = item / H, h = item % H;
        const int4 ct = chunk_tab[gc];
        const bool ok = lane < ct.z;
        gv = ok ? __ldg(g + (size_t)(ct.y + lane) * H + h) : 0.f;
        bv = ok ? __ldg(beta + (size_t)(ct.y + lane) * H + h) : 0.f;
    };

    if (tid == 0) {
        if ((int)blockIdx.x < nitems) issue_tile(blockIdx.x);
        if ((int)blockIdx.x < nitems) issue_prev(blockIdx.x);
    }
    float gv_cur = 0.f, bv_cur = 0.f;
    if (warp == 2 && (int)blockIdx.x < nitems) load_gates(blockIdx.x, gv_cur, bv_cur);

    constexpr uint32_t idG = idesc_bf16(128, 32);
    uint32_t iter = 0;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++iter) {
        GDN_PREP_TRACE(iter, 0);
        const int gc = item / H, h = item % H;
        const int Lr = chunk_tab[gc].z;
        const bool prev = has_prev(gc);

        // Gram products D[r][n] = [K; Q]_r . K_n on the tensor cores, rows in lanes 0..63 (thread 0)
        if (tid == 0) {
            if (!mbar_wait(tile_full, iter & 1u, abort_flag)) {
                tc_abort(status, abort_flag);
            } else {
                tc_fence_after();
                const uint64_t a = sw128_desc(sbase + L::oTile, 0, 64);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint64_t o = sw128_ks_off(ks, 64);
                    mma_bf16(tmem, a + o, a + o, idG, ks > 0);
                }
                mma_commit(mma_bar);
                if (!mbar_wait(mma_bar, iter & 1u, abort_flag)) tc_abort(status, abort_flag);
            }
        } else if (tid == 96) {
            // G' = [K; Q] K_prev^T (thread 96), completes while the gates are applied.  A starts 64
            // rows (8 KB) before the tile, so row r of [K; Q] is row 64 + r of the product: lanes
            // 64..127, and its columns 32..63
            if (!mbar_wait(tile_full, iter & 1u, abort_flag) || !mbar_wait(prev_full, iter & 1u, abort_flag)) {
                tc_abort(status, abort_flag);
            } else {
                tc_fence_after();
                if (prev) {
                    const uint64_t a = sw128_desc(sbase + L::oTile - 8192, 0, 64);
                    const uint64_t bp = sw128_desc(sbase + L::oPrev, 0, 32);
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks)
                        mma_bf16(tmem + 32, a + sw128_ks_off(ks, 64), bp + sw128_ks_off(ks, 32), idG, ks > 0);
                }
                mma_commit(cross_bar);
            }
        }
        if (warp == 2) {
            // local cumulative log-gate and beta of this item; then prefetch the next item's
            float gv = gv_cur;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, gv, o);
                if (lane >= o) gv += y;
            }
            gam[lane] = gv * 1.4426950408889634f;    // log2(e) * gamma: gates become exp2 of differences
            bet[lane] = bv_cur;
            alph[lane] = exp2f(gv_cur * 1.4426950408889634f);
            if (item + (int)gridDim.x < nitems) load_gates(item + gridDim.x, gv_cur, bv_cur);
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 1);
        if (*abort_flag) break;
        tc_fence_after();
        if (warp < 2) {
            // lane r of warp 0: row r of K K^T -> A;  lane r of warp 1: row r of Q K^T -> P
            float d[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), d);
            tmem_ld_wait();
            GDN_PREP_TRACE(iter, 5);
            // lane r: decay ratios exp(gamma_r - gamma_j) = prod_{j < i <= r} exp(g_i) for j < r, as a
            // running product from the diagonal down (one multiply per entry instead of an exp2)
            const int r = lane;
            const float wr = (warp == 0) ? bet[r] : 1.f;
            const int lim = (warp == 0) ? r : r + 1;      // strictly lower for A, incl. diagonal for P
            float vals[32];
            float a = 1.f;
#pragma unroll
            for (int j = 31; j >= 0; --j) {
                a = (j >= r) ? 1.f : a * alph[j + 1];
                vals[j] = (j < lim) ? wr * a * d[j] : 0.f;
            }
            const uint32_t dst = sbase + ((warp == 0) ? L::oG : L::oP) + (uint32_t)(r * LD * 4);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst + q * 16), "f"(vals[4 * q]),
                             "f"(vals[4 * q + 1]), "f"(vals[4 * q + 2]), "f"(vals[4 * q + 3]));
            GDN_PREP_TRACE(iter, 6);
        } else {
            // warps 2 and 3: the tile buffer is free once G' has been formed (the chunk's own Gram
            // was waited for before the barrier above): fetch the next item's [K; Q] rows and
            // previous-chunk keys, then split G'
            if (tid == 64 && !mbar_wait(cross_bar, iter & 1u, abort_flag)) tc_abort(status, abort_flag);
            named_bar(1, 64);
            tc_fence_after();
            if (tid == 64 && !*abort_flag) {
                if (item + (int)gridDim.x < nitems) {
                    issue_tile(item + gridDim.x);
                    issue_prev(item + gridDim.x);
                }
            }
            if (prev) {
                // row (32 (w - 2) + lane) of G', in lane 32 w + lane -> three bf16 parts, K-major
                // 64-byte-swizzled A operand rows
                float e[32];
                tmem_ld32(tmem + 32 + ((uint32_t)(warp * 32) << 16), e);
                tmem_ld_wait();
                uint8_t* rec = op + ((size_t)gc * H + h) * kOpBytesB + kOpBCross;
                const int row = (warp - 2) * 32 + lane;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    uint32_t w1[4], w2[4], w3[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        bf16x2_split3(e[c8 * 8 + 2 * q], e[c8 * 8 + 2 * q + 1], w1[q], w2[q], w3[q]);
                    const uint32_t o = sw64_off_h(row, c8 * 8);
                    stg128(rec + o, w1);
                    stg128(rec + kOpBPart + o, w2);
                    stg128(rec + 2 * kOpBPart + o, w3);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        GDN_PREP_TRACE(iter, 2);

        // T11 (lanes 0..15, column j) and T22 (lanes 16..31, column j - 16) by forward substitution
        if (warp == 0) {
            const int blk = lane >> 4, j = lane & 15, o = blk * 16;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) t[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < 15; ++i) {
#pragma unroll
                for (int r = i + 1; r < 16; ++r) t[r] = fmaf(-G[(o + r) * LD + o + i], t[i], t[r]);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                Tm[(o + r) * LD + o + j] = t[r];
                Tm[(o + r) * LD + (16 - o) + j] = 0.f;   // upper-right block (overwritten below for blk 1)
            }
        }
        __syncthreads();
        {
            // M1 = A21 T11 (16 x 16): two outputs per thread; row r of A21 in four 16-byte loads,
            // the two T11 columns as pairs
            const int r = tid >> 3, c = (tid & 7) * 2;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
                const float4 av = *reinterpret_cast<const float4*>(G + (16 + r) * LD + 4 * m4);
                const float am[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 tv = *reinterpret_cast<const float2*>(Tm + (4 * m4 + e) * LD + c);
                    a0 = fmaf(am[e], tv.x, a0);
                    a1 = fmaf(am[e], tv.y, a1);
                }
            }
            *reinterpret_cast<float2*>(M1 + r * L::LM + c) = make_float2(a0, a1);
        }
        __syncthreads();
        {
            // T21 = -T22 M1, the same way
            const int r = tid >> 3, c = (tid & 7) * 2;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
                const float4 tv4 = *reinterpret_cast<const float4*>(Tm + (16 + r) * LD + 16 + 4 * m4);
                const float tm[4] = {tv4.x, tv4.y, tv4.z, tv4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 mv = *reinterpret_cast<const float2*>(M1 + (4 * m4 + e) * L::LM + c);
                    a0 = fmaf(tm[e], mv.x, a0);
                    a1 = fmaf(tm[e], mv.y, a1);
                }
            }
            *reinterpret_cast<float2*>(Tm + (16 + r) * LD + c) = make_float2(-a0, -a1);
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 3);

        // operator record: thread (a, cb) forms columns 4 cb .. 4 cb + 3 of rows 2a and 2a + 1 of
        // T'' = T diag(beta) and of P T'' = (P T) diag(beta) (a 2 x 4 block: each T row it loads
        // serves both rows), and writes each as three bf16 parts of 8 bytes per row into the
        // 64-byte-swizzled A-operand image (rows 0..31: T'', rows 32..63: P T'')
        uint8_t* dst = op + ((size_t)gc * H + h) * kOpBytesB;
        {
            const int i0 = (tid >> 3) * 2, c0 = (tid & 7) * 4;
            const float4 bv4 = *reinterpret_cast<const float4*>(bet + c0);
            const float bc[4] = {bv4.x, bv4.y, bv4.z, bv4.w};
            float acc[2][4];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[rr][c] = 0.f;
            const float4* p0 = reinterpret_cast<const float4*>(P + i0 * LD);
            const float4* p1 = reinterpret_cast<const float4*>(P + (i0 + 1) * LD);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 u0 = p0[q], u1 = p1[q];
                const float pa[4] = {u0.x, u0.y, u0.z, u0.w}, pb[4] = {u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 t = *reinterpret_cast<const float4*>(Tm + (4 * q + e) * LD + c0);
                    acc[0][0] = fmaf(pa[e], t.x, acc[0][0]);
                    acc[0][1] = fmaf(pa[e], t.y, acc[0][1]);
                    acc[0][2] = fmaf(pa[e], t.z, acc[0][2]);
                    acc[0][3] = fmaf(pa[e], t.w, acc[0][3]);
                    acc[1][0] = fmaf(pb[e], t.x, acc[1][0]);
                    acc[1][1] = fmaf(pb[e], t.y, acc[1][1]);
                    acc[1][2] = fmaf(pb[e], t.z, acc[1][2]);
                    acc[1][3] = fmaf(pb[e], t.w, acc[1][3]);
                }
            }
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int i = i0 + rr;
                const float4 tv4 = *reinterpret_cast<const float4*>(Tm + i * LD + c0);
                const float tv[4] = {tv4.x, tv4.y, tv4.z, tv4.w};
                uint32_t w1[2], w2[2], w3[2], x1[2], x2[2], x3[2];
#pragma unroll
                for (int c = 0; c < 4; c += 2) {
                    bf16x2_split3(tv[c] * bc[c], tv[c + 1] * bc[c + 1], w1[c / 2], w2[c / 2], w3[c / 2]);
                    bf16x2_split3(acc[rr][c] * bc[c], acc[rr][c + 1] * bc[c + 1], x1[c / 2], x2[c / 2], x3[c / 2]);
                }
                const uint32_t ot = sw64_off_h(i, c0), op2 = sw64_off_h(32 + i, c0);
                stg64(dst + ot, w1);
                stg64(dst + kOpBPart + ot, w2);
                stg64(dst + 2 * kOpBPart + ot, w3);
                stg64(dst + op2, x1);
                stg64(dst + kOpBPart + op2, x2);
                stg64(dst + 2 * kOpBPart + op2, x3);
            }
        }
        if (tid < 80) {
            float* gt = reinterpret_cast<float*>(dst + kOpBGate);
            const float gl = gam[31];
            float val = 0.f;
            if (tid < 32) val = exp2f(gam[tid]);
            else if (tid < 64) val = exp2f(gl - gam[tid - 32]);
            else if (tid == 64) val = exp2f(gl);
            gt[tid] = val;
        }
        (void)Lr;
        __syncthreads();
        GDN_PREP_TRACE(iter, 4);
    }
    tc_fence_before();
    __syncthreads();
    if ((tid == 0 || tid == 96) && *abort_flag) {
        // after a timeout, give the products this thread issued a bounded time to finish
        uint64_t* d = &drain[tid == 0 ? 0 : 1];
        mma_commit(d);
        volatile int never = 0;
        mbar_wait(d, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

}  // namespace gdn
