// gdn_prep_pair.cuh -- per-(pair of chunks, head) WY/UT operator for bf16 q/k (sm_100a).
//
// The chunkwise WY/UT form (Ferrite project page, Design section 03) takes each chunk of 32 rows with
// T = (I + A)^-1.  The bf16 scan advances the state once per pair of chunks (rows 0..31: chunk a,
// rows 32..63: chunk b), and this kernel builds the pair's operator record for it:
//
//   A = strictly-lower(diag(beta) (D o K K^T)),  P = lower-incl-diagonal(D o Q K^T),
//   D_ij = exp(gamma_i - gamma_j)   (gamma: cumulative log-gate from the pair's first row),
//   T = (I + A)^-1 = [[T_a, 0], [T_ba, T_b]],   T_a, T_b: the two chunks' 32 x 32 inverses,
//   T_ba = -T_b A_ba T_a,   T'' = T diag(beta),
//
// and writes [T''; P T''] (128 x 64) as three bf16 parts in the 128-byte-swizzled K-major layout of a
// tensor-core A operand, with Gamma_i = exp(gamma_i) and delta_i = exp(gamma_63 - gamma_i).  A
// chunk's own inverse uses the same 2 x 2 block form one level down (16 x 16 blocks by forward
// substitution, then T21 = -T22 A21 T11), which shortens the dependent chain of the substitution.
//
// What is specific to bf16 inputs: the pair's [K; Q] rows are exact bf16 values, so the tensor-
// memory-access engine copies them straight into the operand layout and one bf16 tensor-core product
// (M = 128, N = 64, K = dk) forms both Gram matrices exactly in fp32.  The gates are applied while the
// Gram rows come out of tensor memory.  P T'' is a second tensor-core product (M = 64, N = 64,
// K = 64): P and T'' as three bf16 parts each, the six part products with p + q <= 4 accumulated in
// fp32, which keeps every term above 2^-24 relative (fp32-accurate).  T'' is staged in exactly the
// byte layout of the record's rows 0..63 (the product's B operand), and P T'' the same way for rows
// 64..127; both leave for the record by bulk stores from shared memory.
//
// Rows past a sequence's end (the pair's last rows may hold the next sequence's tokens) get g = 0
// and beta = 0: their rows of A and columns of T'' are zero, so they never reach the scan's state.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "gdn_common.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

template <int DK>
struct PrepPairSmem {
    static constexpr int NP = DK / 64;
    static constexpr uint32_t kPanel = 128 * 128;                    // [K; Q]: 128 rows x 128 B per panel
    // The tile region holds the item's [K; Q] rows until the Gram product has read them, then the
    // block products of the inverse and the three parts of T'' (8 KB each, the B operand of P T''),
    // then the next item's rows (copied once P T'' has read T'').
    static constexpr uint32_t oTile = 0;
    static constexpr uint32_t oTpp = 0;                              // T'' parts: 3 x 64 rows x 128 B
    static constexpr int LM = 36;
    static constexpr uint32_t oM = 3 * 8192;                         // [32][LM] block products
    static constexpr uint32_t kTileRegion0 = (NP * kPanel > oM + 32 * LM * 4) ? NP * kPanel : oM + 32 * LM * 4;
    static constexpr uint32_t kTileRegion = (kTileRegion0 + 1023) & ~1023u;
    static constexpr int LD = 68;                                    // fp32 row pitch (16-byte rows)
    // A and T share one buffer: each block of T is written over a block of A that has been read
    // for the last time (the diagonal blocks by their own substitution, the off-diagonal ones after
    // the product that consumes them).  Column 67 of row i >= 32 holds exp(gamma_i - gamma_31).
    static constexpr uint32_t oA = kTileRegion;                      // [64][LD] A, then T
    static constexpr uint32_t oT = oA;
    static constexpr uint32_t oPp = oA + 64 * LD * 4;                // P parts: 3 x 64 rows x 128 B
    static constexpr uint32_t oGam = oPp + 3 * 8192;                 // [64] log2(e) gamma
    static constexpr uint32_t oBet = oGam + 256;                     // [64] beta
    static constexpr uint32_t oAlph = oBet + 256;                    // [64] exp(g), 4 spare
    static constexpr uint32_t oBar = oAlph + 272;                    // tile_full, gram, pt, drain
    static constexpr uint32_t oTmem = oBar + 32;
    static constexpr uint32_t oClaim = oTmem + 8;                   // the item claimed two ahead
    static constexpr uint32_t oAbort = oClaim + 4;
    static constexpr uint32_t kTotal = oAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;
    static_assert(oA % 1024 == 0 && oPp % 1024 == 0, "operand tiles on 1024-byte boundaries");
};

// CTAs resident per SM (shared memory and registers are sized for it; the launch sizes its grid so)
constexpr int kPrepPairCtasPerSm = 3;
constexpr int kPrepPairThreads = 256;
static_assert(kPrepPairCtasPerSm * (PrepPairSmem<128>::kBytes + 1024) <= 233472, "three CTAs per SM");

template <int DK>
__global__ void __launch_bounds__(kPrepPairThreads, kPrepPairCtasPerSm)
    gdn_prep_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const float* __restrict__ g, const float* __restrict__ beta, int* __restrict__ meta,
                         const int4* __restrict__ chunk_tab, uint8_t* __restrict__ op, int H, int* status)
{
    using namespace sm100;
    using L = PrepPairSmem<DK>;
    constexpr int NP = L::NP;
    constexpr int LD = L::LD, LM = L::LM;
    // launched as a dependent of the plan kernel: its pair table is read below
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float* A = reinterpret_cast<float*>(sm + L::oA);
    float* Tm = reinterpret_cast<float*>(sm + L::oT);
    float* M = reinterpret_cast<float*>(sm + L::oM);
    float* gam = reinterpret_cast<float*>(sm + L::oGam);
    float* bet = reinterpret_cast<float*>(sm + L::oBet);
    float* alph = reinterpret_cast<float*>(sm + L::oAlph);
    uint64_t* tile_full = reinterpret_cast<uint64_t*>(sm + L::oBar);
    uint64_t* mma_bar = tile_full + 1;        // the Gram product done
    uint64_t* pt_bar = tile_full + 2;         // P T'' done
    uint64_t* drain = tile_full + 3;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::oTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::oAbort);
    volatile int* s_claim = reinterpret_cast<volatile int*>(sm + L::oClaim);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nitems = meta[0] * H;
    // Items: each CTA starts with item blockIdx.x, then takes the next unclaimed one from a counter
    // (zeroed by the plan kernel), so that CTAs that finish early take more items.  The item after
    // the current one is claimed an iteration ahead, so its rows and gates can be fetched early.
    auto claim = [&]() { return (int)gridDim.x + atomicAdd(meta + 2, 1); };
    if (tid == 0) {
        mbar_init(tile_full, 1);
        mbar_init(mma_bar, 1);
        mbar_init(pt_bar, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        *s_claim = ((int)blockIdx.x < nitems) ? claim() : nitems;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 64);      // the Gram product (128 lanes x 64 columns), then P T
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    int next = *s_claim;

    // copies the [K; Q] rows of one item into the tile buffer (one thread; issued once the previous
    // item's product has read the buffer).  Panel p: K rows 0..63, then Q rows 0..63.
    auto issue_tile = [&](int item, int t0) {
        const int h = item % H;
        const int t1 = (t0 < INT32_MAX - 32) ? t0 + 32 : INT32_MAX;   // rows past the tensor read as zeros
        mbar_arrive_expect_tx(tile_full, NP * L::kPanel);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            const uint32_t pan = sbase + L::oTile + p * L::kPanel;
            tma_load_2d(pan, &tm_k, h * DK + p * 64, t0, tile_full);
            tma_load_2d(pan + 4096, &tm_k, h * DK + p * 64, t1, tile_full);
            tma_load_2d(pan + 8192, &tm_q, h * DK + p * 64, t0, tile_full);
            tma_load_2d(pan + 12288, &tm_q, h * DK + p * 64, t1, tile_full);
        }
    };
    // gate inputs of one item for lane `lane` of warp 7: rows 2 lane and 2 lane + 1 (zero past the
    // pair's rows)
    auto load_gates = [&](int item, float (&gv)[2], float (&bv)[2]) {
        const int gc = item / H, h = item % H;
        const int4 ct = chunk_tab[gc];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = 2 * lane + e;
            const bool ok = r < ct.z;
            gv[e] = ok ? __ldg(g + (size_t)(ct.y + r) * H + h) : 0.f;
            bv[e] = ok ? __ldg(beta + (size_t)(ct.y + r) * H + h) : 0.f;
        }
    };

    if (tid == 0 && (int)blockIdx.x < nitems) issue_tile(blockIdx.x, chunk_tab[blockIdx.x / H].y);
    float gv_cur[2] = {0.f, 0.f}, bv_cur[2] = {0.f, 0.f};
    if (warp == 7 && (int)blockIdx.x < nitems) load_gates(blockIdx.x, gv_cur, bv_cur);

    constexpr uint32_t idG = idesc_bf16(128, 64);
    constexpr float kLog2e = 1.4426950408889634f;
    uint32_t iter = 0;
    for (int item = blockIdx.x; item < nitems; ++iter) {
        GDN_PREP_TRACE(iter, 0);
        const int gc = item / H, h = item % H;
        // first token of the next item, read now so that its copy can be issued without waiting;
        // and the item after it, published by the barrier below
        int next_t0 = 0;
        if (tid == 64 && next < nitems) {
            next_t0 = chunk_tab[next / H].y;
            *s_claim = claim();
        }

        // Gram products D[r][n] = [K; Q]_r . K_n, n < 64, on the tensor cores (thread 0)
        if (tid == 0) {
            bulk_wait_read();   // the last item's record stores have read the P parts' place
            if (!mbar_wait(tile_full, iter & 1u, abort_flag)) {
                tc_abort(status, abort_flag);
            } else {
                tc_fence_after();
                const uint64_t a = sw128_desc(sbase + L::oTile, 0, 128);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint64_t o = sw128_ks_off(ks, 128);
                    mma_bf16(tmem, a + o, a + o, idG, ks > 0);
                }
                mma_commit(mma_bar);
                if (!mbar_wait(mma_bar, iter & 1u, abort_flag)) tc_abort(status, abort_flag);
            }
        } else if (warp == 7) {
            // cumulative log-gate over the pair (two rows per lane), beta, exp(g), and the running
            // products exp(gamma_i - gamma_31) of the second chunk's rows; then prefetch the next item's
            const float s2 = gv_cur[0] + gv_cur[1];
            float inc = s2;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            const float ex = inc - s2;
            const float a0 = exp2f(gv_cur[0] * kLog2e), a1 = exp2f(gv_cur[1] * kLog2e);
            // product of exp(g) over rows 32 .. 2 lane + 1 (lanes 16..31; the others multiply by 1)
            const float pp = (lane >= 16) ? a0 * a1 : 1.f;
            float incp = pp;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incp, o);
                if (lane >= o) incp *= y;
            }
            const int r = 2 * lane;
            gam[r] = (ex + gv_cur[0]) * kLog2e;
            gam[r + 1] = inc * kLog2e;
            bet[r] = bv_cur[0];
            bet[r + 1] = bv_cur[1];
            alph[r] = a0;
            alph[r + 1] = a1;
            const float exclp = __shfl_up_sync(0xffffffffu, incp, 1);
            if (lane >= 16) {
                A[r * LD + 67] = (lane > 16 ? exclp : 1.f) * a0;
                A[(r + 1) * LD + 67] = incp;
            }
            if (next < nitems) load_gates(next, gv_cur, bv_cur);
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 1);
        const int after_next = (next < nitems) ? *s_claim : nitems;
        if (*abort_flag) break;
        tc_fence_after();
        {
            // thread (q = warp % 4, hf = warp / 4, lane): Gram row r = 32 q + lane, columns 32 hf ..
            // 32 hf + 31.  Rows 0..63: K K^T -> A (times beta_i, strictly lower); rows 64..127:
            // Q K^T -> P (lower, with the diagonal).  Decay ratios exp(gamma_i - gamma_j) as a running
            // product from the diagonal down (one multiply per entry instead of an exp2).
            const int q = warp & 3, hf = warp >> 2;
            const int r = q * 32 + lane;
            const bool isP = r >= 64;
            const int i = r & 63;
            const float wr = isP ? 1.f : bet[i];
            const int lim = isP ? i + 1 : i;
            const int jtop = 32 * hf + 31;
            float a = (i > jtop) ? A[i * LD + 67] : 1.f;
            const uint32_t dst = sbase + L::oA + (uint32_t)(i * LD * 4 + hf * 128);
            // two halves of 16 columns, high half first (the running product goes down the row).
            // A rows: fp32 for the inverse; P rows: three bf16 parts, the A operand of P T''.
            // both halves' tensor-memory loads in flight before one wait
            float dd[2][16];
            tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + 32 * hf + 16, dd[1]);
            tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + 32 * hf, dd[0]);
            tmem_ld_wait();
#pragma unroll
            for (int half = 1; half >= 0; --half) {
                const float (&d)[16] = dd[half];
                float vals[16];
#pragma unroll
                for (int jj = 15; jj >= 0; --jj) {
                    const int j = 32 * hf + 16 * half + jj;
                    if (half == 0 || jj < 15) a = (j >= i) ? 1.f : a * alph[j + 1];
                    vals[jj] = (j < lim) ? wr * a * d[jj] : 0.f;
                }
                if (!isP) {
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst + half * 64 + c4 * 16),
                                     "f"(vals[4 * c4]), "f"(vals[4 * c4 + 1]), "f"(vals[4 * c4 + 2]),
                                     "f"(vals[4 * c4 + 3]));
                } else {
#pragma unroll
                    for (int g8 = 0; g8 < 2; ++g8) {
                        uint32_t w[3][4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            bf16x2_split3(vals[8 * g8 + 2 * e], vals[8 * g8 + 2 * e + 1], w[0][e], w[1][e], w[2][e]);
                        const uint32_t o = sw128_off_h(i, 32 * hf + 16 * half + 8 * g8, 64);
#pragma unroll
                        for (int pp = 0; pp < 3; ++pp)
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sbase + L::oPp + pp * 8192 + o),
                                         "r"(w[pp][0]), "r"(w[pp][1]), "r"(w[pp][2]), "r"(w[pp][3]));
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        GDN_PREP_TRACE(iter, 2);

        if (warp < 2) {
            // the four 16 x 16 diagonal blocks of T by forward substitution: lane -> block
            // 2 warp + lane / 16, column j
            const int blk = 2 * warp + (lane >> 4), j = lane & 15, o = blk * 16;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) t[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < 15; ++i) {
#pragma unroll
                for (int r = i + 1; r < 16; ++r) t[r] = fmaf(-A[(o + r) * LD + o + i], t[i], t[r]);
            }
            __syncwarp();      // every lane has read this block of A before T is written over it
#pragma unroll
            for (int r = 0; r < 16; ++r) Tm[(o + r) * LD + o + j] = t[r];
            if ((blk & 1) == 0) {
#pragma unroll
                for (int r = 0; r < 16; ++r) Tm[(o + r) * LD + o + 16 + j] = 0.f;   // upper right of a chunk
            }
        } else {
            // T is zero above the chunk blocks: rows 0..31, columns 32..63
            for (int e = tid - 64; e < 32 * 8; e += 192) {
                const int r = e >> 3, c4 = e & 7;
                *reinterpret_cast<float4*>(Tm + r * LD + 32 + 4 * c4) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        __syncthreads();
        {
            // per chunk (tid / 128): M16 = A21 T11 (16 x 16), two outputs per thread
            const int ch = tid >> 7, t = tid & 127, o = 32 * ch;
            const int r = t >> 3, c = (t & 7) * 2;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
                const float4 av = *reinterpret_cast<const float4*>(A + (o + 16 + r) * LD + o + 4 * m4);
                const float am[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 tv = *reinterpret_cast<const float2*>(Tm + (o + 4 * m4 + e) * LD + o + c);
                    a0 = fmaf(am[e], tv.x, a0);
                    a1 = fmaf(am[e], tv.y, a1);
                }
            }
            *reinterpret_cast<float2*>(M + ch * 16 * 16 + r * 16 + c) = make_float2(a0, a1);
        }
        __syncthreads();
        {
            // T21 = -T22 M16 inside each chunk
            const int ch = tid >> 7, t = tid & 127, o = 32 * ch;
            const int r = t >> 3, c = (t & 7) * 2;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
                const float4 tv4 = *reinterpret_cast<const float4*>(Tm + (o + 16 + r) * LD + o + 16 + 4 * m4);
                const float tm[4] = {tv4.x, tv4.y, tv4.z, tv4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 mv = *reinterpret_cast<const float2*>(M + ch * 16 * 16 + (4 * m4 + e) * 16 + c);
                    a0 = fmaf(tm[e], mv.x, a0);
                    a1 = fmaf(tm[e], mv.y, a1);
                }
            }
            *reinterpret_cast<float2*>(Tm + (o + 16 + r) * LD + o + c) = make_float2(-a0, -a1);
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 3);
        // four consecutive columns of a row of T'' = T diag(beta) as three bf16 parts (8 bytes each) in
        // the 128-byte-swizzled layout of 64 rows x 64 columns: the B operand of P T'' (K = row, N =
        // column, N-major) and, copied by bulk stores, the record's rows 0..63
        auto put_tpp4 = [&](int row, int col, float4 t) {
            const float4 b = *reinterpret_cast<const float4*>(bet + col);
            uint32_t w[3][2];
            bf16x2_split3(t.x * b.x, t.y * b.y, w[0][0], w[1][0], w[2][0]);
            bf16x2_split3(t.z * b.z, t.w * b.w, w[0][1], w[1][1], w[2][1]);
            const uint32_t o = sw128_off_h(row, col, 64);
#pragma unroll
            for (int pp = 0; pp < 3; ++pp)
                asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sbase + L::oTpp + pp * 8192 + o), "r"(w[pp][0]),
                             "r"(w[pp][1]));
        };
        {
            // M32 = A_ba T_a (32 x 32; T_a lower triangular): thread -> row r, columns c0 .. c0 + 3
            const int r = tid >> 3, c0 = (tid & 7) * 4;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int m = c0; m < 32; m += 4) {
                const float4 av = *reinterpret_cast<const float4*>(A + (32 + r) * LD + m);
                const float am[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 tv = *reinterpret_cast<const float4*>(Tm + (m + e) * LD + c0);
                    acc[0] = fmaf(am[e], tv.x, acc[0]);
                    acc[1] = fmaf(am[e], tv.y, acc[1]);
                    acc[2] = fmaf(am[e], tv.z, acc[2]);
                    acc[3] = fmaf(am[e], tv.w, acc[3]);
                }
            }
            *reinterpret_cast<float4*>(M + r * LM + c0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            // the blocks of T'' that are final already: T_a (rows 0..31), zero above it, T_b
            put_tpp4(r, c0, *reinterpret_cast<const float4*>(Tm + r * LD + c0));
            put_tpp4(r, 32 + c0, make_float4(0.f, 0.f, 0.f, 0.f));
            put_tpp4(32 + r, 32 + c0, *reinterpret_cast<const float4*>(Tm + (32 + r) * LD + 32 + c0));
        }
        __syncthreads();
        {
            // T_ba = -T_b M32 (T_b lower triangular)
            const int r = tid >> 3, c0 = (tid & 7) * 4;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int m = 0; m <= r; m += 4) {
                const float4 tv4 = *reinterpret_cast<const float4*>(Tm + (32 + r) * LD + 32 + m);
                const float tb[4] = {tv4.x, tv4.y, tv4.z, tv4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 mv = *reinterpret_cast<const float4*>(M + (m + e) * LM + c0);
                    acc[0] = fmaf(tb[e], mv.x, acc[0]);
                    acc[1] = fmaf(tb[e], mv.y, acc[1]);
                    acc[2] = fmaf(tb[e], mv.z, acc[2]);
                    acc[3] = fmaf(tb[e], mv.w, acc[3]);
                }
            }
            const float4 tba = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
            *reinterpret_cast<float4*>(Tm + (32 + r) * LD + c0) = tba;
            put_tpp4(32 + r, c0, tba);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        GDN_PREP_TRACE(iter, 4);

        uint8_t* dst = op + ((size_t)gc * H + h) * kPairRecordBytes;
        GDN_PREP_TRACE(iter, 6);
        // P T'' on the tensor cores (thread 0): M = 64 (row r in lane 32 (r / 16) + r % 16), N = 64,
        // K = 64; part products a_p t_q with p + q <= 4 into one fp32 accumulator (the Gram's columns)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idPT = idesc_bf16(64, 64, false, true);
            const uint64_t da = sw128_desc(sbase + L::oPp, 0, 64);
            const uint64_t db = sw128_desc_mn(sbase + L::oTpp, 8192, 1024);
            constexpr int pa[6] = {0, 0, 0, 1, 1, 2}, pb[6] = {0, 1, 2, 0, 1, 0};
#pragma unroll
            for (int ks = 0; ks < kPair / 16; ++ks) {
#pragma unroll
                for (int u = 0; u < 6; ++u)
                    mma_bf16(tmem, da + (uint64_t)(pa[u] * 512 + ks * 2), db + (uint64_t)(pb[u] * 512 + ks * 128), idPT,
                             ks > 0 || u > 0);
            }
            mma_commit(pt_bar);
            if (!mbar_wait(pt_bar, iter & 1u, abort_flag)) tc_abort(status, abort_flag);
        } else if (tid == 64) {
            // record rows 0..63: the T'' images, while the product reads them too (this thread also
            // refills the tile region, after its stores have read it)
#pragma unroll
            for (int pp = 0; pp < 3; ++pp) bulk_store(dst + pp * kPairPart, sbase + L::oTpp + pp * 8192, 8192);
            bulk_commit();
        } else if (tid >= 128) {
            // gates, while P T'' runs: Gamma_i (i < 64), then delta_i = Gamma_63 / Gamma_i as exp2 of
            // the difference
            float* gt = reinterpret_cast<float*>(dst + kPairGate);
            const int e = tid - 128;
            gt[e] = (e < 64) ? exp2f(gam[e]) : exp2f(gam[63] - gam[e - 64]);
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 7);
        tc_fence_after();
        // the tile region is free once P T'' (completed) and the record stores (waited for here) have
        // read T'': fetch the next item's rows
        if (tid == 64) {
            bulk_wait_read();
            if (next < nitems && !*abort_flag) issue_tile(next, next_t0);
        }
        {
            // P T'' rows -> record rows 64..127, staged as three 8 KB images in the P parts' place (the
            // product has read them) and copied by bulk stores.  Rows 16 q .. 16 q + 15 of an M = 64
            // product sit in lanes 0..15 of lane quarter q; warp (q, hf) reads columns 32 hf .. + 31 of
            // them, one half of the columns per half-warp
            const int q = warp & 3, hf = warp >> 2;
            float d[16];
            // lanes 0..15 of the quarter, twice: threads 0..15 columns 32 hf .. + 15, threads 16..31
            // columns 32 hf + 16 .. + 31 of the same rows
            tmem_ld16x2(tmem + ((uint32_t)(q * 32) << 16) + 32 * hf, d);
            tmem_ld_wait();
            {
                const int i = 16 * q + (lane & 15), cb = 32 * hf + 16 * (lane >> 4);
#pragma unroll
                for (int g8 = 0; g8 < 2; ++g8) {
                    uint32_t w[3][4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        bf16x2_split3(d[8 * g8 + 2 * e], d[8 * g8 + 2 * e + 1], w[0][e], w[1][e], w[2][e]);
                    const uint32_t o = sw128_off_h(i, cb + 8 * g8, 64);
#pragma unroll
                    for (int pp = 0; pp < 3; ++pp)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sbase + L::oPp + pp * 8192 + o),
                                     "r"(w[pp][0]), "r"(w[pp][1]), "r"(w[pp][2]), "r"(w[pp][3]));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        GDN_PREP_TRACE(iter, 5);
        if (tid == 0) {
            // record rows 64..127; the P parts' place is rewritten after the next item's first barrier
#pragma unroll
            for (int pp = 0; pp < 3; ++pp)
                bulk_store(dst + pp * kPairPart + 8192, sbase + L::oPp + pp * 8192, 8192);
            bulk_commit();
        }
        item = next;
        next = after_next;
    }
    if (tid == 0 || tid == 64) bulk_wait_all();   // the record stores are complete before the CTA exits
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        // after a timeout, give the product this thread issued a bounded time to finish
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

}  // namespace gdn
