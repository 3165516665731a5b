// gdn_prefill_tc.cuh -- chunkwise WY/UT prefill of the gated delta rule on tcgen05 tensor cores.
//
// Ferrite project page, Design section 03 "Chunked Gated DeltaNet": a prompt is taken 32 rows at a
// time with the WY/UT chunk form of the delta rule, its products on TF32 tensor cores, split three
// ways for fp32-level accuracy, and the decoder continues from the state left at the prompt's end.
//
// Notation for one chunk of L <= 32 rows (rows L..31 are padding: q = k = v = 0, g = 0, beta = 0);
// S is the dv x dk state entering the chunk, s = 1/sqrt(dk):
//
//   gamma_i = g_0 + ... + g_i (chunk-local),  Gamma_i = exp(gamma_i),  delta_i = exp(gamma_31 - gamma_i)
//   A  = strictly-lower( diag(beta) (D o K K^T) ),  D_ij = exp(gamma_i - gamma_j)
//   T  = (I + A)^-1 (unit lower triangular),  T'' = T diag(beta)
//   P  = lower-including-diagonal( D o Q K^T )
//
// With X = K S^T and Z = Q S^T, the delta-rule writes of the chunk solve (I + A) U = diag(beta)
// (V - diag(Gamma) X), so U = T'' Y with Y = V - diag(Gamma) X, and
//
//   O  = s ( diag(Gamma) Z + P U )                 (inter-chunk part + intra-chunk attention)
//   S' = Gamma_31 S + (diag(delta) U)^T K          (inter-chunk state carry)
//
// Kernel 1 (gdn_prep_kernel, every (chunk, head) in parallel) builds the state-independent pieces:
// the Gram matrices [K; Q] K^T on the tensor cores, then A, P, the forward substitution for T,
// T'' and P T''.  It writes the 64 x 32 operator [T''; P T''] and the gate vectors per (chunk, head).
//
// Kernel 2 (gdn_scan_tc_kernel, one CTA per (sequence, head, slice of MS state rows)) walks the
// chunks in order.  Rows of S evolve independently (right multiplication), so a head's dv rows are
// split over dv/MS CTAs.  Per chunk, three dependent tensor-core products:
//
//   MMA_a  [X ; Z]     = [K ; Q] S^T            M=64, N=MS, K=dk
//   MMA_b  [U ; P U]   = [T'' ; P T''] Y        M=64, N=MS, K=32
//   MMA_c  (dS)^T      = K^T (diag(delta) U)    M=dk, N=MS, K=32
//
// with the elementwise steps between them done by the epilogue warps on tensor-memory rows.  Every
// product uses the 3xTF32 split (hi*hi + hi*lo + lo*hi).  These kernels serve fp32 q/k/v (bf16
// inputs take gdn_prep_pair.cuh / gdn_scan_pair.cuh).  The tensor-memory-access engine copies the
// chunks' fp32 q/k/v rows into shared memory and the producer warps split them into the operands
// while the current chunk runs.
#pragma once

#include "gdn_common.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

// Per-(chunk, head) operator record in the workspace.  It is the byte image that the scan kernels
// copy straight into shared memory: the TF32 hi and lo parts of [T''; P T''] (64 x 32, K-major,
// 128-byte swizzle) followed by the gate vectors Gamma[32], delta[32], Gamma_31 (fp32, padded).
constexpr uint32_t kOpHi = 0;
constexpr uint32_t kOpLo = 8192;
constexpr uint32_t kOpGate = 16384;
constexpr uint32_t kOpCopyBytes = 16384 + 80 * 4;   // staged per chunk (operator + gates)
constexpr uint32_t kOpBytes = 16384 + 512;          // record stride in the workspace

template <typename T>
struct ExactTF32 { static constexpr bool value = false; };
template <>
struct ExactTF32<__nv_bfloat16> { static constexpr bool value = true; };

// Shared-memory stores by 32-bit shared address.  No memory clobber: the compiler may move other
// loads and stores across them (none of the kernels' threads reads back what it stores before a
// fence or barrier, and those carry the clobber that orders everything).
__device__ __forceinline__ void sts4(uint32_t base, uint32_t off, float a, float b, float c, float d)
{
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "f"(a), "f"(b), "f"(c), "f"(d));
}
__device__ __forceinline__ void sts1(uint32_t base, uint32_t off, float a)
{
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(base + off), "f"(a));
}
// Global stores with the same property (no memory clobber).
__device__ __forceinline__ void stg1(void* p, float a)
{
    asm volatile("st.global.f32 [%0], %1;" ::"l"(p), "f"(a));
}
__device__ __forceinline__ void stg32(void* p, uint32_t a)
{
    asm volatile("st.global.b32 [%0], %1;" ::"l"(p), "r"(a));
}
__device__ __forceinline__ void stg128(void* p, const uint32_t (&w)[4])
{
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]));
}
__device__ __forceinline__ void stg64(void* p, const uint32_t (&w)[2])
{
    asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(w[0]), "r"(w[1]));
}

// Stores 8 consecutive K-elements (k0 % 8 == 0) of row r of a K-major SW128 tile of R rows, as hi
// (and lo when SPLIT) parts.
template <bool SPLIT>
__device__ __forceinline__ void put8(uint32_t hi, uint32_t lo, int r, int k0, int R, const float (&x)[8])
{
    using namespace sm100;
    const uint32_t o0 = sw128_off(r, k0, R), o1 = sw128_off(r, k0 + 4, R);
    if constexpr (SPLIT) {
        float h[8], l[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) tf32_split(x[i], h[i], l[i]);
        sts4(hi, o0, h[0], h[1], h[2], h[3]);
        sts4(hi, o1, h[4], h[5], h[6], h[7]);
        sts4(lo, o0, l[0], l[1], l[2], l[3]);
        sts4(lo, o1, l[4], l[5], l[6], l[7]);
    } else {
        sts4(hi, o0, x[0], x[1], x[2], x[3]);
        sts4(hi, o1, x[4], x[5], x[6], x[7]);
    }
}

// Stores N consecutive outputs with 16-byte stores (dst 16-byte aligned, N % 8 == 0).
template <typename T, int N>
__device__ __forceinline__ void store_row(T* dst, const float (&x)[N]);
template <int N>
__device__ __forceinline__ void store_row(__nv_bfloat16* dst, const float (&x)[N])
{
#pragma unroll
    for (int i = 0; i < N; i += 8) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(x[i + 2 * e], x[i + 2 * e + 1]);
        *reinterpret_cast<uint4*>(dst + i) = u;
    }
}
template <int N>
__device__ __forceinline__ void store_row(float* dst, const float (&x)[N])
{
#pragma unroll
    for (int i = 0; i < N; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
}

// Abort path shared by the tensor-core kernels: record the timeout once, tell the other warps.
__device__ __forceinline__ void tc_abort(int* status, volatile int* abort_flag)
{
    if (!*abort_flag) {
        *abort_flag = 1;
        report(status, GDN_ERR_TIMEOUT);
    }
}

// Optional phase-timing hooks (compiled out unless a build defines them).
#ifndef GDN_SCAN_TRACE
#define GDN_SCAN_TRACE(chunk, slot)
#endif
#ifndef GDN_PREP_TRACE
#define GDN_PREP_TRACE(iter, slot)
#endif

// Synchronisation rule of both kernels: exactly one thread performs each bounded mbarrier wait and
// records a timeout in the shared abort flag; a CTA-wide (or role-wide) barrier follows, after
// which every thread reads the abort flag.  So a timeout is seen by all threads at the same point,
// no thread is ever left waiting at a hardware barrier, and all of them reach the final barrier
// before the tensor memory is released.

// =================================================================================================
// Kernel 1: per (chunk, head) operator.  Persistent, 128 threads, work item = (global chunk, head).
// =================================================================================================
template <typename T, int DK>
struct PrepSmem {
    static constexpr bool EXACT = ExactTF32<T>::value;
    static constexpr uint32_t kTile = 64 * DK * 4;                    // [K;Q] SW128, 64 rows
    static constexpr uint32_t kTileHi = 0;
    static constexpr uint32_t kTileLo = kTile;                        // fp32 inputs only
    static constexpr uint32_t kF32 = kTile * (EXACT ? 1 : 2);         // start of plain fp32 scratch
    static constexpr int LD = 33;
    static constexpr uint32_t kG = kF32;                              // [32][33] K K^T -> A
    static constexpr uint32_t kP = kG + 32 * LD * 4;                  // [32][33] Q K^T -> P
    static constexpr uint32_t kT = kP + 32 * LD * 4;                  // [32][33] T''
    static constexpr uint32_t kGam = kT + 32 * LD * 4;                // [32] gamma
    static constexpr uint32_t kBet = kGam + 128;                      // [32] beta
    static constexpr uint32_t kBar = kBet + 128;                      // mbarriers: MMA, drain, tile
    static constexpr uint32_t kTmem = kBar + 24;                      // tmem base (4 B)
    static constexpr uint32_t kAbort = kTmem + 4;                     // abort flag (4 B)
    static constexpr uint32_t kTotal = kAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;                 // + alignment slack
};

template <typename T, int DK>
__global__ void __launch_bounds__(128, 4) gdn_prep_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                       const __grid_constant__ CUtensorMap tm_k,
                                                       const float* __restrict__ g, const float* __restrict__ beta,
                                                       const int* __restrict__ meta,
                                                       const int4* __restrict__ chunk_tab, float* __restrict__ op,
                                                       int H, int* status)
{
    using namespace sm100;
    using L = PrepSmem<T, DK>;
    constexpr bool EXACT = L::EXACT;
    static_assert(!EXACT, "fp32 inputs (bf16 inputs take the pair kernels)");
    constexpr int C = kChunk;
    // launched as a dependent of the plan kernel: its chunk table is read below
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float* G = reinterpret_cast<float*>(sm + L::kG);
    float* P = reinterpret_cast<float*>(sm + L::kP);
    float* Tm = reinterpret_cast<float*>(sm + L::kT);
    float* gam = reinterpret_cast<float*>(sm + L::kGam);
    float* bet = reinterpret_cast<float*>(sm + L::kBet);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* tile_full = bar + 2;            // the item's [K; Q] rows have landed
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::kTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kAbort);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar + 1, 1);
        mbar_init(tile_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const int nitems = meta[0] * H;
    constexpr uint32_t idesc = idesc_tf32(64, 32);
    uint32_t iter = 0;

    // The item's [K; Q] rows arrive by the tensor-memory-access engine, in fp32, straight into the
    // hi tile's 128-byte-swizzled layout (32 features x 32 rows per box: K rows 0..31, Q rows 32..63
    // of each 8 KB panel); the copy of the next item is issued once the Gram product has read the
    // tile, so it overlaps the triangular solve and the record.  Its gates are loaded a step ahead.
    auto issue_tile = [&](int item) {
        const int gc = item / H, h = item % H;
        const int t0 = chunk_tab[gc].y;
        mbar_arrive_expect_tx(tile_full, 64 * DK * 4);
#pragma unroll
        for (int p = 0; p < DK / 32; ++p) {
            tma_load_2d(sbase + L::kTileHi + p * 8192, &tm_k, h * DK + 32 * p, t0, tile_full);
            tma_load_2d(sbase + L::kTileHi + p * 8192 + 4096, &tm_q, h * DK + 32 * p, t0, tile_full);
        }
    };
    struct Pre {
        float gv, bv;
        int gc, h, Lr;
    };
    auto load_item = [&](Pre& p, int item) {
        p.gc = item / H;
        p.h = item % H;
        const int4 ct = chunk_tab[p.gc];
        const int64_t t0 = ct.y;
        p.Lr = ct.z;
        const bool ok = tid < p.Lr;
        p.gv = ok ? __ldg(g + (size_t)(t0 + tid) * H + p.h) : 0.f;
        p.bv = ok ? __ldg(beta + (size_t)(t0 + tid) * H + p.h) : 0.f;
    };
    Pre cur, nxt;
    if ((int)blockIdx.x < nitems) {
        load_item(cur, blockIdx.x);
        if (tid == 0) issue_tile(blockIdx.x);
    }

    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++iter) {
        GDN_PREP_TRACE(iter, 0);
        if (item + (int)gridDim.x < nitems) load_item(nxt, item + gridDim.x);
        const int gc = cur.gc, h = cur.h;

        // TF32 parts of the [K; Q] tile, in place: hi = x with its 13 low mantissa bits cleared, lo =
        // x - hi; rows past the chunk's end (the next tokens, or zeros past the tensor) become zero
        if (!mbar_wait(tile_full, iter & 1u, abort_flag)) tc_abort(status, abort_flag);
#pragma unroll 4
        for (int u = 0; u < 64 * DK / 4 / 128; ++u) {
            const int idx = tid + 128 * u;
            const int r = idx / (DK / 4), k0 = (idx % (DK / 4)) * 4;
            const uint32_t o = sw128_off(r, k0, 64);
            float4 x;
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                         : "r"(sbase + L::kTileHi + o));
            if ((r & 31) >= cur.Lr) x = make_float4(0.f, 0.f, 0.f, 0.f);
            float hi[4], lo[4];
            tf32_split(x.x, hi[0], lo[0]);
            tf32_split(x.y, hi[1], lo[1]);
            tf32_split(x.z, hi[2], lo[2]);
            tf32_split(x.w, hi[3], lo[3]);
            sts4(sbase + L::kTileHi, o, hi[0], hi[1], hi[2], hi[3]);
            sts4(sbase + L::kTileLo, o, lo[0], lo[1], lo[2], lo[3]);
        }
        if (tid < 32) {
            float gv = cur.gv;
            bet[tid] = cur.bv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                float y = __shfl_up_sync(0xffffffffu, gv, o);
                if (tid >= o) gv += y;
            }
            gam[tid] = gv;
        }
        fence_async_smem();
        __syncthreads();
        GDN_PREP_TRACE(iter, 1);

        // Gram matrices on the tensor cores: D[r][n] = [K;Q]_r . K_n  (M=64, N=32, K=DK)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dh = sw128_desc(sbase + L::kTileHi, 0, 64), dl = sw128_desc(sbase + L::kTileLo, 0, 64);
#pragma unroll
            for (int ks = 0; ks < DK / 8; ++ks) {
                const uint64_t o = sw128_ks_off(ks, 64);
                mma_tf32(tmem, dh + o, dh + o, idesc, ks > 0);
                if constexpr (!EXACT) {
                    mma_tf32(tmem, dh + o, dl + o, idesc, 1);
                    mma_tf32(tmem, dl + o, dh + o, idesc, 1);
                }
            }
            mma_commit(bar);
            if (!mbar_wait(bar, iter & 1u, abort_flag)) tc_abort(status, abort_flag);
            // the tile has been read: the next item's rows may land in it
            else if (item + (int)gridDim.x < nitems) issue_tile(item + gridDim.x);
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 2);
        if (*abort_flag) break;
        tc_fence_after();
        {
            float d[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), d);
            tmem_ld_wait();
            if (lane < 16) {
                const int r = warp * 16 + lane;             // M=64 accumulator: row 16w+t in lane 32w+t
                float* dst = (r < 32) ? (G + r * L::LD) : (P + (r - 32) * L::LD);
#pragma unroll
                for (int n = 0; n < 32; ++n) dst[n] = d[n];
            }
        }
        tc_fence_before();
        __syncthreads();
        GDN_PREP_TRACE(iter, 3);

        // gates: A (strictly lower) and P (lower incl. diagonal)
        for (int idx = tid; idx < C * C; idx += 128) {
            const int i = idx >> 5, j = idx & 31;
            const float dd = (j <= i) ? expf(gam[i] - gam[j]) : 0.f;
            G[i * L::LD + j] = (j < i) ? bet[i] * dd * G[i * L::LD + j] : 0.f;
            P[i * L::LD + j] = dd * P[i * L::LD + j];
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 4);
        // T = (I + A)^-1 by forward substitution, one lane per column j of T with the column in
        // registers.  Column-oriented: once t[i] is final it is subtracted, times column i of A,
        // from every later row, so each of the 31 steps is a set of independent FMAs.
        // T'' = T diag(beta).
        if (warp == 0) {
            const int j = lane;
            float t[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) t[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < 31; ++i) {
#pragma unroll
                for (int r = i + 1; r < 32; ++r) t[r] = fmaf(-G[r * L::LD + i], t[i], t[r]);
            }
            const float bj = bet[j];
#pragma unroll
            for (int i = 0; i < 32; ++i) Tm[i * L::LD + j] = t[i] * bj;
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 5);
        // operator record: [T''; P T''] split into TF32 hi/lo in the swizzled image, and the gates.
        // Thread (row group rg, column j) keeps column j of T'' in registers and forms 8 rows of
        // P T'' with full 32-term sums (P is zero above and T'' below the diagonal).
        uint8_t* dst = reinterpret_cast<uint8_t*>(op) + ((size_t)gc * H + h) * kOpBytes;
        {
            const int j = tid & 31, rg = tid >> 5;
            float tc[32];
#pragma unroll
            for (int m = 0; m < 32; ++m) tc[m] = Tm[m * L::LD + j];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i = rg * 8 + r;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 32; ++m) acc = fmaf(P[i * L::LD + m], tc[m], acc);
                float hi, lo;
                tf32_split(Tm[i * L::LD + j], hi, lo);          // row i of T''
                uint32_t o = sw128_off(i, j, 64);
                *reinterpret_cast<float*>(dst + kOpHi + o) = hi;
                *reinterpret_cast<float*>(dst + kOpLo + o) = lo;
                tf32_split(acc, hi, lo);                         // row 32 + i: (P T'')_i
                o = sw128_off(32 + i, j, 64);
                *reinterpret_cast<float*>(dst + kOpHi + o) = hi;
                *reinterpret_cast<float*>(dst + kOpLo + o) = lo;
            }
        }
        if (tid < 80) {
            float* gt = reinterpret_cast<float*>(dst + kOpGate);
            const float gl = gam[31];
            float val = 0.f;
            if (tid < 32) val = expf(gam[tid]);
            else if (tid < 64) val = expf(gl - gam[tid - 32]);
            else if (tid == 64) val = expf(gl);
            gt[tid] = val;
        }
        __syncthreads();
        GDN_PREP_TRACE(iter, 6);
        cur = nxt;
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        // after a timeout, give an MMA still in flight a bounded time to finish
        mma_commit(bar + 1);
        volatile int never = 0;
        mbar_wait(bar + 1, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 32);
}

// =================================================================================================
// Kernel 2: chunk-sequential scan on the tensor cores.
// grid (N, H, DV / MS), 256 threads: warps 0-3 consumers (tensor-memory epilogues; thread 0 issues
// the MMAs), warps 4-7 producers (operand staging for the next chunks, STAGES buffers).
// =================================================================================================
template <typename T, int DK, int MS, int STAGES>
struct ScanSmem {
    static constexpr bool EXACT = ExactTF32<T>::value;
    static constexpr uint32_t kAKQ = 64 * DK * 4;                     // [K;Q], 64 x DK
    static constexpr uint32_t kAKT = DK * 32 * 4;                     // K^T, DK x 32
    static constexpr uint32_t kAB = 64 * 32 * 4;                      // [T'';PT''], 64 x 32
    static constexpr uint32_t kB32 = ((2 * MS * 32 * 4) + 1023) & ~1023u; // [hi; lo] 2MS x 32 tile
    // one stage
    static constexpr uint32_t oAKQh = 0;
    static constexpr uint32_t oAKQl = oAKQh + kAKQ;
    static constexpr uint32_t oAKTh = oAKQl + (EXACT ? 0 : kAKQ);
    static constexpr uint32_t oAKTl = oAKTh + kAKT;
    static constexpr uint32_t oABh = oAKTl + (EXACT ? 0 : kAKT);
    static constexpr uint32_t oABl = oABh + kAB;
    static constexpr uint32_t oGate = oABl + kAB;                     // fp32 [80] (copied with the operator)
    static constexpr uint32_t oV = oGate + 80 * 4;                    // fp32 [MS][33] (V^T, padded)
    static constexpr uint32_t kStage = ((oV + 33 * MS * 4) + 1023) & ~1023u;
    // shared by all stages
    // B operands hold hi rows 0..MS-1 and lo rows MS..2MS-1 of one tile, so one MMA of N = 2MS
    // forms both the hi and the lo product of the split
    static constexpr uint32_t oBS = STAGES * kStage;                  // S: 2MS x DK
    static constexpr uint32_t oBY = oBS + 2 * MS * DK * 4;            // Y: 2MS x 32
    static constexpr uint32_t oBU = oBY + kB32;                       // U~: 2MS x 32
    // the next chunk's rows as copied by the tensor-memory-access engine, before they are split:
    // [K; Q] fp32 in the 128-byte-swizzled layout of the [K; Q] tile, V rows 0..31 x MS unswizzled
    static constexpr uint32_t oRawKQ = ((oBU + kB32) + 1023) & ~1023u;
    static constexpr uint32_t oRawV = oRawKQ + kAKQ;
    static constexpr uint32_t oBar = oRawV + 32 * MS * 4;             // full[S], empty[S], a, b, c, drain, raw
    static constexpr uint32_t oTmem = oBar + 8 * (2 * STAGES + 5);
    static constexpr uint32_t oAbort = oTmem + 4;
    static constexpr uint32_t kTotal = oAbort + 4;
    static constexpr uint32_t kBytes = kTotal + 1024;
};

template <typename T, int DK, int DV, int MS, int STAGES, int MINB>
__global__ void __launch_bounds__(256, MINB) gdn_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                             const __grid_constant__ CUtensorMap tm_k,
                                                             const __grid_constant__ CUtensorMap tm_v,
                                                             const int* __restrict__ meta,
                                                             const int* __restrict__ chunk_off,
                                                             const int4* __restrict__ chunk_tab,
                                                             const float* __restrict__ op,
                                                             const float* state_in, T* __restrict__ out,
                                                             float* state_out, float* __restrict__ snaps, int H,
                                                             int* status)
{
    using namespace sm100;
    using L = ScanSmem<T, DK, MS, STAGES>;
    constexpr bool EXACT = L::EXACT;
    static_assert(!EXACT, "fp32 inputs (bf16 inputs take the pair kernels)");
    // launched as a dependent of the prep kernel: its records (and the plan's table) are read below
    grid_dep_wait();
    static_assert(MS == 16 || MS == 32, "MS");
    static_assert(DK == 64 || DK == 128, "DK");
    static_assert(DV % MS == 0, "DV");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::oBar);
    uint64_t* empty = full + STAGES;
    uint64_t* bar_a = empty + STAGES;
    uint64_t* bar_b = bar_a + 1;
    uint64_t* bar_c = bar_a + 2;
    uint64_t* bar_drain = bar_a + 3;
    uint64_t* raw_full = bar_a + 4;           // the next chunk's raw rows have landed
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + L::oTmem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::oAbort);

    if (meta[1]) return;   // bad cu_seqlens: nothing is written
    const int n = blockIdx.x, h = blockIdx.y, r0 = blockIdx.z * MS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c_begin = chunk_off[n], c_end = chunk_off[n + 1];
    const int nch = c_end - c_begin;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(bar_a, 1);
        mbar_init(bar_b, 1);
        mbar_init(bar_c, 1);
        mbar_init(bar_drain, 1);
        mbar_init(raw_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tD1 = tmem, tD2 = tmem + 64, tD3 = tmem + 128;  // accumulators, 2MS columns each

    if (warp >= 4) {
        // ------------------------------------------------------------------ producers
        // The tensor-memory-access engine copies chunk cl + 1's [K; Q] rows (fp32, 32 features x 32
        // rows per box, in the [K; Q] tile's 128-byte-swizzled layout) and its V rows (MS columns)
        // into one raw buffer while chunk cl is converted; the [T''; P T''] image and the gates come
        // by one bulk copy per stage.  Per chunk and thread: DK/64 blocks of 4 tokens x 8 features of
        // K or Q and one 8-element group of the V slice, read back from the raw buffer, split into
        // TF32 hi and lo parts and stored as the MMA operands (K also transposed).  Rows past the
        // chunk's end (the next tokens, or zeros past the tensor) become zero.
        const int ptid = tid - 128;
        constexpr int NB = DK / 64;
        constexpr int NVG = 4 * MS;                    // 8-element groups in the V slice
        auto chunk_t0 = [&](int cl) { return chunk_tab[c_begin + cl].y; };
        auto issue_raw = [&](int cl) {
            const int t0 = chunk_t0(cl);
            mbar_arrive_expect_tx(raw_full, L::kAKQ + 32 * MS * 4);
#pragma unroll
            for (int p = 0; p < DK / 32; ++p) {
                tma_load_2d(sbase + L::oRawKQ + p * 8192, &tm_k, h * DK + 32 * p, t0, raw_full);
                tma_load_2d(sbase + L::oRawKQ + p * 8192 + 4096, &tm_q, h * DK + 32 * p, t0, raw_full);
            }
            tma_load_2d(sbase + L::oRawV, &tm_v, h * DV + r0, t0, raw_full);
        };
        // elements k0 .. k0 + 7 of a raw [K; Q] row: two 16-byte chunks, each at its swizzled place
        auto raw8 = [&](int row, int k0, float (&x)[8]) {
            const uint32_t o0 = sw128_off(row, k0, 64), o1 = sw128_off(row, k0 + 4, 64);
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]) : "r"(sbase + L::oRawKQ + o0));
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(x[4]), "=f"(x[5]), "=f"(x[6]), "=f"(x[7]) : "r"(sbase + L::oRawKQ + o1));
        };
        auto store_chunk = [&](int Lr, int s) {
            const uint32_t st = sbase + s * L::kStage;
            float* stf = reinterpret_cast<float*>(sm + s * L::kStage);
#pragma unroll
            for (int u = 0; u < NB; ++u) {
                const int b = ptid + 128 * u;
                const bool isq = b >= DK;
                const int bb = isq ? b - DK : b;
                const int jg = bb & 7, kg = bb >> 3;
                float x[4][8];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int j = 4 * jg + r;
                    raw8((isq ? 32 : 0) + j, kg * 8, x[r]);
                    if (j >= Lr) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[r][e] = 0.f;
                    }
                    put8<true>(st + L::oAKQh, st + L::oAKQl, (isq ? 32 : 0) + j, kg * 8, 64, x[r]);
                }
                if (!isq) {
                    // K^T: feature rows, 4 consecutive tokens per 16-byte store
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t o = sw128_off(kg * 8 + e, 4 * jg, DK);
                        float hi[4], lo[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) tf32_split(x[r][e], hi[r], lo[r]);
                        sts4(st + L::oAKTh, o, hi[0], hi[1], hi[2], hi[3]);
                        sts4(st + L::oAKTl, o, lo[0], lo[1], lo[2], lo[3]);
                    }
                }
            }
            if (ptid < NVG) {
                const int j = ptid / (MS / 8), cg = ptid % (MS / 8);
                float x[8];
                const float* vr = reinterpret_cast<const float*>(sm + L::oRawV) + j * MS + cg * 8;
                const float4 v0 = *reinterpret_cast<const float4*>(vr);
                const float4 v1 = *reinterpret_cast<const float4*>(vr + 4);
                x[0] = v0.x; x[1] = v0.y; x[2] = v0.z; x[3] = v0.w; x[4] = v1.x; x[5] = v1.y; x[6] = v1.z; x[7] = v1.w;
                float* Vt = stf + L::oV / 4;
#pragma unroll
                for (int e = 0; e < 8; ++e) Vt[(cg * 8 + e) * 33 + j] = (j < Lr) ? x[e] : 0.f;
            }
        };

        if (nch > 0 && ptid == 0) issue_raw(0);
        int issued = nch > 0 ? 1 : 0;
        for (int cl = 0; cl < nch; ++cl) {
            const int s = cl % STAGES;
            GDN_SCAN_TRACE(cl, 10);
            bool ok = mbar_wait(raw_full, (uint32_t)cl & 1u, abort_flag);
            if (ptid == 0 && ok && cl >= STAGES)
                ok = mbar_wait(&empty[s], (uint32_t)((cl / STAGES) - 1) & 1u, abort_flag);
            if (!ok) tc_abort(status, abort_flag);
            if (named_bar_any(1, 128, *abort_flag)) break;
            GDN_SCAN_TRACE(cl, 11);
            if (ptid == 0) {
                // operator image and gates: one bulk copy, counted by the same barrier
                mbar_expect_tx(&full[s], kOpCopyBytes);
                bulk_load(sbase + s * L::kStage + L::oABh,
                          reinterpret_cast<const uint8_t*>(op) + ((size_t)(c_begin + cl) * H + h) * kOpBytes,
                          kOpCopyBytes, &full[s]);
            }
            store_chunk(chunk_tab[c_begin + cl].z, s);
            fence_async_smem();
            mbar_arrive(&full[s]);
            // every producer has read the raw buffer: the next chunk's rows may land in it
            named_bar(1, 128);
            if (ptid == 0 && cl + 1 < nch) {
                issue_raw(cl + 1);
            }
            if (cl + 1 < nch) issued = cl + 2;
            GDN_SCAN_TRACE(cl, 12);
        }
        // after an abort, a copy still in flight lands before the CTA exits (bounded)
        if (ptid == 0 && issued > 0 && *abort_flag) {
            volatile int never = 0;
            mbar_wait(raw_full, (uint32_t)(issued - 1) & 1u, &never, 100000000ull);
        }
    } else {
        // ------------------------------------------------------------------ consumers
        // thread (warp, lane) owns column c of the state slice: S[0..MS)[c]
        const int c_own = (DK == 128) ? (warp * 32 + lane) : (warp * 16 + lane);
        const bool owns = (DK == 128) || (lane < 16);
        float S[MS];
#pragma unroll
        for (int i = 0; i < MS; ++i)
            S[i] = (state_in && owns) ? state_in[(((size_t)n * H + h) * DV + r0 + i) * DK + c_own] : 0.f;

        const float scale = rsqrtf((float)DK);
        constexpr uint32_t idA1 = idesc_tf32(64, MS), idA2 = idesc_tf32(64, 2 * MS);
        constexpr uint32_t idC1 = idesc_tf32(DK, MS), idC2 = idesc_tf32(DK, 2 * MS);
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int row16 = warp * 16 + lane;          // accumulator row of an M=64 product in this lane
        const int tok = (warp < 2) ? row16 : (row16 - 32);
        bool aborted = false;

        for (int cl = 0; cl <= nch; ++cl) {
            GDN_SCAN_TRACE(cl, 0);
            // S (initial, or after the previous chunk's carry) -> B operand of MMA_a
            if (owns) {
#pragma unroll
                for (int i = 0; i < MS; ++i) {
                    float hi, lo;
                    tf32_split(S[i], hi, lo);
                    sts1(sbase + L::oBS, sw128_off(i, c_own, 2 * MS), hi);
                    sts1(sbase + L::oBS, sw128_off(MS + i, c_own, 2 * MS), lo);
                }
            }
            if (cl == nch) break;
            fence_async_smem();
            tc_fence_before();
            named_bar(2, 128);      // every column of S written before MMA_a reads it
            GDN_SCAN_TRACE(cl, 1);
            const int s = cl % STAGES;
            const uint32_t st = sbase + s * L::kStage;
            const float* stf = reinterpret_cast<const float*>(sm + s * L::kStage);

            // ---- MMA_a: [X; Z] = [K; Q] S^T   (N = 2MS: columns [0, MS) hi, [MS, 2MS) lo)
            if (tid == 0) {
                if (!mbar_wait(&full[s], (uint32_t)(cl / STAGES) & 1u, abort_flag)) {
                    tc_abort(status, abort_flag);
                } else {
                    GDN_SCAN_TRACE(cl, 2);
                    tc_fence_after();
                    const uint64_t ah = sw128_desc(st + L::oAKQh, 0, 64), al = sw128_desc(st + L::oAKQl, 0, 64);
                    const uint64_t b = sw128_desc(sbase + L::oBS, 0, 2 * MS);
#pragma unroll
                    for (int ks = 0; ks < DK / 8; ++ks) {
                        const uint64_t oa = sw128_ks_off(ks, 64), ob = sw128_ks_off(ks, 2 * MS);
                        mma_tf32(tD1, ah + oa, b + ob, idA2, ks > 0);
                        if constexpr (!EXACT) mma_tf32(tD1, al + oa, b + ob, idA1, 1);   // lo x hi rows
                    }
                    mma_commit(bar_a);
                    GDN_SCAN_TRACE(cl, 3);
                    if (!mbar_wait(bar_a, (uint32_t)cl & 1u, abort_flag)) tc_abort(status, abort_flag);
                    GDN_SCAN_TRACE(cl, 4);
                }
            }
            named_bar(2, 128);
            GDN_SCAN_TRACE(cl, 13);
            if (*abort_flag) { aborted = true; break; }
            tc_fence_after();
            const int4 ctab = chunk_tab[c_begin + cl];
            const int64_t t0 = ctab.y;
            const int Lr = ctab.z;
            const float* gate = stf + L::oGate / 4;
            const float* Vs = stf + L::oV / 4;
            const float Gam = (lane < 16) ? gate[tok] : 0.f;
            const float del = (lane < 16 && warp < 2) ? gate[32 + tok] : 0.f;
            const float GamC = gate[64];
            float za[MS];
            {
                float xh[MS], xl[MS];
                tmem_ld<MS>(tD1 + lane_base, xh);
                tmem_ld<MS>(tD1 + lane_base + MS, xl);
                tmem_ld_wait();
                GDN_SCAN_TRACE(cl, 14);
#pragma unroll
                for (int i = 0; i < MS; ++i) za[i] = xh[i] + xl[i];
            }
            if (warp < 2) {
                // Y = V - diag(Gamma) X  ->  B operand of MMA_b (row i of S, K index = token)
                if (lane < 16) {
                    float vt[MS];
#pragma unroll
                    for (int i = 0; i < MS; ++i) vt[i] = Vs[i * 33 + tok];
#pragma unroll
                    for (int i = 0; i < MS; ++i) {
                        float hi, lo;
                        tf32_split(vt[i] - Gam * za[i], hi, lo);
                        sts1(sbase + L::oBY, sw128_off(i, tok, 2 * MS), hi);
                        sts1(sbase + L::oBY, sw128_off(MS + i, tok, 2 * MS), lo);
                    }
                }
                GDN_SCAN_TRACE(cl, 15);
                fence_async_smem();
            }
            tc_fence_before();
            named_bar(2, 128);
            // ---- MMA_b: [U; PU] = [T''; PT''] Y
            if (tid == 0) {
                GDN_SCAN_TRACE(cl, 5);
                tc_fence_after();
                const uint64_t ah = sw128_desc(st + L::oABh, 0, 64), al = sw128_desc(st + L::oABl, 0, 64);
                const uint64_t b = sw128_desc(sbase + L::oBY, 0, 2 * MS);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t oa = sw128_ks_off(ks, 64), ob = sw128_ks_off(ks, 2 * MS);
                    mma_tf32(tD2, ah + oa, b + ob, idA2, ks > 0);
                    mma_tf32(tD2, al + oa, b + ob, idA1, 1);       // lo x hi rows
                }
                mma_commit(bar_b);
                if (!mbar_wait(bar_b, (uint32_t)cl & 1u, abort_flag)) tc_abort(status, abort_flag);
                GDN_SCAN_TRACE(cl, 6);
            }
            named_bar(2, 128);
            if (*abort_flag) { aborted = true; break; }
            tc_fence_after();
            {
                float u[MS], ul[MS];
                tmem_ld<MS>(tD2 + lane_base, u);
                tmem_ld<MS>(tD2 + lane_base + MS, ul);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MS; ++i) u[i] += ul[i];
                if (warp < 2) {
                    // U~ = diag(delta) U  ->  B operand of MMA_c
                    if (lane < 16) {
#pragma unroll
                        for (int i = 0; i < MS; ++i) {
                            float hi, lo;
                            tf32_split(del * u[i], hi, lo);
                            sts1(sbase + L::oBU, sw128_off(i, tok, 2 * MS), hi);
                            sts1(sbase + L::oBU, sw128_off(MS + i, tok, 2 * MS), lo);
                        }
                    }
                    fence_async_smem();
                } else if (lane < 16 && tok < Lr) {
                    // O = s (diag(Gamma) Z + P U)
                    float o[MS];
#pragma unroll
                    for (int i = 0; i < MS; ++i) o[i] = scale * fmaf(Gam, za[i], u[i]);
                    store_row<MS>(out + ((size_t)(t0 + tok) * H + h) * DV + r0, o);
                }
            }
            tc_fence_before();
            named_bar(2, 128);
            // ---- MMA_c: dS^T = K^T U~   (its completion also frees the stage buffer)
            if (tid == 0) {
                GDN_SCAN_TRACE(cl, 7);
                tc_fence_after();
                const uint64_t ah = sw128_desc(st + L::oAKTh, 0, DK), al = sw128_desc(st + L::oAKTl, 0, DK);
                const uint64_t b = sw128_desc(sbase + L::oBU, 0, 2 * MS);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t oa = sw128_ks_off(ks, DK), ob = sw128_ks_off(ks, 2 * MS);
                    mma_tf32(tD3, ah + oa, b + ob, idC2, ks > 0);
                    if constexpr (!EXACT) mma_tf32(tD3, al + oa, b + ob, idC1, 1);   // lo x hi rows
                }
                mma_commit(bar_c);
                mma_commit(&empty[s]);
                if (!mbar_wait(bar_c, (uint32_t)cl & 1u, abort_flag)) tc_abort(status, abort_flag);
                GDN_SCAN_TRACE(cl, 8);
            }
            named_bar(2, 128);
            if (*abort_flag) { aborted = true; break; }
            tc_fence_after();
            {
                // S' = Gamma_31 S + dS   (row c_own of dS^T; for dk = 64 the M=64 layout puts row
                // 16w+t in lane 32w+t, which is c_own of that lane)
                float ds[MS], dl[MS];
                tmem_ld<MS>(tD3 + lane_base, ds);
                tmem_ld<MS>(tD3 + lane_base + MS, dl);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < MS; ++i) S[i] = fmaf(GamC, S[i], ds[i] + dl[i]);
                // the state at a cut point the caller asked a snapshot of
                const int snap = chunk_tab[c_begin + cl].w;
                if (snap >= 0 && snaps != nullptr && owns) {
#pragma unroll
                    for (int i = 0; i < MS; ++i) snaps[(((size_t)snap * H + h) * DV + r0 + i) * DK + c_own] = S[i];
                }
            }
            GDN_SCAN_TRACE(cl, 9);
            tc_fence_before();
        }
        if (state_out && owns && !aborted) {
#pragma unroll
            for (int i = 0; i < MS; ++i) state_out[(((size_t)n * H + h) * DV + r0 + i) * DK + c_own] = S[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {
        // after a timeout, give MMAs still in flight a bounded time to finish before the tensor
        // memory they write is released
        mma_commit(bar_drain);
        volatile int never = 0;
        mbar_wait(bar_drain, 0, &never, 100000000ull);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace gdn
