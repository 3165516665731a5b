// gdn_plan.cuh -- chunk tables of a packed prefill call, and the workspace layout.
//
// Chunks of C = 32 rows restart at every sequence start (Ferrite project page, Design section 03:
// prompt rows go through the layer in chunks of 32; section 07: prompts are cut at the same points
// with or without a resume).  One CTA validates cu_seqlens on the device, counts the chunks of
// each sequence, scans them into per-sequence chunk offsets and fills a table that maps a global
// chunk index to (sequence, first token, rows).  Every later kernel reads these tables, so the
// host never has to read cu_seqlens back.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

// Workspace layout of gdn_chunk_prefill (all offsets 256-byte aligned).
struct PrefillLayout {
    int64_t nc_max;       // upper bound on the number of chunks: floor(T / C) + N
    size_t off_meta;      // int32[8]: [0] chunk count, [1] seqlens error flag
    size_t off_chunk_off; // int32[N + 1]: first global chunk of each sequence
    size_t off_chunk_tab; // int4[nc_max]: (sequence, first token, rows, 0)
    size_t off_op;        // [nc_max][H] operator records (up to 25088 bytes each)
    size_t total;

    static size_t align(size_t x) { return (x + 255) & ~size_t(255); }

    PrefillLayout(int64_t T, int N, int H, int dk)
    {
        nc_max = T / kChunk + N;
        size_t o = 0;
        off_meta = o;      o = align(o + 8 * sizeof(int));
        off_chunk_off = o; o = align(o + (size_t)(N + 1) * sizeof(int));
        off_chunk_tab = o; o = align(o + (size_t)nc_max * sizeof(int4));
        off_op = o;        o = align(o + (size_t)nc_max * H * 25088);   // largest record of the two paths
        total = o;
        (void)dk;
    }
};

// inclusive scan over a block of 1024 threads
__device__ __forceinline__ int block_inclusive_scan_1024(int x, int* warp_tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    if (warp > 0) x += warp_tot[warp - 1];
    __syncthreads();
    return x;
}

// <<<1, 1024>>>.  cu_seqlens may be null: N sequences of equal length `fixed_len`.
__global__ void __launch_bounds__(1024) gdn_plan_kernel(const int32_t* __restrict__ cu, int N, int64_t T,
                                                    int fixed_len, int* meta, int* chunk_off,
                                                    int4* chunk_tab, int* status)
{
    __shared__ int warp_tot[32];
    __shared__ int s_err;
    __shared__ int s_running;
    if (threadIdx.x == 0) { s_err = 0; s_running = 0; }
    __syncthreads();

    for (int base = 0; base < N; base += 1024) {
        const int n = base + threadIdx.x;
        int nch = 0;
        if (n < N) {
            int64_t a = cu ? (int64_t)cu[n] : (int64_t)n * fixed_len;
            int64_t b = cu ? (int64_t)cu[n + 1] : (int64_t)(n + 1) * fixed_len;
            bool bad = (b < a) || (n == 0 && a != 0) || (n == N - 1 && b != T) || b > T;
            if (bad) s_err = 1;
            int64_t L = bad ? 0 : b - a;
            nch = (int)((L + kChunk - 1) / kChunk);
        }
        const int incl = block_inclusive_scan_1024(nch, warp_tot);
        if (n < N) chunk_off[n] = s_running + incl - nch;
        __syncthreads();
        if (threadIdx.x == 1023) s_running += incl;
        __syncthreads();
    }
    const int nc = s_running;
    if (threadIdx.x == 0) {
        chunk_off[N] = nc;
        meta[0] = s_err ? 0 : nc;
        meta[1] = s_err;
        if (s_err) report(status, GDN_ERR_BAD_SEQLENS);
    }
    if (s_err) return;
    __syncthreads();
    // global chunk -> (sequence, first token, rows)
    for (int gc = threadIdx.x; gc < nc; gc += 1024) {
        int lo = 0, hi = N - 1;               // largest n with chunk_off[n] <= gc
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (chunk_off[mid] <= gc) lo = mid; else hi = mid - 1;
        }
        const int n = lo;
        const int64_t a = cu ? (int64_t)cu[n] : (int64_t)n * fixed_len;
        const int64_t b = cu ? (int64_t)cu[n + 1] : (int64_t)(n + 1) * fixed_len;
        const int64_t t0 = a + (int64_t)(gc - chunk_off[n]) * kChunk;
        const int64_t rows = (b - t0 < kChunk) ? (b - t0) : kChunk;
        chunk_tab[gc] = make_int4(n, (int)t0, (int)rows, 0);
    }
}

}  // namespace gdn
