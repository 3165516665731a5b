// gdn_plan.cuh -- chunk tables of a packed prefill call, and the workspace layout.
//
// Chunks of C = 32 rows (the fp32 path) or pairs of them (64 rows, the bf16 path) restart at every
// sequence start (Ferrite project page, Design section 03:
// the layer takes a prompt 32 rows at a time) and at every cut point the caller asks a state
// snapshot for (section 07: the prompt cache saves state where each turn ends and splits a prompt at
// identical places with or without a resume, which is what makes a resumed reply equal to a full one).
// A segment is the piece of a sequence between two such boundaries.  One CTA validates cu_seqlens
// and the cut points on the device, places the segments in token order, counts and scans their
// chunks, and fills a table that maps a global chunk index to (sequence, first token, rows,
// snapshot index or -1); the last chunk of a segment that ends at cut i carries i.  Every later
// kernel reads these tables, so the host never has to read cu_seqlens back.
#pragma once

#include "gdn_common.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_sm100.cuh"

namespace gdn {

// Workspace layout of gdn_chunk_prefill (all offsets 256-byte aligned).  NS = number of segments
// (sequences + cut points).
struct PrefillLayout {
    int64_t nc_max;       // upper bound on the number of 32-row chunks: floor(T / 32) + NS
    int64_t np_max;       // upper bound on the number of 64-row pairs: floor(T / 64) + NS
    size_t off_meta;      // int32[8]: [0] chunk (or pair) count, [1] error flag, [2] prep item counter
    size_t off_chunk_off; // int32[NS + 1]: first global chunk (or pair) of each sequence
    size_t off_chunk_tab; // int4[nc_max]: (sequence, first token, rows, snapshot index or -1)
    size_t off_seg;       // int32[6 NS + 1]: segment start, sequence, cut, end, snapshot, chunk offset
    size_t off_order;     // int32[NS]: the sequences in the order the bf16 scan takes them
    size_t off_op;        // operator records: [nc_max][H] x 16,896 B (fp32 path) or
                          // [np_max][H] x 49,664 B (bf16 path), whichever is larger
    size_t total;

    static size_t align(size_t x) { return (x + 255) & ~size_t(255); }

    PrefillLayout(int64_t T, int NS, int H, int dk)
    {
        nc_max = T / kChunk + NS;
        np_max = T / kPair + NS;
        const size_t rec_f32 = (size_t)nc_max * H * kOpBytes;
        const size_t rec_pair = (size_t)np_max * H * kPairRecordBytes;
        size_t o = 0;
        off_meta = o;      o = align(o + 8 * sizeof(int));
        off_chunk_off = o; o = align(o + (size_t)(NS + 1) * sizeof(int));
        off_chunk_tab = o; o = align(o + (size_t)nc_max * sizeof(int4));
        off_seg = o;       o = align(o + (size_t)(6 * NS + 1) * sizeof(int));
        off_order = o;     o = align(o + (size_t)NS * sizeof(int));
        off_op = o;        o = align(o + (rec_f32 > rec_pair ? rec_f32 : rec_pair));
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

// number of elements of the sorted array a[0..n) that are < x (or <= x)
__device__ __forceinline__ int count_less(const int32_t* a, int n, int64_t x, bool or_equal)
{
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const bool below = or_equal ? ((int64_t)a[mid] <= x) : ((int64_t)a[mid] < x);
        if (below) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// <<<1, 1024>>>.  cu_seqlens may be null: N sequences of equal length `fixed_len`.  cuts: n_cuts
// token offsets, strictly increasing, each strictly inside one sequence (may be null when n_cuts
// is 0).  seg: the workspace's segment arrays, 6 (N + n_cuts) + 1 ints.
// The order in which the bf16 scan takes the sequences of a packed call: most chunks first (ties by
// index).  The scan's CTAs are numbered with the sequence's rank slowest, so the longest sequences'
// CTAs start first and shorter ones fill the SMs behind them; a packed call then ends close to
// max(longest sequence, total chunks / SMs) instead of whenever its longest sequence happened to
// start.  Ranks are counted in one pass per sequence (sequences <= 1024), identity order beyond.
__device__ __forceinline__ void plan_order(int N, const int* chunk_off, int* order, int* s_cnt)
{
    if (N > 1024) {
        for (int n = threadIdx.x; n < N; n += 1024) order[n] = n;
        return;
    }
    const int n = threadIdx.x;
    if (n < N) s_cnt[n] = chunk_off[n + 1] - chunk_off[n];
    __syncthreads();
    if (n < N) {
        const int cn = s_cnt[n];
        int r = 0;
        for (int m = 0; m < N; ++m) {
            const int cm = s_cnt[m];
            r += (cm > cn) || (cm == cn && m < n);
        }
        order[r] = n;
    }
}

// CL: rows per table entry (32: chunks, 64: pairs of chunks).
template <int CL>
__global__ void __launch_bounds__(1024) gdn_plan_kernel(const int32_t* __restrict__ cu, int N, int64_t T,
                                                    int fixed_len, const int32_t* __restrict__ cuts, int n_cuts,
                                                    int* meta, int* chunk_off, int4* chunk_tab, int* seg,
                                                    int* order, int* status)
{
    __shared__ int s_cnt[1024];
    __shared__ int warp_tot[32];
    __shared__ int s_err;
    __shared__ int s_running;
    // the prep kernel is launched as a dependent: let it become resident while this runs (it waits
    // for this kernel's writes before reading them)
    sm100::grid_dep_launch();
    if (threadIdx.x == 0) { s_err = 0; s_running = 0; }
    __syncthreads();
    auto start_of = [&](int n) -> int64_t { return cu ? (int64_t)cu[n] : (int64_t)n * fixed_len; };
    const int NS = N + n_cuts;
    int* seg_start = seg;
    int* seg_seq = seg + NS;
    int* seg_cut = seg + 2 * NS;
    int* seg_end = seg + 3 * NS;
    int* seg_snap = seg + 4 * NS;
    int* seg_off = seg + 5 * NS;        // NS + 1

    if (n_cuts == 0) {
        // no cut points: one segment per sequence, chunk counts scanned directly
        for (int base = 0; base < N; base += 1024) {
            const int n = base + threadIdx.x;
            int nch = 0;
            if (n < N) {
                const int64_t a = start_of(n), b = start_of(n + 1);
                const bool bad = (b < a) || (n == 0 && a != 0) || (n == N - 1 && b != T) || b > T;
                if (bad) s_err = 1;
                nch = bad ? 0 : (int)((b - a + CL - 1) / CL);
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
            meta[2] = 0;                  // the bf16 prep's item counter
            if (s_err) report(status, GDN_ERR_BAD_SEQLENS);
        }
        if (s_err) return;
        __syncthreads();
        for (int gc = threadIdx.x; gc < nc; gc += 1024) {
            int lo = 0, hi = N - 1;               // largest n with chunk_off[n] <= gc
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (chunk_off[mid] <= gc) lo = mid; else hi = mid - 1;
            }
            const int64_t t0 = start_of(lo) + (int64_t)(gc - chunk_off[lo]) * CL;
            const int64_t e = start_of(lo + 1);
            chunk_tab[gc] = make_int4(lo, (int)t0, (int)((e - t0) < CL ? (e - t0) : CL), -1);
        }
        plan_order(N, chunk_off, order, s_cnt);
        return;
    }

    // validation
    for (int n = threadIdx.x; n < N; n += 1024) {
        const int64_t a = start_of(n), b = start_of(n + 1);
        if ((b < a) || (n == 0 && a != 0) || (n == N - 1 && b != T) || b > T) s_err = 1;
    }
    for (int i = threadIdx.x; i < n_cuts; i += 1024) {
        const int64_t c = cuts[i];
        if (i + 1 < n_cuts && (int64_t)cuts[i + 1] <= c) s_err = 1;
        if (c <= 0 || c >= T) s_err = 1;
    }
    __syncthreads();
    if (!s_err) {
        // a cut must lie strictly inside the sequence that starts last at or before it
        for (int i = threadIdx.x; i < n_cuts; i += 1024) {
            const int64_t c = cuts[i];
            int lo = 0, hi = N - 1;                // largest m with start(m) <= c
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (start_of(mid) <= c) lo = mid; else hi = mid - 1;
            }
            if (!(start_of(lo) < c && c < start_of(lo + 1))) s_err = 1;
        }
    }
    __syncthreads();
    if (s_err) {
        if (threadIdx.x == 0) {
            meta[0] = 0;
            meta[1] = 1;
            report(status, GDN_ERR_BAD_SEQLENS);
        }
        return;
    }
    // segments in token order: sequence starts merged with cut points
    for (int n = threadIdx.x; n < N; n += 1024) {
        const int64_t a = start_of(n);
        const int j = n + (n_cuts ? count_less(cuts, n_cuts, a, false) : 0);
        seg_start[j] = (int)a;
        seg_seq[j] = n;
        seg_cut[j] = -1;
        chunk_off[n] = j;                   // replaced by the chunk offset below
    }
    for (int i = threadIdx.x; i < n_cuts; i += 1024) {
        const int64_t c = cuts[i];
        int lo = 0, hi = N - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (start_of(mid) <= c) lo = mid; else hi = mid - 1;
        }
        const int j = i + lo + 1;
        seg_start[j] = (int)c;
        seg_seq[j] = lo;
        seg_cut[j] = i;
    }
    __syncthreads();
    // segment ends, snapshot indices and chunk counts; scan into chunk offsets
    for (int base = 0; base < NS; base += 1024) {
        const int j = base + threadIdx.x;
        int nch = 0;
        if (j < NS) {
            const int sq = seg_seq[j];
            int end, snap;
            if (j + 1 < NS && seg_seq[j + 1] == sq && seg_cut[j + 1] >= 0) {
                end = seg_start[j + 1];
                snap = seg_cut[j + 1];
            } else {
                end = (int)start_of(sq + 1);
                snap = -1;
            }
            seg_end[j] = end;
            seg_snap[j] = snap;
            nch = (end - seg_start[j] + CL - 1) / CL;
        }
        const int incl = block_inclusive_scan_1024(nch, warp_tot);
        if (j < NS) seg_off[j] = s_running + incl - nch;
        __syncthreads();
        if (threadIdx.x == 1023) s_running += incl;
        __syncthreads();
    }
    const int nc = s_running;
    for (int n = threadIdx.x; n < N; n += 1024) chunk_off[n] = seg_off[chunk_off[n]];
    if (threadIdx.x == 0) {
        seg_off[NS] = nc;
        chunk_off[N] = nc;
        meta[0] = nc;
        meta[1] = 0;
        meta[2] = 0;
    }
    __syncthreads();
    // global chunk -> (sequence, first token, rows, snapshot index)
    for (int gc = threadIdx.x; gc < nc; gc += 1024) {
        int lo = 0, hi = NS - 1;              // largest j with seg_off[j] <= gc and a chunk of its own
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (seg_off[mid] <= gc) lo = mid; else hi = mid - 1;
        }
        while (lo + 1 < NS && seg_off[lo + 1] <= gc) ++lo;
        const int j = lo;
        const int t0 = seg_start[j] + (gc - seg_off[j]) * CL;
        const int rows = (seg_end[j] - t0 < CL) ? (seg_end[j] - t0) : CL;
        const int snap = (t0 + rows == seg_end[j]) ? seg_snap[j] : -1;
        chunk_tab[gc] = make_int4(seg_seq[j], t0, rows, snap);
    }
    plan_order(N, chunk_off, order, s_cnt);
}

}  // namespace gdn
