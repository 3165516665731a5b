// gdn_api.cu -- C ABI of libgdn.so: argument checks, workspace layout and kernel launches.
//
// Every entry point declared in include/gdn.h is defined here.  The kernels live in the .cuh files
// included below, so the whole library is one translation unit and the per-device status word is
// one symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>
#include <type_traits>
#include <utility>
#include <string>
#include <vector>

#include "gdn_common.cuh"
#include "gdn_decode.cuh"
#include "gdn_norm.cuh"
#include "gdn_plan.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_prep_pair.cuh"
#include "gdn_scan_pair.cuh"

namespace gdn {

// First device-detected error since the last gdn_get_device_status (one per device).
__device__ int g_status;

static int* status_ptr()
{
    static std::mutex mu;
    static int* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<int*>(p);
    }
    return cache[dev];
}

// ---- detail of the last CUDA error met by a library call on this thread (gdn_last_error) ----------
static thread_local char g_last_err[256] = "";

// Returns e == cudaSuccess; otherwise records "what: <CUDA's message>" for gdn_last_error.
static bool cuda_ok(cudaError_t e, const char* what)
{
    if (e == cudaSuccess) return true;
    snprintf(g_last_err, sizeof(g_last_err), "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
    return false;
}

template <typename K>
static bool set_dyn_smem(K kernel, size_t bytes, const char* name)
{
    return cuda_ok(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes), name);
}

// ---- optional per-kernel event timing (gdn_profile_start / gdn_profile_stop) ----------------------
struct ProfRec {
    const char* name;
    cudaEvent_t a, b;
};
static std::mutex g_prof_mu;
static bool g_prof_on = false;
static std::vector<ProfRec> g_prof_recs;
static std::vector<cudaEvent_t> g_prof_pool;

static cudaEvent_t prof_event()
{
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Records an event pair around one launch when profiling is on.
struct ProfScope {
    ProfRec rec{nullptr, nullptr, nullptr};
    cudaStream_t st;
    ProfScope(const char* name, cudaStream_t s) : st(s)
    {
        std::lock_guard<std::mutex> lock(g_prof_mu);
        if (!g_prof_on) return;
        rec.name = name;
        rec.a = prof_event();
        rec.b = prof_event();
        cudaEventRecord(rec.a, st);
    }
    ~ProfScope()
    {
        if (!rec.name) return;
        cudaEventRecord(rec.b, st);
        std::lock_guard<std::mutex> lock(g_prof_mu);
        g_prof_recs.push_back(rec);
    }
};

// Launches `kernel` as a programmatic dependent of the previous kernel in the stream: it may become
// resident before that kernel ends and waits for it (grid_dep_wait) before reading its results.
template <typename... Params, typename... Args>
static cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                    Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    cuda_ok(e, "cudaLaunchKernelEx");
    return e;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
static bool head_ok(int d) { return d == 64 || d == 128; }

template <typename T, int DK, int DV>
static int launch_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         float* state, void* out, int B, int H, bool norm, cudaStream_t st)
{
    ProfScope prof("gdn_decode_step_kernel", st);
    auto kern = norm ? gdn_decode_step_kernel<T, DK, DV, true> : gdn_decode_step_kernel<T, DK, DV, false>;
    constexpr int RB = (GDN_DECODE_RB < DV) ? GDN_DECODE_RB : DV;
    if (launch_dependent(kern, dim3((unsigned)B * H * (DV / RB)), dim3(GDN_DECODE_NT), 0, st, static_cast<const T*>(q),
                         static_cast<const T*>(k), static_cast<const T*>(v), g, beta, state, static_cast<T*>(out),
                         H) != cudaSuccess)
        return GDN_ERR_LAUNCH;
    return GDN_OK;
}

template <typename T>
static int dispatch_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           float* state, void* out, int B, int H, int dk, int dv, bool norm, cudaStream_t st)
{
    if (dk == 128 && dv == 128) return launch_decode<T, 128, 128>(q, k, v, g, beta, state, out, B, H, norm, st);
    if (dk == 128 && dv == 64) return launch_decode<T, 128, 64>(q, k, v, g, beta, state, out, B, H, norm, st);
    if (dk == 64 && dv == 128) return launch_decode<T, 64, 128>(q, k, v, g, beta, state, out, B, H, norm, st);
    return launch_decode<T, 64, 64>(q, k, v, g, beta, state, out, B, H, norm, st);
}

template <typename T, int DK, int DV>
static int launch_verify(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         const float* state_in, float* states_out, void* out, const int32_t* parents, int B,
                         int Tk, int H, bool norm, cudaStream_t st)
{
    int* status = status_ptr();
    if (!status) return GDN_ERR_CUDA;
    ProfScope prof("gdn_decode_verify_kernel", st);
    auto kern = parents ? (norm ? gdn_decode_verify_kernel<T, DK, DV, true, true>
                                : gdn_decode_verify_kernel<T, DK, DV, false, true>)
                        : (norm ? gdn_decode_verify_kernel<T, DK, DV, true, false>
                                : gdn_decode_verify_kernel<T, DK, DV, false, false>);
    constexpr int RB = (GDN_DECODE_RB < DV) ? GDN_DECODE_RB : DV;
    if (launch_dependent(kern, dim3((unsigned)B * H * (DV / RB)), dim3(256), 0, st, static_cast<const T*>(q),
                         static_cast<const T*>(k), static_cast<const T*>(v), g, beta, state_in, states_out,
                         static_cast<T*>(out), parents, status, H, Tk) != cudaSuccess)
        return GDN_ERR_LAUNCH;
    return GDN_OK;
}

template <typename T>
static int dispatch_verify(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const float* state_in, float* states_out, void* out, const int32_t* parents, int B,
                           int Tk, int H, int dk, int dv, bool norm, cudaStream_t st)
{
#define GDN_VF(DK_, DV_)                                                                                   \
    if (dk == DK_ && dv == DV_)                                                                            \
        return launch_verify<T, DK_, DV_>(q, k, v, g, beta, state_in, states_out, out, parents, B, Tk, H, norm, st);
    GDN_VF(128, 128)
    GDN_VF(128, 64)
    GDN_VF(64, 128)
#undef GDN_VF
    return launch_verify<T, 64, 64>(q, k, v, g, beta, state_in, states_out, out, parents, B, Tk, H, norm, st);
}

// ---- tensor maps (2-D tiled views of q/k/v) -------------------------------------------------------
// cuTensorMapEncodeTiled is taken from the driver through the runtime's entry-point query, so the
// library does not link libcuda directly.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [rows, inner] matrix of 2-byte (bf16) or 4-byte (fp32) elements with row stride `row_elems`,
// tiles of box_rows x box_inner elements; rows past the end read as zeros.
// swizzle: 128 or 64 (bytes of the swizzle span), 0 for none
static bool make_tmap(CUtensorMap* m, bool f32, const void* base, uint64_t inner, uint64_t rows, uint64_t row_elems,
                      uint32_t box_inner, uint32_t box_rows, int swizzle)
{
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_elems * (f32 ? 4 : 2)};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                             : (swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE),
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

#ifndef GDN_SCAN_MS
#define GDN_SCAN_MS 32
#endif
#ifndef GDN_SCAN_MINB
#define GDN_SCAN_MINB 1
#endif

// column groups per lane quarter of the bf16 scan's chain warps (compile-time tuning knob)
#ifndef GDN_PAIR_NQ
#define GDN_PAIR_NQ 2
#endif

static int g_num_sms = 0;

// cut points of one prefill call and where their state snapshots go (n = 0: none)
struct Cuts {
    const int32_t* pos = nullptr;
    int n = 0;
    float* snaps = nullptr;
};

template <typename T, int DK, int DV>
static int launch_prefill(const PrefillLayout& lay, char* ws, const void* q, const void* k, const void* v,
                          const float* g, const float* beta, const int32_t* cu, int N, int64_t T_total,
                          int fixed_len, const float* state_in, void* out, float* state_out, int H,
                          const Cuts& cuts, cudaStream_t st)
{
    int* status = status_ptr();
    if (!status) return GDN_ERR_CUDA;
    int* meta = reinterpret_cast<int*>(ws + lay.off_meta);
    int* chunk_off = reinterpret_cast<int*>(ws + lay.off_chunk_off);
    int4* chunk_tab = reinterpret_cast<int4*>(ws + lay.off_chunk_tab);
    float* op = reinterpret_cast<float*>(ws + lay.off_op);
    int* seg = reinterpret_cast<int*>(ws + lay.off_seg);
    int* order = reinterpret_cast<int*>(ws + lay.off_order);
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) g_num_sms = 148;
    }

    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    {
        // table entries: pairs of chunks on the bf16 path, chunks on the fp32 path
        ProfScope prof("gdn_plan_kernel", st);
        gdn_plan_kernel<kBf16 ? kPair : kChunk><<<1, 1024, 0, st>>>(cu, N, T_total, fixed_len, cuts.pos, cuts.n, meta,
                                                                    chunk_off, chunk_tab, seg, order, status);
    }
    if (!cuda_ok(cudaPeekAtLastError(), "gdn_plan_kernel launch")) return GDN_ERR_LAUNCH;

    // Tensor maps of q, k, v: 32-row boxes.  bf16: 64 features (128 bytes) per box row of q/k, 128-byte
    // swizzle; 32 v columns, 64-byte swizzle.  fp32: 32 features (128 bytes) of q/k, 128-byte
    // swizzle; the scan's MS v columns unswizzled.
    constexpr int MSF = GDN_SCAN_MS;
    CUtensorMap tq{}, tk{}, tv{};
    {
        const uint64_t Tn = (uint64_t)(T_total > 0 ? T_total : 1);
        const bool f32 = !kBf16;
        const uint32_t kbox = kBf16 ? 64 : 32, vbox = kBf16 ? 32 : MSF;
        if (!make_tmap(&tq, f32, q, (uint64_t)H * DK, Tn, (uint64_t)H * DK, kbox, 32, 128) ||
            !make_tmap(&tk, f32, k, (uint64_t)H * DK, Tn, (uint64_t)H * DK, kbox, 32, 128) ||
            !make_tmap(&tv, f32, v, (uint64_t)H * DV, Tn, (uint64_t)H * DV, vbox, 32, kBf16 ? 64 : 0))
            return GDN_ERR_CUDA;
    }
    if constexpr (kBf16) {
      if (lay.np_max > 0 && T_total > 0) {
        using PL = PrepPairSmem<DK>;
        auto k1 = gdn_prep_pair_kernel<DK>;
        if (!set_dyn_smem(k1, PL::kBytes, "cudaFuncSetAttribute(max dynamic shared memory)"))
            return GDN_ERR_LAUNCH;
        const int64_t items = lay.np_max * (int64_t)H;
        const int64_t cap = (int64_t)g_num_sms * kPrepPairCtasPerSm;
        const unsigned grid = (unsigned)(items < cap ? items : cap);
        ProfScope prof("gdn_prep_pair_kernel", st);
        if (launch_dependent(k1, dim3(grid), dim3(kPrepPairThreads), PL::kBytes, st, tq, tk, g, beta,
                             meta, (const int4*)chunk_tab, reinterpret_cast<uint8_t*>(op), H,
                             status) != cudaSuccess)
            return GDN_ERR_LAUNCH;
      }
    } else if (lay.nc_max > 0 && T_total > 0) {
        using PL = PrepSmem<T, DK>;
        auto k1 = gdn_prep_kernel<T, DK>;
        if (!set_dyn_smem(k1, PL::kBytes, "cudaFuncSetAttribute(max dynamic shared memory)"))
            return GDN_ERR_LAUNCH;
        const int64_t items = lay.nc_max * (int64_t)H;
        const int64_t cap = (int64_t)g_num_sms * 4;
        const unsigned grid = (unsigned)(items < cap ? items : cap);
        ProfScope prof("gdn_prep_kernel", st);
        if (launch_dependent(k1, dim3(grid), dim3(128), PL::kBytes, st, tq, tk, g, beta, (const int*)meta,
                             (const int4*)chunk_tab, op, H, status) != cudaSuccess)
            return GDN_ERR_LAUNCH;
    }
    if constexpr (kBf16) {
        // bf16 inputs: operands staged by tensor maps, bf16 tensor-core products, two chunks per step
        using SP = ScanPairSmem<DK>;
        static_assert(SP::kBytes <= 227 * 1024, "bf16 scan shared memory");
        constexpr int NQ = GDN_PAIR_NQ;
        auto kb = cuts.n > 0 ? gdn_scan_pair_kernel<DK, DV, true, NQ> : gdn_scan_pair_kernel<DK, DV, false, NQ>;
        if (!set_dyn_smem(kb, SP::kBytes, "cudaFuncSetAttribute(max dynamic shared memory)"))
            return GDN_ERR_LAUNCH;
        {
            ProfScope prof("gdn_scan_pair_kernel", st);
            // one CTA per (32 state rows, head, sequence), the sequence's rank in `order` slowest
            const int64_t ctas = (int64_t)(DV / 32) * H * N;
            if (ctas > INT32_MAX) return GDN_ERR_INVALID_ARG;
            if (launch_dependent(kb, dim3((unsigned)ctas), dim3(scan_pair_threads(NQ)), SP::kBytes, st, tq, tk,
                                 tv, (const int*)meta, (const int*)order, (const int*)chunk_off, (const int4*)chunk_tab,
                                 reinterpret_cast<const uint8_t*>(op), state_in, static_cast<__nv_bfloat16*>(out),
                                 state_out, cuts.snaps, H, status) != cudaSuccess)
                return GDN_ERR_LAUNCH;
        }
        return GDN_OK;
    }
    if constexpr (!kBf16) {
        // state rows per CTA and CTAs per SM of the scan (compile-time tuning knobs)
        constexpr int MS = GDN_SCAN_MS;
        using S1 = ScanSmem<T, DK, MS, 1>;
        using S2 = ScanSmem<T, DK, MS, 2>;
        constexpr int MINB = ((S1::kBytes + 1024) * GDN_SCAN_MINB <= 228 * 1024) ? GDN_SCAN_MINB : 1;
        constexpr int STAGES = ((S2::kBytes + 1024) * MINB <= 228 * 1024) ? 2 : 1;
        using SL = ScanSmem<T, DK, MS, STAGES>;
        static_assert((SL::kBytes + 1024) * MINB <= 228 * 1024, "scan kernel shared memory");
        auto k2 = gdn_scan_tc_kernel<T, DK, DV, MS, STAGES, MINB>;
        if (!set_dyn_smem(k2, SL::kBytes, "cudaFuncSetAttribute(max dynamic shared memory)"))
            return GDN_ERR_LAUNCH;
        {
            ProfScope prof("gdn_scan_tc_kernel", st);
            if (launch_dependent(k2, dim3((unsigned)N, H, DV / MS), dim3(256), SL::kBytes, st, tq, tk, tv, (const int*)meta,
                                 (const int*)chunk_off, (const int4*)chunk_tab, (const float*)op, state_in,
                                 static_cast<T*>(out), state_out, cuts.snaps, H, status) != cudaSuccess)
                return GDN_ERR_LAUNCH;
        }
    }
    return GDN_OK;
}

template <typename T>
static int dispatch_prefill(int dk, int dv, const PrefillLayout& lay, char* ws, const void* q, const void* k,
                            const void* v, const float* g, const float* beta, const int32_t* cu, int N,
                            int64_t T_total, int fixed_len, const float* state_in, void* out,
                            float* state_out, int H, const Cuts& cuts, cudaStream_t st)
{
#define GDN_PF(DK_, DV_)                                                                                   \
    if (dk == DK_ && dv == DV_)                                                                            \
        return launch_prefill<T, DK_, DV_>(lay, ws, q, k, v, g, beta, cu, N, T_total, fixed_len, state_in, \
                                           out, state_out, H, cuts, st);
    GDN_PF(128, 128)
    GDN_PF(128, 64)
    GDN_PF(64, 128)
    GDN_PF(64, 64)
#undef GDN_PF
    return GDN_ERR_UNSUPPORTED;
}

// ---- scratch for the allocation-free prefill entry point -----------------------------------------
// A fixed 64 MiB block of device memory per GPU, part of this library's module: it exists on every
// device that loads the library, from module load until the process exits.  Host code must not use
// the symbol itself as an address; noalloc_scratch_ptr() asks the runtime for the device address.
constexpr size_t kNoallocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once per device.
static void* noalloc_scratch_ptr()
{
    static std::mutex mu;
    static void* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        cache[dev] = p;
    }
    return cache[dev];
}

// dtype argument: GDN_F32 or GDN_BF16, optionally with the GDN_QK_L2NORM flag
static bool split_dtype(int code, int& dtype, bool& norm)
{
    if (code & ~(0xff | GDN_QK_L2NORM)) return false;
    dtype = code & 0xff;
    norm = (code & GDN_QK_L2NORM) != 0;
    return dtype == GDN_F32 || dtype == GDN_BF16;
}

// bytes of the normalised q and k copies that the prefill's pre-pass writes after the layout
static size_t norm_bytes(int64_t T, int H, int dk, int dtype)
{
    return PrefillLayout::align((size_t)T * H * dk * (dtype == GDN_F32 ? 4 : 2)) * 2;
}

template <typename T>
static int launch_l2norm(const void* q, const void* k, void* qn, void* kn, int64_t nvec, int dk, cudaStream_t st)
{
    ProfScope prof("gdn_l2norm_kernel", st);
    const int64_t vpw = (dk == 128 ? 1 : 2) * kNormU;          // vectors per warp
    const int64_t warps = (nvec + vpw - 1) / vpw;
    const unsigned grid = (unsigned)((warps + 7) / 8);
    if (dk == 128)
        gdn_l2norm_kernel<T, 128><<<grid, 256, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                                        static_cast<T*>(qn), static_cast<T*>(kn), nvec);
    else
        gdn_l2norm_kernel<T, 64><<<grid, 256, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                                       static_cast<T*>(qn), static_cast<T*>(kn), nvec);
    return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_LAUNCH;
}

static int chunk_prefill(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, const float* state_in,
                         void* out, float* state_out, int H, int dk, int dv, int dtype, const Cuts& cuts,
                         void* workspace, size_t workspace_bytes, void* stream)
{
    if (num_seqs < 1 || H < 1 || total_tokens < 0 || total_tokens > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (cuts.n < 0 || (cuts.n > 0 && (!cuts.pos || !cuts.snaps))) return GDN_ERR_INVALID_ARG;
    if ((int64_t)num_seqs + cuts.n > INT32_MAX / 8) return GDN_ERR_INVALID_ARG;
    bool norm = false;
    if (!split_dtype(dtype, dtype, norm)) return GDN_ERR_INVALID_ARG;
    if (!head_ok(dk) || !head_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (total_tokens > 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_INVALID_ARG;
    int fixed_len = 0;
    if (!cu_seqlens) {
        if (total_tokens % num_seqs != 0) return GDN_ERR_INVALID_ARG;
        fixed_len = (int)(total_tokens / num_seqs);
    }
    const void* ptrs[] = {q, k, v, state_in, out, state_out, cuts.snaps};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    const void* small[] = {g, beta, cu_seqlens, cuts.pos};
    for (const void* p : small)
        if (p && !aligned4(p)) return GDN_ERR_MISALIGNED;
    PrefillLayout lay(total_tokens, num_seqs + cuts.n, H, dk);
    const size_t need = lay.total + (norm ? norm_bytes(total_tokens, H, dk, dtype) : 0);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return GDN_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    if (norm && total_tokens > 0) {
        // raw q and k: normalised copies in the workspace replace them for the rest of the call
        char* qn = ws + lay.total;
        char* kn = qn + norm_bytes(total_tokens, H, dk, dtype) / 2;
        const int rc = dtype == GDN_F32 ? launch_l2norm<float>(q, k, qn, kn, total_tokens * H, dk, st)
                                        : launch_l2norm<__nv_bfloat16>(q, k, qn, kn, total_tokens * H, dk, st);
        if (rc != GDN_OK) return rc;
        q = qn;
        k = kn;
    }
    if (dtype == GDN_F32)
        return dispatch_prefill<float>(dk, dv, lay, ws, q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens,
                                       fixed_len, state_in, out, state_out, H, cuts, st);
    return dispatch_prefill<__nv_bfloat16>(dk, dv, lay, ws, q, k, v, g, beta, cu_seqlens, num_seqs,
                                           total_tokens, fixed_len, state_in, out, state_out, H, cuts, st);
}

}  // namespace gdn

using namespace gdn;

extern "C" {

const char* gdn_status_string(int s)
{
    switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: invalid argument";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: dk and dv must be 64 or 128";
    case GDN_ERR_MISALIGNED: return "GDN_ERR_MISALIGNED: q/k/v/out/state need 16-byte, g/beta/cu_seqlens 4-byte alignment";
    case GDN_ERR_LAUNCH: return "GDN_ERR_LAUNCH: kernel launch failed";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case GDN_ERR_BAD_SEQLENS: return "GDN_ERR_BAD_SEQLENS: cu_seqlens is not 0..T_total non-decreasing";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a bounded wait inside a kernel expired";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a CUDA runtime call failed";
    case GDN_ERR_BAD_PARENTS: return "GDN_ERR_BAD_PARENTS: a draft-tree parent is not -1 or an earlier token";
    default: return "unknown gdn status";
    }
}

int gdn_version(void) { return 100; }

const char* gdn_last_error(void) { return g_last_err; }

size_t gdn_chunk_prefill_workspace_bytes(int64_t total_tokens, int num_seqs, int H, int dk, int dv)
{
    if (total_tokens < 0 || num_seqs < 1 || H < 1 || !head_ok(dk) || !head_ok(dv)) return 0;
    return PrefillLayout(total_tokens, num_seqs, H, dk).total;
}

size_t gdn_chunk_prefill_workspace_bytes_ex(int64_t total_tokens, int num_segments, int H, int dk, int dv, int dtype)
{
    bool norm = false;
    if (!split_dtype(dtype, dtype, norm)) return 0;
    const size_t base = gdn_chunk_prefill_workspace_bytes(total_tokens, num_segments, H, dk, dv);
    if (base == 0) return 0;
    return base + (norm ? norm_bytes(total_tokens, H, dk, dtype) : 0);
}

int gdn_chunk_prefill(const void* q, const void* k, const void* v, const float* g, const float* beta,
                      const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, const float* state_in,
                      void* out, float* state_out, int H, int dk, int dv, int dtype, void* workspace,
                      size_t workspace_bytes, void* stream)
{
    return chunk_prefill(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, state_in, out, state_out, H, dk, dv,
                         dtype, Cuts{}, workspace, workspace_bytes, stream);
}

int gdn_chunk_prefill_cuts(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, const int32_t* cuts,
                           int num_cuts, const float* state_in, void* out, float* state_out, float* snapshots,
                           int H, int dk, int dv, int dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    Cuts c;
    c.pos = cuts;
    c.n = num_cuts;
    c.snaps = snapshots;
    if (num_cuts < 1) return GDN_ERR_INVALID_ARG;
    return chunk_prefill(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, state_in, out, state_out, H, dk, dv,
                         dtype, c, workspace, workspace_bytes, stream);
}

int gdn_chunk_prefill_noalloc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                              const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens,
                              const float* state_in, void* out, float* state_out, int H, int dk, int dv,
                              int dtype, void* stream)
{
    // the scratch must hold the whole workspace of this call; refuse before touching the device
    const size_t need = gdn_chunk_prefill_workspace_bytes_ex(total_tokens, num_seqs, H, dk, dv, dtype);
    if (need > kNoallocScratchBytes) return GDN_ERR_WORKSPACE;
    void* scratch = noalloc_scratch_ptr();
    if (!scratch) return GDN_ERR_CUDA;
    // nothing in the scratch has to start at zero: the kernels write every part they read
    return gdn_chunk_prefill(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, state_in, out, state_out, H,
                             dk, dv, dtype, scratch, kNoallocScratchBytes, stream);
}

int gdn_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                    float* state_inout, void* out, int B, int H, int dk, int dv, int dtype, void* stream)
{
    if (B < 0 || H < 1) return GDN_ERR_INVALID_ARG;
    bool norm = false;
    if (!split_dtype(dtype, dtype, norm)) return GDN_ERR_INVALID_ARG;
    if (!head_ok(dk) || !head_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state_inout) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, state_inout, out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    if (!aligned4(g) || !aligned4(beta)) return GDN_ERR_MISALIGNED;
    if ((int64_t)B * H > INT32_MAX) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == GDN_F32) return dispatch_decode<float>(q, k, v, g, beta, state_inout, out, B, H, dk, dv, norm, st);
    return dispatch_decode<__nv_bfloat16>(q, k, v, g, beta, state_inout, out, B, H, dk, dv, norm, st);
}

// Checks and dispatch shared by the chain and tree verify (parents == nullptr: a chain).
static int verify_entry(const void* q, const void* k, const void* v, const float* g, const float* beta,
                        const int32_t* parents, const float* state_in, float* states_out, void* out, int B, int Tk,
                        int H, int dk, int dv, int dtype, void* stream)
{
    if (B < 0 || Tk < 1 || H < 1) return GDN_ERR_INVALID_ARG;
    bool norm = false;
    if (!split_dtype(dtype, dtype, norm)) return GDN_ERR_INVALID_ARG;
    if (!head_ok(dk) || !head_ok(dv)) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state_in) return GDN_ERR_INVALID_ARG;
    if (!states_out && !out) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, state_in, states_out, out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    if (!aligned4(g) || !aligned4(beta)) return GDN_ERR_MISALIGNED;
    if (parents && !aligned4(parents)) return GDN_ERR_MISALIGNED;
    if ((int64_t)B * H > INT32_MAX || (int64_t)B * Tk * H > INT32_MAX) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == GDN_F32)
        return dispatch_verify<float>(q, k, v, g, beta, state_in, states_out, out, parents, B, Tk, H, dk, dv, norm,
                                      st);
    return dispatch_verify<__nv_bfloat16>(q, k, v, g, beta, state_in, states_out, out, parents, B, Tk, H, dk, dv,
                                          norm, st);
}

int gdn_decode_verify(const void* q, const void* k, const void* v, const float* g, const float* beta,
                      const float* state_in, float* states_out, void* out, int B, int Tk, int H, int dk, int dv,
                      int dtype, void* stream)
{
    return verify_entry(q, k, v, g, beta, nullptr, state_in, states_out, out, B, Tk, H, dk, dv, dtype, stream);
}

int gdn_decode_verify_tree(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const int32_t* parents, const float* state_in, float* states_out, void* out, int B,
                           int Tk, int H, int dk, int dv, int dtype, void* stream)
{
    if (B > 0 && (!parents || !states_out)) return GDN_ERR_INVALID_ARG;
    return verify_entry(q, k, v, g, beta, parents, state_in, states_out, out, B, Tk, H, dk, dv, dtype, stream);
}

// Failure-path self-test: one thread waits on an mbarrier that nothing arrives on.  The bounded
// wait gives up after about limit_ns, the kernel records GDN_ERR_TIMEOUT in the status word and
// returns normally (the context stays usable), exactly as a timed-out wait in the prefill does.
__global__ void gdn_selftest_timeout_kernel(int* status, unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int never;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
        never = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, &never, limit_ns)) report(status, GDN_ERR_TIMEOUT);
}

int gdn_selftest_wait_timeout(long long limit_ns, void* stream)
{
    if (limit_ns < 1000000LL || limit_ns > 2000000000LL) return GDN_ERR_INVALID_ARG;
    int* status = status_ptr();
    if (!status) return GDN_ERR_CUDA;
    gdn_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status,
                                                                                 (unsigned long long)limit_ns);
    return cudaPeekAtLastError() == cudaSuccess ? GDN_OK : GDN_ERR_LAUNCH;
}

int gdn_get_device_status(void* stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDN_ERR_CUDA;
    int* p = status_ptr();
    if (!p) return GDN_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return GDN_ERR_CUDA;
    return v;
}

int gdn_profile_start(void)
{
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (g_prof_on) return GDN_ERR_INVALID_ARG;
    for (int i = 0; i < 256; ++i) {
        cudaEvent_t e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) return GDN_ERR_CUDA;
        g_prof_pool.push_back(e);
    }
    g_prof_recs.clear();
    g_prof_on = true;
    return GDN_OK;
}

int gdn_profile_stop(int max_kernels, char* names, double* total_ms, int* launches)
{
    std::vector<ProfRec> recs;
    {
        std::lock_guard<std::mutex> lock(g_prof_mu);
        if (!g_prof_on) return GDN_ERR_INVALID_ARG;
        g_prof_on = false;
        recs.swap(g_prof_recs);
    }
    std::vector<std::string> uniq;
    std::vector<double> tot;
    std::vector<int> cnt;
    int rc = GDN_OK;
    for (const ProfRec& r : recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            rc = GDN_ERR_CUDA;
        size_t i = 0;
        while (i < uniq.size() && uniq[i] != r.name) ++i;
        if (i == uniq.size()) { uniq.push_back(r.name); tot.push_back(0.0); cnt.push_back(0); }
        tot[i] += ms;
        cnt[i] += 1;
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    {
        std::lock_guard<std::mutex> lock(g_prof_mu);
        for (cudaEvent_t e : g_prof_pool) cudaEventDestroy(e);
        g_prof_pool.clear();
    }
    if (rc != GDN_OK) return rc;
    const int n = (int)uniq.size();
    for (int i = 0; i < n && i < max_kernels; ++i) {
        if (names) {
            snprintf(names + 64 * i, 64, "%s", uniq[i].c_str());
        }
        if (total_ms) total_ms[i] = tot[i];
        if (launches) launches[i] = cnt[i];
    }
    return n;
}

}  // extern "C"
