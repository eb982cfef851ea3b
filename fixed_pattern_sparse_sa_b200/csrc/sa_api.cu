// sa_api.cu -- C ABI entry points of libsa.so (declared in include/sa.h).
//
// Host code only validates, sizes workspace and launches; every step of the
// computation runs in the kernels of attn_gather.cuh, indexer.cuh and
// nsa_misc.cuh.  There is no CPU fallback.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/sa.h"
#include "attn_bwd.cuh"
#include "attn_gather.cuh"
#include "attn_tc.cuh"
#include "attn_cmp_tc.cuh"
#include "attn_tile.cuh"
#include "dist.cuh"
#include "full_score.cuh"
#include "indexer.cuh"
#include "indexer_filter.cuh"
#include "nsa_misc.cuh"
#include "nsa_bwd_tc.cuh"
#include "probe_gather.cuh"

using namespace sa;

// ------------------------------------------------------------- error state --
static thread_local std::string g_last_error;

static int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

// Kernels enqueued by this process (all devices), for launch accounting.
static std::atomic<unsigned long long> g_launches{0};

// SA_LOG=1 in the environment prints every kernel launch (name, grid, block,
// dynamic shared memory) to stderr.
static bool log_enabled() {
    static const bool on = [] {
        const char *e = std::getenv("SA_LOG");
        return e && *e && std::strcmp(e, "0") != 0;
    }();
    return on;
}
static void log_launch(const char *name, dim3 g, dim3 b, size_t smem) {
    if (log_enabled())
        std::fprintf(stderr, "[sa] %s grid=(%u,%u,%u) block=(%u,%u,%u) smem=%zu\n", name, g.x, g.y, g.z, b.x, b.y,
                     b.z, smem);
}

// Every kernel is launched with programmatic stream serialization allowed
// (the kernels begin with grid_dependency_sync), so a dependent kernel's
// blocks are scheduled while the previous grid's last blocks finish; in a
// CUDA graph this removes most of the gap between back-to-back launches.
// SA_PDL=0 launches plainly (for comparison).
static bool pdl_enabled() {
    static const bool on = [] {
        const char *e = std::getenv("SA_PDL");
        return !(e && std::strcmp(e, "0") == 0);
    }();
    return on;
}
template <typename... P, typename... A>
static void launch_k(const char *name, void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     A &&...args) {
    log_launch(name, grid, block, smem);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    (void)cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);   // errors are read by SA_CHECK_LAUNCH
}

// NVTX range around each C-ABI call (visible to profilers and tracers;
// a no-op when none is attached).
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
};
#define SA_TRACE(name) TraceRange sa_trace_range_(name)

#define SA_CHECK_LAUNCH(what)                                                              \
    do {                                                                                   \
        cudaError_t e_ = cudaGetLastError();                                               \
        if (e_ != cudaSuccess) return fail(SA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_)); \
        g_launches.fetch_add(1, std::memory_order_relaxed);                                \
    } while (0)

// Device error word: one per device, set with atomicOr by kernels that find a
// bad index; read and cleared by sa_check_device_status().
__device__ unsigned g_sa_device_error;

static constexpr int kMaxDevices = 64;
static unsigned *g_err_ptr[kMaxDevices];
static std::mutex g_err_mu;

static int device_error_word(unsigned **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(SA_ERR_UNSUPPORTED, "device id %d", dev);
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_sa_device_error);
        if (e != cudaSuccess)
            return fail(SA_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        g_err_ptr[dev] = static_cast<unsigned *>(p);
    }
    *out = g_err_ptr[dev];
    return SA_OK;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
static cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }
static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

template <typename K>
static int set_smem(K kernel, int bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return SA_OK;
}

static int sm_count() {
    static int cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// ------------------------------------------------------------ tensor maps --
typedef CUresult (*TensorMapEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                      const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                      CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);

// The CUDA driver API's tensor-map encoder, looked up once through the runtime (no
// link-time dependency on libcuda).
static TensorMapEncodeFn tensor_map_encoder() {
    static TensorMapEncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncodeFn>(f);
    });
    return fn;
}

// 2-D bf16 map over `rows` rows of `cols` contiguous elements; box = 64
// columns (128 bytes) x box_rows rows, 128-byte swizzle.
static int bf16_tensor_map(CUtensorMap *m, const void *base, long long rows, int cols, int box_rows) {
    TensorMapEncodeFn enc = tensor_map_encoder();
    if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1u, 1u};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SA_OK;
}


// 3-D bf16 map over [rows, hkv, d] (d contiguous); box = 64 columns (128
// bytes) x 1 head x box_rows rows, 128-byte swizzle.
static int bf16_tensor_map_3d(CUtensorMap *m, const void *base, int d, int hkv, long long rows, int box_rows) {
    TensorMapEncodeFn enc = tensor_map_encoder();
    if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)hkv, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)hkv * d * 2};
    cuuint32_t box[3] = {64u, 1u, (cuuint32_t)box_rows};
    cuuint32_t es[3] = {1u, 1u, 1u};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled(3d) failed (%d)", (int)r);
    return SA_OK;
}

// SA_GATHER_TMA=1 loads the NSA selected branch's 16-row block chunks by TMA
// box loads (for comparison); by default they take the per-row cp.async
// copies of the explicit-list path, measured faster (64K NSA step 30.9 vs
// 33.9 ms) since those copies issue whole 128-byte lines from per-lane
// addresses with immediate offsets.
static bool gather_tma_allowed() {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_GATHER_TMA");
        v = (e && std::strcmp(e, "1") == 0) ? 1 : 0;
    }
    return v != 0;
}

// SA_GATHER_SMALL=warp: small explicit-list launches keep one warp per item
// instead of the CTA-merged pieces (for comparison).
static bool gather_small_per_warp() {
    static const bool v = [] {
        const char *e = std::getenv("SA_GATHER_SMALL");
        return e && std::strcmp(e, "warp") == 0;
    }();
    return v;
}
#ifndef SA_ATTN_NW
#define SA_ATTN_NW 12
#endif
// SA_THRESHOLD=block: one CTA per row for the sampled threshold for every
// call (for comparison); by default one warp per row when there are rows
// for 8 warps per SM.
static bool threshold_per_warp() {
    static const bool v = [] {
        const char *e = std::getenv("SA_THRESHOLD");
        return !(e && std::strcmp(e, "block") == 0);
    }();
    return v;
}

// -------------------------------------------------------- gather launches --
// Launch shape: 12 warps per CTA streaming 16-key chunks through a 2-stage
// ring (8 warps when the lo-key tile is also staged); ~200 KB of shared
// memory, one CTA and 12 gathering warps per SM.  Small launches (fewer
// items than 12 per SM, e.g. decode with a few hundred split pieces) use
// 4-warp CTAs so that every SM gets work.
template <int D, int SRC, bool BIAS, bool KLO, int NW, int STAGES_ = 2, int NK_ = 16, bool TMAB = false,
          bool CTAM = false>
static int launch_gather_nw(const GatherParams &p, long long items, cudaStream_t st,
                            const CUtensorMap *km = nullptr, const CUtensorMap *vm = nullptr) {
    constexpr int NK = NK_;
    constexpr int STAGES = KLO ? 2 : STAGES_;
    constexpr int smem = gather_smem_bytes<D, STAGES, KLO, NK, NW, SRC == KS_PROWS, BIAS, TMAB>();
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = gather_attn_kernel<D, STAGES, SRC, BIAS, KLO, NK, NW, TMAB, CTAM>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    static const CUtensorMap unused{};                   // the row-gather modes take no tensor map
    const long long blocks = CTAM ? items : (items + NW - 1) / NW;
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)blocks, NW * 32, smem, st, p, km ? *km : unused, vm ? *vm : unused);
    SA_CHECK_LAUNCH("gather_attn_kernel");
    return SA_OK;
}

template <int D, int SRC, bool BIAS, bool KLO = false>
static int launch_gather_t(const GatherParams &p, cudaStream_t st) {
    const long long items = (long long)p.B * p.q_units * p.Hkv * p.n_hchunk * p.n_split;
    if (items == 0) return SA_OK;
    if constexpr (SRC == KS_IDX && D == 128 && !BIAS && !KLO) {
        // ring depth / warps per CTA of the explicit-list kernel: SA_ATTN_CFG
        // = "9x3" (9 warps, 3 stages), "6x4", "4x3w" (32-key chunks);
        // default 12 warps x 2 stages of 16 keys
        static int cfg = -1;
        if (cfg < 0) {
            const char *e = std::getenv("SA_ATTN_CFG");
            cfg = !e ? 0 : !std::strcmp(e, "9x3") ? 1 : !std::strcmp(e, "6x4") ? 2 : !std::strcmp(e, "4x3w") ? 3 : 0;
        }
        if (items >= (long long)sm_count() * SA_ATTN_NW) {
            if (cfg == 1) return launch_gather_nw<D, SRC, BIAS, KLO, 9, 3, 16>(p, items, st);
            if (cfg == 2) return launch_gather_nw<D, SRC, BIAS, KLO, 6, 4, 16>(p, items, st);
            if (cfg == 3) return launch_gather_nw<D, SRC, BIAS, KLO, 4, 3, 32>(p, items, st);
        }
    }
    if constexpr (SRC == KS_BLOCKS && D == 128 && !BIAS && !KLO) {
        // NSA selected blocks: 16-row chunks of a block by TMA box loads (opt-in,
        // SA_GATHER_TMA=1; by default the row gather below)
        if (p.block % 16 == 0 && (long long)p.B * p.Lk < INT_MAX && items >= (long long)sm_count() * SA_ATTN_NW &&
            gather_tma_allowed()) {
            CUtensorMap km, vm;
            int rc = bf16_tensor_map_3d(&km, p.k, 128, p.Hkv, (long long)p.B * p.Lk, 16);
            if (rc) return rc;
            rc = bf16_tensor_map_3d(&vm, p.v, 128, p.Hkv, (long long)p.B * p.Lk, 16);
            if (rc) return rc;
            return launch_gather_nw<D, SRC, BIAS, KLO, SA_ATTN_NW, 2, 16, true>(p, items, st, &km, &vm);
        }
    }
    if constexpr (KLO) {
        return launch_gather_nw<D, SRC, BIAS, KLO, 8>(p, items, st);
    } else {
        // small launches (decode pieces, fewer items than 12 per SM): with
        // explicit lists, one CTA of 8 warps per item, the warps splitting the
        // item's entries and merging in shared memory (8x the warps of one
        // warp per item, same partial rows); otherwise 4-warp CTAs.
        // SA_GATHER_SMALL=warp selects the 4-warp form for lists too (for
        // comparison).
        if (items < (long long)sm_count() * SA_ATTN_NW) {
            if constexpr (SRC == KS_IDX && !BIAS) {
                if (!gather_small_per_warp())
                    return launch_gather_nw<D, SRC, BIAS, KLO, 8, 2, 16, false, true>(p, items, st);
            }
            return launch_gather_nw<D, SRC, BIAS, KLO, 4>(p, items, st);
        }
        // fixed-graph rows (KS_PROWS): SA_PROWS_NW = 16 or 20 warps per CTA
        // (fewer registers each, more warps per SM; for comparison)
        if constexpr (SRC == KS_PROWS && D == 64) {
            static const int prows_nw = [] {
                const char *e = std::getenv("SA_PROWS_NW");
                return e ? std::atoi(e) : 12;
            }();
            if (prows_nw == 16) return launch_gather_nw<D, SRC, BIAS, KLO, 16>(p, items, st);
            if (prows_nw == 20) return launch_gather_nw<D, SRC, BIAS, KLO, 20>(p, items, st);
        }
        return launch_gather_nw<D, SRC, BIAS, KLO, SA_ATTN_NW>(p, items, st);
    }
}

template <int D>
static int launch_gather_d(const GatherParams &p, int src, bool bias, cudaStream_t st) {
    switch (src) {
        case KS_IDX: return bias ? launch_gather_t<D, KS_IDX, true>(p, st) : launch_gather_t<D, KS_IDX, false>(p, st);
        case KS_PATTERN:
            return bias ? launch_gather_t<D, KS_PATTERN, true>(p, st) : launch_gather_t<D, KS_PATTERN, false>(p, st);
        case KS_BLOCKS: return launch_gather_t<D, KS_BLOCKS, false>(p, st);
        case KS_RANGE: return launch_gather_t<D, KS_RANGE, false>(p, st);
        case KS_PROWS:
            return bias ? launch_gather_t<D, KS_PROWS, true>(p, st) : launch_gather_t<D, KS_PROWS, false>(p, st);
    }
    return fail(SA_ERR_UNSUPPORTED, "key source %d", src);
}

static int launch_gather(const GatherParams &p, int d, int src, bool bias, cudaStream_t st) {
    // the kernel forms a key row's offset as a 32-bit row stride (Hkv * d * 2 bytes) times the key
    if ((long long)p.Hkv * d * 2 >= (1LL << 32)) return fail(SA_ERR_UNSUPPORTED, "gather: Hkv * d too large");
    if (d == 64) return launch_gather_d<64>(p, src, bias, st);
    if (d == 128) return launch_gather_d<128>(p, src, bias, st);
    return fail(SA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
}

// ------------------------------------------- tensor-core gather launches --

// SA_ATTN_PATH=tc routes explicit-list attention (head dim 128, <= 16 heads
// per KV head, no bias) through attn_tc_kernel.  It is opt-in: with 64-KB
// K/V stages it keeps fewer gathered bytes in flight per SM than the
// per-warp mma.sync kernel and measured slower (5.4 vs 3.4 ms for the
// 32K-token prefill attention).
static bool attn_tc_allowed() {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_ATTN_PATH");
        v = (e && std::strcmp(e, "tc") == 0) ? 1 : 0;
    }
    return v != 0;
}

static bool attn_tc_applies(const GatherParams &p, int d, int src, bool bias) {
    const bool blocks_ok = src != KS_BLOCKS || (p.block == 32 || p.block == 64 || p.block == 128);
    return attn_tc_allowed() && (src == KS_IDX || src == KS_BLOCKS) && blocks_ok && !bias && d == 128 &&
           p.G <= 16 && !p.klo && (!p.out_f32 || p.n_split == 1) && (long long)p.B * p.Lk * p.Hkv < INT_MAX &&
           (long long)p.B * p.Tq * p.Hq + 16 < INT_MAX;
}

template <int SRC>
static int launch_attn_tc(const GatherParams &p, cudaStream_t st) {
    const long long items = (long long)p.B * p.Tq * p.Hkv * p.n_split;
    if (items == 0) return SA_OK;
    if (items > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "attn_tc: %lld work items", items);
    CUtensorMap qm;
    int rc = bf16_tensor_map(&qm, p.q, (long long)p.B * p.Tq * p.Hq, 128, 16);
    if (rc) return rc;
    // K and V maps for the TMA block loads (selected NSA blocks); unused
    // when rows are gathered one by one
    CUtensorMap km = qm, vm = qm;
    if (SRC == KS_BLOCKS) {
        rc = bf16_tensor_map_3d(&km, p.k, 128, p.Hkv, (long long)p.B * p.Lk, p.block);
        if (rc) return rc;
        rc = bf16_tensor_map_3d(&vm, p.v, 128, p.Hkv, (long long)p.B * p.Lk, p.block);
        if (rc) return rc;
    }
    AtcParams ap{};
    ap.g = p;
    ap.n_items = (int)items;
    constexpr int smem = AtcSmem<128>::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = attn_tc_kernel<128, SRC>;
    rc = set_smem(kern, smem);
    if (rc) return rc;
    const int grid = (int)std::min<long long>(items, sm_count());
    launch_k(__PRETTY_FUNCTION__, kern, grid, ATC_THREADS, smem, st, qm, km, vm, ap);
    SA_CHECK_LAUNCH("attn_tc_kernel");
    return SA_OK;
}

static int launch_combine(const float *po, const float *pl, int n_split, long long rows, int d,
                          void *out, float *lse, cudaStream_t st) {
    if (rows == 0) return SA_OK;
    const unsigned blocks = (unsigned)((rows + COMBINE_ROWS - 1) / COMBINE_ROWS);
    constexpr int threads = COMBINE_ROWS * 32;
    if (d == 64)
        launch_k("lse_combine_kernel<64>", lse_combine_kernel<64>, blocks, threads, 0, st, po, pl, n_split, rows,
            (__nv_bfloat16 *)out, lse);
    else if (d == 128)
        launch_k("lse_combine_kernel<128>", lse_combine_kernel<128>, blocks, threads, 0, st, po, pl, n_split, rows,
            (__nv_bfloat16 *)out, lse);
    else
        return fail(SA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    SA_CHECK_LAUNCH("lse_combine_kernel");
    return SA_OK;
}

// Public entry points: C linkage comes from the declarations in sa.h.

int sa_version(void) { return 100; }

uint64_t sa_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

const char *sa_last_error_string(void) { return g_last_error.c_str(); }

const char *sa_status_string(int s) {
    switch (s) {
        case SA_OK: return "SA_OK";
        case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
        case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
        case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
        case SA_ERR_CUDA: return "SA_ERR_CUDA";
        case SA_ERR_DEVICE_ASSERT: return "SA_ERR_DEVICE_ASSERT";
        case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
    }
    return "SA_ERR_UNKNOWN";
}

int sa_check_device_status(void *stream) {
    SA_TRACE("sa_check_device_status");
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
    unsigned word = 0;
    e = cudaMemcpy(&word, ew, sizeof word, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
    if (word) {
        const unsigned zero = 0;
        e = cudaMemcpy(ew, &zero, sizeof zero, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return fail(SA_ERR_CUDA, "clear error word: %s", cudaGetErrorString(e));
        // a timeout leaves outputs undefined, so it outranks a skipped index
        return fail((word & ERR_TIMEOUT) ? SA_ERR_TIMEOUT : SA_ERR_DEVICE_ASSERT, "device error word 0x%x:%s%s%s",
                    word,
                    (word & ERR_BAD_INDEX) ? " index out of range or after the query position;" : "",
                    (word & ERR_BAD_BLOCK) ? " NSA block id outside the sequence;" : "",
                    (word & ERR_TIMEOUT) ? " a bounded barrier wait ran out of its spin limit;" : "");
    }
    return SA_OK;
}

// ------------------------------------------------------- debug controls --
int sa_debug_set_spin_limit(long cycles) {
    const long long v = cycles > 0 ? (long long)cycles : kDefaultSpinCycles;
    cudaError_t e = cudaMemcpyToSymbol(g_sa_spin_cycles, &v, sizeof v);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "set spin limit: %s", cudaGetErrorString(e));
    return SA_OK;
}

int sa_debug_inject_stall(int on) {
    const int v = on ? 1 : 0;
    cudaError_t e = cudaMemcpyToSymbol(g_sa_debug_stall, &v, sizeof v);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "inject stall: %s", cudaGetErrorString(e));
    return SA_OK;
}

int64_t sa_debug_exact_recompute_rows(void) {
    unsigned long long n = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&n, g_sa_recompute_rows, sizeof n);
    if (e != cudaSuccess) return -(int64_t)fail(SA_ERR_CUDA, "read recompute counter: %s", cudaGetErrorString(e));
    const unsigned long long zero = 0;
    e = cudaMemcpyToSymbol(g_sa_recompute_rows, &zero, sizeof zero);
    if (e != cudaSuccess) return -(int64_t)fail(SA_ERR_CUDA, "clear recompute counter: %s", cudaGetErrorString(e));
    return (int64_t)n;
}

// ------------------------------------------------------ sparse attention --
// Split-KV workspace: partial rows, partial LSEs and one arrival ticket per
// (b, t, KV group, 16-head chunk) -- at most B * Tq * Hq of them.
size_t sa_sparse_attn_workspace_size(int B, int Tq, int Hq, int d, int n_split) {
    if (n_split <= 1 || B <= 0 || Tq <= 0 || Hq <= 0 || d <= 0) return 0;
    const size_t rows = (size_t)B * Tq * Hq;
    return round_up((size_t)n_split * rows * d * 4, 256) + round_up((size_t)n_split * rows * 4, 256) +
           round_up(rows * 4, 256);
}

int sa_sparse_attn_fwd(const void *q, const void *k, const void *v, int B, int Tq, int L, int Hq,
                       int Hkv, int d, int64_t q_pos0, const int32_t *idx, int idx_heads, int K,
                       const sa_pattern *pattern, const float *cq, const float *ck,
                       const float *beta, float scale, int n_split, void *out, float *lse,
                       float *part_o, float *part_lse, void *workspace, size_t workspace_bytes,
                       void *stream) {
    SA_TRACE("sa_sparse_attn_fwd");
    if (B <= 0 || Tq < 0 || L <= 0 || Hq <= 0 || Hkv <= 0 || n_split < 1)
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: bad sizes B=%d Tq=%d L=%d Hq=%d Hkv=%d n_split=%d",
                    B, Tq, L, Hq, Hkv, n_split);
    if (Hq % Hkv) return fail(SA_ERR_INVALID_ARG, "sparse_attn: Hq %% Hkv != 0");
    if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "sparse_attn: head dim %d", d);
    if (q_pos0 < 0 || q_pos0 + Tq > L)
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: query positions [%lld, %lld) outside [0, L=%d)",
                    (long long)q_pos0, (long long)q_pos0 + Tq, L);
    if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v))
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: q/k/v must be non-null and 16-byte aligned");
    if (!idx && !pattern) return fail(SA_ERR_INVALID_ARG, "sparse_attn: need idx or pattern");
    if (idx && (K < 0 || !(idx_heads == 1 || idx_heads == Hkv) || !aligned4(idx)))
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: idx_heads must be 1 or Hkv, K >= 0");
    if (!idx && (pattern->window < 1))
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: pattern window must be >= 1");
    const bool bias = cq || ck || beta;
    if (bias && !(cq && ck && beta))
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: cq, ck and beta go together");
    if (bias && (!aligned4(cq) || !aligned4(ck) || !aligned4(beta)))
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: coordinate pointers must be 4-byte aligned");
    if (n_split == 1 && !out) return fail(SA_ERR_INVALID_ARG, "sparse_attn: out is NULL");
    if (out && !aligned16(out)) return fail(SA_ERR_INVALID_ARG, "sparse_attn: out must be 16-byte aligned");
    if (!std::isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "sparse_attn: scale");
    if (Tq == 0) return SA_OK;

    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;

    const long long rows = (long long)B * Tq * Hq;
    float *po = part_o, *pl = part_lse;
    int *tickets = nullptr;
    if (n_split > 1 && (!po || !pl)) {
        const size_t need = sa_sparse_attn_workspace_size(B, Tq, Hq, d, n_split);
        if (!workspace || workspace_bytes < need)
            return fail(SA_ERR_WORKSPACE, "sparse_attn: workspace %zu < %zu", workspace_bytes, need);
        if (!aligned16(workspace)) return fail(SA_ERR_INVALID_ARG, "sparse_attn: workspace alignment");
        const size_t o_bytes = round_up((size_t)n_split * rows * d * 4, 256);
        po = static_cast<float *>(workspace);
        pl = reinterpret_cast<float *>(static_cast<char *>(workspace) + o_bytes);
        tickets = reinterpret_cast<int *>(static_cast<char *>(workspace) + o_bytes +
                                          round_up((size_t)n_split * rows * 4, 256));
    }
    if (n_split > 1 && (!aligned16(po) || !aligned4(pl)))
        return fail(SA_ERR_INVALID_ARG, "sparse_attn: partial buffers alignment");

    GatherParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.B = B; p.Tq = Tq; p.Lk = L; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
    p.q_pos0 = q_pos0;
    p.idx = idx; p.idx_heads = idx_heads; p.K = K;
    int src;
    if (idx) {
        src = KS_IDX;
        p.entries = K;
    } else {
        p.window = pattern->window;
        p.dilated = pattern->dilated ? 1 : 0;
        const int G = Hq / Hkv;
        if (G < 16 && 16 % G == 0) {
            // rows = 16/G consecutive queries x G heads over the union of their sets
            src = KS_PROWS;
            const int nqw = 16 / G;
            p.entries = pattern->window + nqw - 1 + (p.dilated ? 32 * nqw : 0);
            p.q_units = (Tq + nqw - 1) / nqw;
        } else {
            src = KS_PATTERN;
            p.entries = pattern->window + (p.dilated ? 32 : 0);
        }
    }
    p.n_split = n_split;
    p.per_split = n_split > 1 ? (p.entries + n_split - 1) / n_split : p.entries;
    p.n_hchunk = src == KS_PROWS ? 1 : (p.G + 15) / 16;
    if (src != KS_PROWS) p.q_units = Tq;
    p.cq = cq; p.ck = ck; p.beta = beta;
    p.scale_log2 = scale * kLog2e;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.part_o = po; p.part_lse = pl;
    p.err = ew;
    cudaStream_t st = as_stream(stream);
    const bool tc = attn_tc_applies(p, d, src, bias);
    // with a ticket array the gather kernel's last piece of each group does
    // the merge itself (no separate combine launch)
    // The pieces are merged by a separate combine launch, unless
    // SA_SPLIT_MERGE=fused: then the last piece of each group to arrive
    // merges them (its warp, or its whole CTA in the CTA-merged form).  One
    // launch fewer, but the ticket reset and the serial merge after the
    // last piece measured slower for the 32 x 128K decode (per F S S S step:
    // 0.211 vs 0.156 ms one warp per piece, 0.156 vs 0.142 ms CTA-merged).
    static int fused = -1;
    if (fused < 0) {
        const char *e = std::getenv("SA_SPLIT_MERGE");
        fused = (e && std::strcmp(e, "fused") == 0) ? 1 : 0;
    }
    if (fused && !tc && n_split > 1 && n_split <= 32 && out && tickets) {
        const size_t nt = (size_t)B * Tq * Hkv * p.n_hchunk;
        cudaError_t e = cudaMemsetAsync(tickets, 0, nt * 4, st);
        if (e != cudaSuccess) return fail(SA_ERR_CUDA, "sparse_attn tickets: %s", cudaGetErrorString(e));
        p.merge_cnt = tickets;
    }
    rc = tc ? launch_attn_tc<KS_IDX>(p, st) : launch_gather(p, d, src, bias, st);
    if (rc) return rc;
    if (n_split > 1 && out && !p.merge_cnt) return launch_combine(po, pl, n_split, rows, d, out, lse, st);
    return SA_OK;
}

// --------------------------------------- split-KV without any allocation --
// Some callers cannot allocate device memory when they call us: a serving
// runtime whose device memory is all handed out up front, plugin hosts that
// pass only input/output buffers, or paths where a cudaMalloc would
// synchronise the device.  For them
// the split-KV attention keeps its partial results in a fixed array that is
// part of the library image instead of a caller workspace.  The array is
// 8 MiB per GPU that loads the library and lives until the process exits.
static constexpr size_t kStaticSplitBytes = (size_t)8 << 20;
static __device__ __align__(256) unsigned char g_static_split[kStaticSplitBytes];
static unsigned char *g_static_split_ptr[kMaxDevices];
static std::mutex g_static_split_mu;

// Device address of this device's copy of the array.  Host code must not use
// the symbol itself as a device pointer: the address is looked up once per
// device, with that device current, on its first call.
static int static_split_scratch(unsigned char **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(SA_ERR_UNSUPPORTED, "device id %d", dev);
    std::lock_guard<std::mutex> lk(g_static_split_mu);
    if (!g_static_split_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_split);
        if (e != cudaSuccess)
            return fail(SA_ERR_CUDA, "cudaGetSymbolAddress(static split scratch): %s", cudaGetErrorString(e));
        g_static_split_ptr[dev] = static_cast<unsigned char *>(p);
    }
    *out = g_static_split_ptr[dev];
    return SA_OK;
}

int sa_sparse_attn_fwd_split_static(const void *q, const void *k, const void *v, int B, int Tq, int L,
                                    int Hq, int Hkv, int d, int64_t q_pos0, const int32_t *idx,
                                    int idx_heads, int K, float scale, int n_split, void *out,
                                    float *lse, void *stream) {
    SA_TRACE("sa_sparse_attn_fwd_split_static");
    if (n_split < 2) return fail(SA_ERR_INVALID_ARG, "split_static: n_split must be >= 2 (got %d)", n_split);
    if (!idx || !out) return fail(SA_ERR_INVALID_ARG, "split_static: idx and out are required");
    if (B <= 0 || Tq < 0 || Hq <= 0 || (d != 64 && d != 128))
        return fail(SA_ERR_INVALID_ARG, "split_static: bad sizes B=%d Tq=%d Hq=%d d=%d", B, Tq, Hq, d);
    // n_split * B * Tq * Hq * (d + 1) * 4 with every product checked: a
    // wrapped size must not pass the limit
    size_t rows = 0, parts = 0, o_elems = 0;
    if (__builtin_mul_overflow((size_t)B, (size_t)Tq, &rows) || __builtin_mul_overflow(rows, (size_t)Hq, &rows) ||
        __builtin_mul_overflow(rows, (size_t)n_split, &parts) || __builtin_mul_overflow(parts, (size_t)d, &o_elems) ||
        o_elems > kStaticSplitBytes / 4 || parts > kStaticSplitBytes / 4)
        return fail(SA_ERR_WORKSPACE,
                    "split_static: n_split * B * Tq * Hq * (d + 1) * 4 exceeds the built-in %zu-byte scratch; "
                    "use sa_sparse_attn_fwd with a workspace", kStaticSplitBytes);
    const size_t o_bytes = round_up(o_elems * 4, 256);
    const size_t need = o_bytes + round_up(parts * 4, 256);
    if (need > kStaticSplitBytes)
        return fail(SA_ERR_WORKSPACE,
                    "split_static: partials need %zu bytes but the built-in scratch holds %zu "
                    "(n_split * B * Tq * Hq * (d + 1) * 4 must fit); use sa_sparse_attn_fwd with a workspace",
                    need, kStaticSplitBytes);
    if (Tq == 0) return SA_OK;
    unsigned char *scratch = nullptr;
    int rc = static_split_scratch(&scratch);
    if (rc) return rc;
    float *po = reinterpret_cast<float *>(scratch);
    float *pl = reinterpret_cast<float *>(scratch + o_bytes);
    return sa_sparse_attn_fwd(q, k, v, B, Tq, L, Hq, Hkv, d, q_pos0, idx, idx_heads, K, nullptr, nullptr,
                              nullptr, nullptr, scale, n_split, out, lse, po, pl, nullptr, 0, stream);
}

int sa_lse_combine(const float *part_o, const float *part_lse, int n_split, int64_t rows, int d,
                   void *out, float *lse, void *stream) {
    SA_TRACE("sa_lse_combine");
    if (n_split < 1 || rows < 0) return fail(SA_ERR_INVALID_ARG, "lse_combine: n_split=%d rows=%lld", n_split, (long long)rows);
    if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "lse_combine: head dim %d", d);
    if (!part_o || !part_lse || !out || !aligned16(part_o) || !aligned4(part_lse) || !aligned16(out))
        return fail(SA_ERR_INVALID_ARG, "lse_combine: null or misaligned pointer");
    if (lse && !aligned4(lse)) return fail(SA_ERR_INVALID_ARG, "lse_combine: lse alignment");
    return launch_combine(part_o, part_lse, n_split, rows, d, out, lse, as_stream(stream));
}

// ------------------------------------------------------------- indexer --
// Rows per chunk: sample scores, thresholds and candidate lists of a chunk
// take about kIdxChunkBudget bytes of workspace.
static constexpr size_t kIdxChunkBudget = (size_t)1 << 30;

static bool indexer_shape_ok(int Hi, int di) {
    return (Hi == 1 || Hi == 2 || Hi == 4 || Hi == 8 || Hi == 16) && (di == 32 || di == 64 || di == 128);
}

// Decode-like shapes (a query or two per sequence) score on CUDA cores
// (memory-bound matrix-vector products); the rest on tcgen05 with 256-column
// tiles.  The sample stride is shared by a block of nq queries.
static bool indexer_decode_path(int Tq, int Hi) { return Tq * Hi <= 16; }

static int indexer_m_cap(int nq_block) { return (int)round_up((size_t)(2 * SAMPLE_TARGET + nq_block), 4); }

// Candidate list capacity per row.  With sample stride s the threshold sits
// at sample rank r = e + z*sqrt(r) (e = k/s, as in idx_threshold_kernel), so
// about s*r candidates reach it, with a standard deviation of about s*sqrt(r);
// the list holds s*r + z standard deviations.
static int indexer_cand_cap(int topk, int L) {
    const double s = std::max(1.0, std::floor((double)L / SAMPLE_TARGET));
    const double e = topk / s;
    double r = e + SAMPLE_Z * std::sqrt(e) + 2.0;
    for (int it = 0; it < 3; ++it) r = e + SAMPLE_Z * std::sqrt(r) + 2.0;
    const double cap = std::max((double)topk, s * r + SAMPLE_Z * s * std::sqrt(r)) + 256.0;
    return (int)round_up((size_t)cap, 64);
}

static size_t indexer_row_bytes(int m_cap, int cap) { return (size_t)m_cap * 4 + 8 + (size_t)cap * 8; }

static int indexer_chunk_rows(int B, int Tq, int nq_block, int m_cap, int cap) {
    size_t rows = kIdxChunkBudget / ((size_t)B * indexer_row_bytes(m_cap, cap));
    if (rows < 1) rows = 1;
    if (rows >= (size_t)nq_block) rows = rows / nq_block * nq_block;
    if (rows > (size_t)Tq) rows = Tq;
    if (rows > 65535) rows = 65535;   // grid.y limit
    return (int)rows;
}

struct IdxLayout {
    bool decode, filter_tc;
    int nq, m_cap, cap, rt;
    size_t sample_off, tau_off, cnt_off, cand_off, qf_off, wf_off, total;
};

// The persistent filter kernel (indexer_filter.cuh) serves prefill-shaped
// calls with 2..16 indexer heads; SA_IDX_FILTER=tiles selects the earlier
// per-tile kernel instead (kept for comparison).
static bool filter_tc_allowed() {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_IDX_FILTER");
        v = (e && std::strcmp(e, "tiles") == 0) ? 0 : 1;
    }
    return v != 0;
}

static IdxLayout indexer_layout(int B, int Tq, int L, int Hi, int di, int topk) {
    IdxLayout l{};
    l.decode = indexer_decode_path(Tq, Hi);
    l.filter_tc = !l.decode && Hi >= 2 && filter_tc_allowed();
    l.nq = l.decode ? 1 : 256 / Hi;
    l.m_cap = indexer_m_cap(l.nq);
    l.cap = indexer_cand_cap(topk, L);
    l.rt = indexer_chunk_rows(B, Tq, l.nq, l.m_cap, l.cap);
    const size_t rows = (size_t)B * l.rt;
    size_t off = 0;
    l.sample_off = off; off += round_up(rows * l.m_cap * 4, 256);
    l.tau_off = off; off += round_up(rows * 4, 256);
    l.cnt_off = off; off += round_up(rows * 4, 256);
    l.cand_off = off; off += round_up(rows * l.cap * 8, 256);
    // weights folded into the query operand (persistent filter kernel only)
    l.qf_off = off; off += l.filter_tc ? round_up((size_t)B * Tq * Hi * di, 256) : 0;
    l.wf_off = off; off += l.filter_tc ? round_up((size_t)B * Tq * Hi * 4, 256) : 0;
    l.total = off;
    return l;
}

size_t sa_indexer_topk_workspace_size(int B, int Tq, int L, int Hi, int di, int topk, int window) {
    (void)window;
    if (B <= 0 || Tq <= 0 || L <= 0 || topk < 0 || !(Hi == 1 || Hi == 2 || Hi == 4 || Hi == 8 || Hi == 16)) return 0;
    if (!(di == 32 || di == 64 || di == 128)) return 0;
    return indexer_layout(B, Tq, L, Hi, di, topk).total;
}

template <int HI, int DI, int NCOL, int MODE>
static int launch_score_t(const IdxParams &p, long long n_keys_max, cudaStream_t st) {
    constexpr int NQ = NCOL / HI;
    constexpr int smem = tc_smem_bytes<HI, DI, NCOL, MODE>();
    auto kern = idx_score_tc_kernel<HI, DI, NCOL, MODE>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    dim3 grid((unsigned)((n_keys_max + TC_KT * 128 - 1) / (TC_KT * 128)), (unsigned)((p.Rt + NQ - 1) / NQ),
              (unsigned)p.B);
    launch_k(__PRETTY_FUNCTION__, kern, grid, tc_threads(NCOL), smem, st, p);
    SA_CHECK_LAUNCH("idx_score_tc_kernel");
    return SA_OK;
}

template <int DI, int MODE>
static int launch_dp4a_t(const IdxParams &p, long long n_keys_max, cudaStream_t st) {
    dim3 grid((unsigned)((n_keys_max + DEC_KEYS - 1) / DEC_KEYS), (unsigned)p.Rt, (unsigned)p.B);
    launch_k("idx_score_dp4a_kernel<DI, MODE>", idx_score_dp4a_kernel<DI, MODE>, grid, DEC_THREADS, 0, st, p);
    SA_CHECK_LAUNCH("idx_score_dp4a_kernel");
    return SA_OK;
}

template <int MODE>
static int launch_dec_mma_t(const IdxParams &p, long long n_keys_max, cudaStream_t st) {
    constexpr int kpc = dmma_keys(MODE);
    dim3 grid((unsigned)((n_keys_max + kpc - 1) / kpc), (unsigned)p.Rt, (unsigned)p.B);
    launch_k("idx_score_dec_mma_kernel<MODE>", idx_score_dec_mma_kernel<MODE>, grid, DMMA_THREADS, 0, st, p);
    SA_CHECK_LAUNCH("idx_score_dec_mma_kernel");
    return SA_OK;
}

template <int HI, int DI, int MODE>
static int launch_score_n(const IdxParams &p, bool decode, long long n_keys_max, cudaStream_t st) {
    if (decode) {
        if constexpr (HI == 8 && DI == 64) return launch_dec_mma_t<MODE>(p, n_keys_max, st);
        return launch_dp4a_t<DI, MODE>(p, n_keys_max, st);
    }
    return launch_score_t<HI, DI, 256, MODE>(p, n_keys_max, st);
}

template <int MODE>
static int launch_score(const IdxParams &p, bool decode, long long n_keys_max, cudaStream_t st) {
#define SA_SCORE_DI(HI)                                                                 \
    if (p.di == 32) return launch_score_n<HI, 32, MODE>(p, decode, n_keys_max, st);    \
    if (p.di == 64) return launch_score_n<HI, 64, MODE>(p, decode, n_keys_max, st);    \
    return launch_score_n<HI, 128, MODE>(p, decode, n_keys_max, st);
    switch (p.Hi) {
        case 1: { SA_SCORE_DI(1) }
        case 2: { SA_SCORE_DI(2) }
        case 4: { SA_SCORE_DI(4) }
        case 8: { SA_SCORE_DI(8) }
        case 16: { SA_SCORE_DI(16) }
    }
#undef SA_SCORE_DI
    return fail(SA_ERR_UNSUPPORTED, "indexer heads %d", p.Hi);
}

// int8 2-D tensor map over `rows` rows of `di` bytes; box = one whole row
// (di bytes, swizzled with the matching 32B/64B/128B pattern) x box_rows rows.
static int i8_tensor_map(CUtensorMap *m, const void *base, long long rows, int di, int box_rows) {
    TensorMapEncodeFn enc = tensor_map_encoder();
    if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {(cuuint64_t)di, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)di};
    cuuint32_t box[2] = {(cuuint32_t)di, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1u, 1u};
    const CUtensorMapSwizzle sw = di == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : di == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled(int8) failed (%d)", (int)r);
    return SA_OK;
}

template <int HI, int DI>
static int launch_filter_tc_t(const IdxParams &p, const int8_t *qf, const int32_t *wf, cudaStream_t st) {
    constexpr int NQ = FT_NCOL / HI;
    const long long n_units = (long long)p.B * ((p.Rt + NQ - 1) / NQ);
    if (n_units == 0) return SA_OK;
    CUtensorMap am, bm;
    int rc = i8_tensor_map(&am, p.k, (long long)p.B * p.L, DI, 128);
    if (rc) return rc;
    rc = i8_tensor_map(&bm, qf, (long long)p.B * p.Tq * HI, DI, FT_NCOL);
    if (rc) return rc;
    FtParams fp{p, wf, (int)n_units};
    constexpr int smem = FtSmem<DI>::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = idx_filter_tc_kernel<HI, DI>;
    rc = set_smem(kern, smem);
    if (rc) return rc;
    const int grid = (int)std::min<long long>(n_units, sm_count());
    launch_k(__PRETTY_FUNCTION__, kern, grid, FT_THREADS, smem, st, am, bm, fp);
    SA_CHECK_LAUNCH("idx_filter_tc_kernel");
    return SA_OK;
}

template <int DI>
static int launch_filter_tc_d(const IdxParams &p, const int8_t *qf, const int32_t *wf, cudaStream_t st) {
    switch (p.Hi) {
        case 2: return launch_filter_tc_t<2, DI>(p, qf, wf, st);
        case 4: return launch_filter_tc_t<4, DI>(p, qf, wf, st);
        case 8: return launch_filter_tc_t<8, DI>(p, qf, wf, st);
        case 16: return launch_filter_tc_t<16, DI>(p, qf, wf, st);
    }
    return fail(SA_ERR_UNSUPPORTED, "filter: indexer heads %d", p.Hi);
}

static int launch_fold(const IdxParams &p, int8_t *qf, int32_t *wf, cudaStream_t st) {
    const long long n = (long long)p.B * p.Tq * p.Hi;
    const unsigned blocks = (unsigned)((n + 255) / 256);
    if (p.di == 32) launch_k("idx_fold_kernel<32>", idx_fold_kernel<32>, blocks, 256, 0, st, p.q, p.w, qf, wf, n);
    else if (p.di == 64) launch_k("idx_fold_kernel<64>", idx_fold_kernel<64>, blocks, 256, 0, st, p.q, p.w, qf, wf, n);
    else launch_k("idx_fold_kernel<128>", idx_fold_kernel<128>, blocks, 256, 0, st, p.q, p.w, qf, wf, n);
    SA_CHECK_LAUNCH("idx_fold_kernel");
    return SA_OK;
}

// One CTA per row; when there are few rows (decode) a row gets 1024 threads.
template <int DI, int NT>
static int launch_select_nt(const IdxParams &p, int words, cudaStream_t st) {
    const int smem = select_smem_staged<DI>(words, p.cand_cap);
    auto kern = topk_select_kernel<DI, NT>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    launch_k(__PRETTY_FUNCTION__, kern, dim3(1u, (unsigned)p.Rt, (unsigned)p.B), NT, smem, st, p);
    SA_CHECK_LAUNCH("topk_select_kernel");
    return SA_OK;
}

template <int DI>
static int launch_select_t(const IdxParams &p, int words, cudaStream_t st) {
    // few rows (decode): 1024-thread CTAs (measured faster than 512 or 256
    // threads for 32 rows of 131072 candidates)
    if ((long long)p.B * p.Rt <= sm_count()) return launch_select_nt<DI, 1024>(p, words, st);
    return launch_select_nt<DI, SEL_THREADS>(p, words, st);
}

int sa_indexer_topk(const int8_t *q_idx, const int8_t *k_idx, const int32_t *w, int B, int Tq, int L,
                    int Hi, int di, int64_t q_pos0, int topk, int window, int32_t *out_idx,
                    int32_t *out_count, void *workspace, size_t workspace_bytes, void *stream) {
    SA_TRACE("sa_indexer_topk");
    if (B <= 0 || Tq < 0 || L <= 0 || topk < 0 || window < 0 || topk + window < 1)
        return fail(SA_ERR_INVALID_ARG, "indexer_topk: bad sizes B=%d Tq=%d L=%d topk=%d window=%d", B, Tq,
                    L, topk, window);
    if (!indexer_shape_ok(Hi, di))
        return fail(SA_ERR_UNSUPPORTED, "indexer_topk: Hi=%d di=%d (Hi in 1,2,4,8,16; di in 32,64,128)", Hi, di);
    if (q_pos0 < 0 || q_pos0 + Tq > L)
        return fail(SA_ERR_INVALID_ARG, "indexer_topk: query positions [%lld, %lld) outside [0, L=%d)",
                    (long long)q_pos0, (long long)q_pos0 + Tq, L);
    if (!q_idx || !k_idx || !w || !out_idx || !aligned16(q_idx) || !aligned16(k_idx) || !aligned4(w) ||
        !aligned4(out_idx) || (out_count && !aligned4(out_count)))
        return fail(SA_ERR_INVALID_ARG, "indexer_topk: null or misaligned pointer");
    if (Tq == 0) return SA_OK;
    const long long n_max_all = std::max(0LL, (long long)(window > 0 ? q_pos0 + Tq - window : q_pos0 + Tq));
    if (n_max_all > SEL_MAX_N)
        return fail(SA_ERR_UNSUPPORTED, "indexer_topk: %lld candidates per query exceed %d", n_max_all, SEL_MAX_N);
    const IdxLayout lay = indexer_layout(B, Tq, L, Hi, di, topk);
    if (!workspace || workspace_bytes < lay.total)
        return fail(SA_ERR_WORKSPACE, "indexer_topk: workspace %zu < %zu", workspace_bytes, lay.total);
    if (!aligned16(workspace)) return fail(SA_ERR_INVALID_ARG, "indexer_topk: workspace alignment");
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    cudaStream_t st = as_stream(stream);
    char *ws = static_cast<char *>(workspace);

    IdxParams p{};
    p.q = q_idx; p.k = k_idx; p.w = w;
    p.B = B; p.Tq = Tq; p.L = L; p.Hi = Hi; p.di = di;
    p.q_pos0 = q_pos0; p.window = window; p.topk = topk; p.Kout = topk + window;
    p.nq_block = lay.nq; p.m_cap = lay.m_cap; p.cand_cap = lay.cap;
    p.sample = reinterpret_cast<int32_t *>(ws + lay.sample_off);
    p.tau = reinterpret_cast<int32_t *>(ws + lay.tau_off);
    p.cand_cnt = reinterpret_cast<int32_t *>(ws + lay.cnt_off);
    p.cand = reinterpret_cast<int2 *>(ws + lay.cand_off);
    p.out_idx = out_idx; p.out_count = out_count; p.err = ew;
    int8_t *qf = reinterpret_cast<int8_t *>(ws + lay.qf_off);
    int32_t *wf = reinterpret_cast<int32_t *>(ws + lay.wf_off);
    const bool filter_tc = lay.filter_tc && (long long)B * L < INT_MAX && (long long)B * Tq * Hi < INT_MAX;
    if (filter_tc) {
        rc = launch_fold(p, qf, wf, st);
        if (rc) return rc;
    }
    for (int t0 = 0; t0 < Tq; t0 += lay.rt) {
        const int rows = std::min(lay.rt, Tq - t0);
        p.t0 = t0; p.Rt = rows;
        const long long pmax = q_pos0 + t0 + rows - 1;
        const long long ncand = std::max(0LL, window > 0 ? pmax - window + 1 : pmax + 1);
        // the threshold kernel zeroes each row's list length (no rows have
        // candidates when ncand == 0, and the select then reads none)
        if (ncand > 0) {
            rc = launch_score<MODE_SAMPLE>(p, lay.decode, (long long)lay.m_cap, st);
            if (rc) return rc;
            // one warp per row when the rows fill the SMs (prefill); one CTA
            // per row for a few rows (decode), where a row's latency decides
            if (threshold_per_warp() && (long long)B * rows >= (long long)sm_count() * THW_WARPS) {
                const unsigned blocks = (unsigned)(((long long)B * rows + THW_WARPS - 1) / THW_WARPS);
                launch_k("idx_threshold_warp_kernel", idx_threshold_warp_kernel, blocks, THW_WARPS * 32, 0, st, p);
            } else {
                launch_k("idx_threshold_kernel", idx_threshold_kernel, dim3(1u, (unsigned)rows, (unsigned)B),
                         SEL_THREADS, 0, st, p);
            }
            SA_CHECK_LAUNCH("idx_threshold_kernel");
            if (filter_tc)
                rc = di == 32 ? launch_filter_tc_d<32>(p, qf, wf, st)
                              : di == 64 ? launch_filter_tc_d<64>(p, qf, wf, st) : launch_filter_tc_d<128>(p, qf, wf, st);
            else
                rc = launch_score<MODE_FILTER>(p, lay.decode, ncand, st);
            if (rc) return rc;
        }
        const int words = (int)((std::max(ncand, 1LL) + 31) / 32);
        rc = di == 32 ? launch_select_t<32>(p, words, st)
                      : di == 64 ? launch_select_t<64>(p, words, st) : launch_select_t<128>(p, words, st);
        if (rc) return rc;
    }
    return SA_OK;
}

// ----------------------------------------------------------------- NSA --
struct NsaLayout {
    int nc, n_blocks;
    size_t kc_off, klo_off, vc_off, o3_off, l3_off, sel_off, total;
};

static NsaLayout nsa_layout(int B, int T, int Hq, int Hkv, int d, int cmp_len, int cmp_stride,
                            int sel_block, int sel_topk) {
    NsaLayout lay{};
    lay.nc = T >= cmp_len ? (T - cmp_len) / cmp_stride + 1 : 0;
    lay.n_blocks = (T + sel_block - 1) / sel_block;
    const size_t rows = (size_t)B * T * Hq;
    size_t off = 0;
    lay.kc_off = off; off += round_up((size_t)B * std::max(lay.nc, 1) * Hkv * d * 2, 256);
    lay.klo_off = off; off += round_up((size_t)B * std::max(lay.nc, 1) * Hkv * d * 2, 256);
    lay.vc_off = off; off += round_up((size_t)B * std::max(lay.nc, 1) * Hkv * d * 2, 256);
    lay.o3_off = off; off += round_up(3 * rows * d * 4, 256);
    lay.l3_off = off; off += round_up(3 * rows * 4, 256);
    lay.sel_off = off; off += round_up((size_t)B * T * Hkv * sel_topk * 4, 256);
    lay.total = off;
    return lay;
}

size_t sa_nsa_workspace_size(int B, int T, int Hq, int Hkv, int d, int cmp_len, int cmp_stride,
                             int sel_block, int sel_topk) {
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || cmp_len <= 0 || cmp_stride <= 0 ||
        sel_block <= 0 || sel_topk <= 0)
        return 0;
    return nsa_layout(B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk).total;
}

template <int D>
static int launch_nsa_select(const NsaSelectParams &p, cudaStream_t st) {
    const int smem = nsa_select_smem<D>(p.n_blocks);
    if (smem > 227 * 1024) return fail(SA_ERR_UNSUPPORTED, "nsa: %d selection blocks exceed shared memory", p.n_blocks);
    auto kern = nsa_select_kernel<D>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    const long long ctas = (long long)p.B * p.Hkv * ((p.T + NSA_TW - 1) / NSA_TW);
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)ctas, NSA_TW * 32, smem, st, p);
    SA_CHECK_LAUNCH("nsa_select_kernel");
    return SA_OK;
}

// Compressed and window branches: 8 consecutive queries of a KV group per CTA
// share each staged key chunk.
constexpr int kTileWarps = 8;
template <int D, int SRC>
static int launch_tile_t(const TileParams &p, cudaStream_t st) {
    constexpr int STAGES = 3;
    constexpr int smem = tile_smem_bytes<D, STAGES, SRC>();
    auto kern = tile_attn_kernel<D, STAGES, SRC, kTileWarps>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    const long long ctas = (long long)p.B * p.Hkv * ((p.T + kTileWarps - 1) / kTileWarps);
    if (ctas == 0) return SA_OK;
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)ctas, kTileWarps * 32, smem, st, p);
    SA_CHECK_LAUNCH("tile_attn_kernel");
    return SA_OK;
}


template <int SRC>
static int launch_nsa_tc(const TileParams &p, unsigned *err, cudaStream_t st) {
    const long long items = (long long)p.B * p.Hkv * ((p.T + CT_Q - 1) / CT_Q);
    if (items == 0) return SA_OK;
    if (items > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "nsa_tc: %lld items", items);
    CUtensorMap qm, khm, klm, vm;
    int rc = bf16_tensor_map(&qm, p.q, (long long)p.B * p.T * p.Hq, 128, 16);
    if (rc) return rc;
    rc = bf16_tensor_map_3d(&khm, p.k, 128, p.Hkv, (long long)p.B * p.Lk, NT_KT);
    if (rc) return rc;
    rc = bf16_tensor_map_3d(&klm, SRC == TS_CMP ? p.klo : p.k, 128, p.Hkv, (long long)p.B * p.Lk, NT_KT);
    if (rc) return rc;
    rc = bf16_tensor_map_3d(&vm, p.v, 128, p.Hkv, (long long)p.B * p.Lk, NT_KT);
    if (rc) return rc;
    CmpTcParams cp{p, err, (int)items};
    constexpr int smem = CtSmem::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = nsa_tc_kernel<SRC>;
    rc = set_smem(kern, smem);
    if (rc) return rc;
    const int grid = (int)std::min<long long>(items, sm_count());   // persistent: one CTA per SM
    launch_k(__PRETTY_FUNCTION__, kern, grid, NT_THREADS, smem, st, qm, khm, klm, vm, cp);
    SA_CHECK_LAUNCH("nsa_tc_kernel");
    return SA_OK;
}

static int launch_imp_tc(const NsaSelectParams &sp, unsigned *err, cudaStream_t st) {
    TileParams p{};
    p.q = sp.q; p.k = sp.kc; p.klo = sp.klo;
    p.B = sp.B; p.T = sp.T; p.Lk = std::max(sp.nc, 1); p.Hq = sp.Hq; p.Hkv = sp.Hkv; p.G = sp.G;
    p.cmp_len = sp.cmp_len; p.cmp_stride = sp.cmp_stride; p.scale_log2 = sp.scale_log2;
    const long long items = (long long)p.B * p.Hkv * ((p.T + CT_Q - 1) / CT_Q);
    if (items == 0) return SA_OK;
    if (items > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "imp_tc: %lld items", items);
    CUtensorMap qm, khm, klm;
    int rc = bf16_tensor_map(&qm, p.q, (long long)p.B * p.T * p.Hq, 128, 16);
    if (rc) return rc;
    rc = bf16_tensor_map_3d(&khm, p.k, 128, p.Hkv, (long long)p.B * p.Lk, IT_KT);
    if (rc) return rc;
    rc = bf16_tensor_map_3d(&klm, p.klo, 128, p.Hkv, (long long)p.B * p.Lk, IT_KT);
    if (rc) return rc;
    ImpTcParams ip{p, sp.lse_cmp, sp.sel_block, sp.sel_topk, sp.n_blocks, sp.sel_idx, err, (int)items};
    const int smem = ItSmem::alloc(sp.n_blocks);
    if (smem > 227 * 1024) return fail(SA_ERR_UNSUPPORTED, "imp_tc: %d blocks", sp.n_blocks);
    rc = set_smem(nsa_imp_tc_kernel, smem);
    if (rc) return rc;
    const int grid = (int)std::min<long long>(items, sm_count());
    launch_k("nsa_imp_tc_kernel", nsa_imp_tc_kernel, grid, IT_THREADS, smem, st, qm, khm, klm, ip);
    SA_CHECK_LAUNCH("nsa_imp_tc_kernel");
    return SA_OK;
}

static bool imp_tc_applies(const NsaSelectParams &sp, int d) {
    const int cpb = sp.sel_block / sp.cmp_stride;
    return d == 128 && sp.G <= 16 && sp.imp_out == nullptr && sp.n_blocks <= IT_MAX_BLOCKS &&
           (cpb == 4 || cpb == 8 || cpb == 16 || cpb == 32 || cpb == 64) && sp.sel_topk <= 32 &&
           (long long)sp.B * sp.T * sp.Hq + 16 < INT_MAX && (long long)sp.B * sp.nc < INT_MAX;
}

static bool cmp_tc_applies(const TileParams &p, int d) {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_NSA_CMP_PATH");
        v = (e && std::strcmp(e, "mma") == 0) ? 0 : 1;
    }
    return v && d == 128 && p.G <= 16 && (long long)p.B * p.T * p.Hq + 16 < INT_MAX &&
           (long long)p.B * p.Lk < INT_MAX;
}

static int launch_tile(const TileParams &p, int d, int src, cudaStream_t st) {
    if (d == 64) return src == TS_CMP ? launch_tile_t<64, TS_CMP>(p, st) : launch_tile_t<64, TS_WINDOW>(p, st);
    return src == TS_CMP ? launch_tile_t<128, TS_CMP>(p, st) : launch_tile_t<128, TS_WINDOW>(p, st);
}

static int nsa_fwd_impl(const void *q, const void *k, const void *v, const float *gates, int B, int T, int Hq,
                        int Hkv, int d, int cmp_len, int cmp_stride, int sel_block, int sel_topk, int window,
                        float scale, void *out, float *lse_branches, int32_t *sel_idx_out, float *o_branches,
                        void *workspace, size_t workspace_bytes, void *stream) {
    if (B <= 0 || T < 0 || Hq <= 0 || Hkv <= 0 || cmp_len <= 0 || cmp_stride <= 0 || sel_block <= 0 ||
        sel_topk <= 0 || window <= 0)
        return fail(SA_ERR_INVALID_ARG, "nsa: bad sizes");
    if (Hq % Hkv) return fail(SA_ERR_INVALID_ARG, "nsa: Hq %% Hkv != 0");
    if (Hq / Hkv > 16) return fail(SA_ERR_UNSUPPORTED, "nsa: more than 16 query heads per KV head");
    if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "nsa: head dim %d", d);
    if (sel_block % cmp_stride || sel_topk > 32)
        return fail(SA_ERR_UNSUPPORTED, "nsa: need cmp_stride | sel_block and sel_topk <= 32");
    if (!q || !k || !v || !gates || !out || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        !aligned4(gates) || !aligned16(out))
        return fail(SA_ERR_INVALID_ARG, "nsa: null or misaligned pointer");
    if (!std::isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "nsa: scale");
    if (T == 0) return SA_OK;
    const NsaLayout lay = nsa_layout(B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk);
    if (!workspace || workspace_bytes < lay.total)
        return fail(SA_ERR_WORKSPACE, "nsa: workspace %zu < %zu", workspace_bytes, lay.total);
    if (!aligned16(workspace)) return fail(SA_ERR_INVALID_ARG, "nsa: workspace alignment");
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    cudaStream_t st = as_stream(stream);
    char *ws = static_cast<char *>(workspace);
    __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(ws + lay.kc_off);
    __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(ws + lay.vc_off);
    __nv_bfloat16 *klo = reinterpret_cast<__nv_bfloat16 *>(ws + lay.klo_off);
    float *o3 = o_branches ? o_branches : reinterpret_cast<float *>(ws + lay.o3_off);
    float *l3 = reinterpret_cast<float *>(ws + lay.l3_off);
    int32_t *sel = sel_idx_out ? sel_idx_out : reinterpret_cast<int32_t *>(ws + lay.sel_off);
    const long long rows = (long long)B * T * Hq;
    const int G = Hq / Hkv;

    // 1. compression
    if (lay.nc > 0) {
        const long long n2 = (long long)B * lay.nc * Hkv * (d / 2);
        launch_k("nsa_compress_kernel", nsa_compress_kernel, (unsigned)((n2 + 255) / 256), 256, 0, st,
            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, B, T, Hkv, d, lay.nc, cmp_len, cmp_stride, kc, klo,
            vc);
        SA_CHECK_LAUNCH("nsa_compress_kernel");
    }
    GatherParams base{};
    base.q = static_cast<const __nv_bfloat16 *>(q);
    base.B = B; base.Tq = T; base.Hq = Hq; base.Hkv = Hkv; base.G = G;
    base.q_pos0 = 0; base.n_split = 1; base.n_hchunk = 1; base.q_units = T;
    base.scale_log2 = scale * kLog2e;
    base.err = ew;
    // 2. compressed branch -> o3[0], l3[0]
    TileParams tp{};
    tp.q = base.q; tp.B = B; tp.T = T; tp.Hq = Hq; tp.Hkv = Hkv; tp.G = G;
    tp.scale_log2 = base.scale_log2;
    {
        TileParams p = tp;
        p.k = kc; p.klo = klo; p.v = vc; p.Lk = std::max(lay.nc, 1);
        p.cmp_len = cmp_len; p.cmp_stride = cmp_stride;
        p.out_f32 = o3; p.lse = l3;
        // nc == 0: zero rows, lse = -inf
        rc = cmp_tc_applies(p, d) ? launch_nsa_tc<TS_CMP>(p, ew, st) : launch_tile(p, d, TS_CMP, st);
        if (rc) return rc;
    }
    // 3. importance + block top-k
    {
        NsaSelectParams sp{};
        sp.q = base.q; sp.kc = kc; sp.klo = klo; sp.lse_cmp = l3;
        sp.B = B; sp.T = T; sp.Hq = Hq; sp.Hkv = Hkv; sp.G = G; sp.nc = lay.nc;
        sp.cmp_len = cmp_len; sp.cmp_stride = cmp_stride; sp.sel_block = sel_block;
        sp.sel_topk = sel_topk; sp.n_blocks = lay.n_blocks;
        sp.scale_log2 = base.scale_log2;
        sp.sel_idx = sel; sp.imp_out = nullptr;
        if (cmp_tc_applies(tp, d) && imp_tc_applies(sp, d))
            rc = launch_imp_tc(sp, ew, st);
        else
            rc = d == 64 ? launch_nsa_select<64>(sp, st) : launch_nsa_select<128>(sp, st);
        if (rc) return rc;
    }
    // 4. selected branch -> o3[1], l3[1]
    {
        GatherParams p = base;
        p.k = static_cast<const __nv_bfloat16 *>(k); p.v = static_cast<const __nv_bfloat16 *>(v);
        p.Lk = T; p.idx = sel; p.K = sel_topk; p.block = sel_block;
        p.block_shift = (sel_block & (sel_block - 1)) == 0 ? __builtin_ctz((unsigned)sel_block) : -1;
        p.entries = sel_topk * sel_block; p.per_split = p.entries;
        p.out_f32 = o3 + rows * d; p.lse = l3 + rows;
        rc = attn_tc_applies(p, d, KS_BLOCKS, false) ? launch_attn_tc<KS_BLOCKS>(p, st)
                                                     : launch_gather(p, d, KS_BLOCKS, false, st);
        if (rc) return rc;
    }
    // 5. window branch -> o3[2], l3[2]
    {
        TileParams p = tp;
        p.k = static_cast<const __nv_bfloat16 *>(k); p.v = static_cast<const __nv_bfloat16 *>(v);
        p.Lk = T; p.window = window;
        p.out_f32 = o3 + 2 * rows * d; p.lse = l3 + 2 * rows;
        rc = cmp_tc_applies(p, d) ? launch_nsa_tc<TS_WINDOW>(p, ew, st) : launch_tile(p, d, TS_WINDOW, st);
        if (rc) return rc;
    }
    // 6. gated sum
    {
        const long long n2 = rows * (d / 2);
        launch_k("nsa_gate_kernel", nsa_gate_kernel, (unsigned)((n2 + 255) / 256), 256, 0, st, o3, rows * d, gates,
            rows, d, (__nv_bfloat16 *)out);
        SA_CHECK_LAUNCH("nsa_gate_kernel");
        if (lse_branches) {
            launch_k("nsa_lse_pack_kernel", nsa_lse_pack_kernel, (unsigned)((rows + 255) / 256), 256, 0, st, l3, rows,
                lse_branches);
            SA_CHECK_LAUNCH("nsa_lse_pack_kernel");
        }
    }
    return SA_OK;
}

int sa_nsa_fwd(const void *q, const void *k, const void *v, const float *gates, int B, int T, int Hq,
               int Hkv, int d, int cmp_len, int cmp_stride, int sel_block, int sel_topk, int window,
               float scale, void *out, float *lse_branches, int32_t *sel_idx_out, void *workspace,
               size_t workspace_bytes, void *stream) {
    SA_TRACE("sa_nsa_fwd");
    return nsa_fwd_impl(q, k, v, gates, B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk, window, scale,
                        out, lse_branches, sel_idx_out, nullptr, workspace, workspace_bytes, stream);
}

int sa_nsa_fwd_train(const void *q, const void *k, const void *v, const float *gates, int B, int T, int Hq,
                     int Hkv, int d, int cmp_len, int cmp_stride, int sel_block, int sel_topk, int window,
                     float scale, void *out, float *lse_branches, int32_t *sel_idx_out, float *o_branches,
                     void *workspace, size_t workspace_bytes, void *stream) {
    SA_TRACE("sa_nsa_fwd_train");
    if (!lse_branches || !sel_idx_out || !o_branches || !aligned4(lse_branches) || !aligned4(sel_idx_out) ||
        !aligned16(o_branches))
        return fail(SA_ERR_INVALID_ARG, "nsa_fwd_train: null or misaligned saved-tensor pointer");
    return nsa_fwd_impl(q, k, v, gates, B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk, window, scale,
                        out, lse_branches, sel_idx_out, o_branches, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------ NSA backward --
constexpr int KV_SEL_SPLIT = 256;     // queries per work item of the selected branch's key-major pass

struct NsaBwdLayout {
    int nc, nb;
    long long n_lists, n_entries, max_items;
    size_t kc_off, klo_off, vc_off, dkc_off, dvc_off, dt_off;
    size_t cnt_off, qoff_off, cur_off, items_off, nitems_off, qlist_off, scal_off, total;
};

static NsaBwdLayout nsa_bwd_layout(int B, int T, int Hq, int Hkv, int d, int cmp_len, int cmp_stride,
                                   int sel_block, int sel_topk) {
    NsaBwdLayout lay{};
    lay.nc = T >= cmp_len ? (T - cmp_len) / cmp_stride + 1 : 0;
    lay.nb = (T + sel_block - 1) / sel_block;
    lay.n_lists = (long long)B * Hkv * lay.nb;
    lay.n_entries = (long long)B * T * Hkv * sel_topk;
    lay.max_items = lay.n_lists + (lay.n_entries + KV_SEL_SPLIT - 1) / KV_SEL_SPLIT;
    const size_t crow = (size_t)B * std::max(lay.nc, 1) * Hkv * d;
    size_t off = 0;
    lay.kc_off = off; off += round_up(crow * 2, 256);
    lay.klo_off = off; off += round_up(crow * 2, 256);
    lay.vc_off = off; off += round_up(crow * 2, 256);
    lay.dkc_off = off; off += round_up(crow * 4, 256);
    lay.dvc_off = off; off += round_up(crow * 4, 256);
    lay.dt_off = off; off += round_up((size_t)3 * B * T * Hq * 4, 256);
    lay.cnt_off = off; off += round_up((size_t)lay.n_lists * 4, 256);
    lay.qoff_off = off; off += round_up((size_t)(lay.n_lists + 1) * 4, 256);
    lay.cur_off = off; off += round_up((size_t)lay.n_lists * 4, 256);
    lay.items_off = off; off += round_up((size_t)lay.max_items * 8, 256);
    lay.nitems_off = off; off += 256;
    lay.qlist_off = off; off += round_up((size_t)lay.n_entries * 4, 256);
    // packed lse / D / gate of one branch for the tensor-core key-major pass
    lay.scal_off = off; off += round_up((size_t)B * Hkv * T * 16 * 16, 256);
    lay.total = off;
    return lay;
}

size_t sa_nsa_bwd_workspace_size(int B, int T, int Hq, int Hkv, int d, int cmp_len, int cmp_stride,
                                 int sel_block, int sel_topk) {
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || cmp_len <= 0 || cmp_stride <= 0 ||
        sel_block <= 0 || sel_topk <= 0)
        return 0;
    return nsa_bwd_layout(B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk).total;
}

template <int D, int SRC, bool HILO, bool DKV = true>
static int launch_bwd_branch(const BwdParams &p, cudaStream_t st) {
    constexpr int NW = (HILO && D == 128) ? 6 : 8;    // shared memory: 3 arrays per stage with HILO
    constexpr int smem = attn_bwd_smem_bytes<D, NW, HILO>();
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = attn_bwd_kernel<D, NW, SRC, HILO, DKV>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    const long long items = (long long)p.B * p.Tq * p.Hkv * ((p.G + 15) / 16);
    if (items == 0) return SA_OK;
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)((items + NW - 1) / NW), NW * 32, smem, st, p);
    SA_CHECK_LAUNCH("attn_bwd_kernel");
    return SA_OK;
}

// dq of the selected branch, one warp per (query, KV group) (at most 16 heads
// per KV head and 32 blocks); SA_NSA_BWD_SEL=v1 selects the generic kernel.
template <int D>
static int launch_bwd_dq_blocks(const BwdParams &p, cudaStream_t st) {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_NSA_BWD_SEL");
        v = (e && std::strcmp(e, "v1") == 0) ? 0 : 1;
    }
    if (!v || p.G > 16 || p.K > 32) return launch_bwd_branch<D, BW_BLOCKS, false, false>(p, st);
    constexpr int smem = attn_bwd_dq_blocks_smem<D>();
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = attn_bwd_dq_blocks_kernel<D>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    const long long items = (long long)p.B * p.Tq * p.Hkv;
    if (items == 0) return SA_OK;
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)((items + DQB_WARPS - 1) / DQB_WARPS), DQB_WARPS * 32, smem, st, p);
    SA_CHECK_LAUNCH("attn_bwd_dq_blocks_kernel");
    return SA_OK;
}

// dq of a range branch with the key chunks shared by 8 consecutive queries.
template <int D, bool HILO>
static int launch_bwd_dq_tile(const BwdParams &p, cudaStream_t st) {
    constexpr int smem = attn_bwd_dq_tile_smem<D, HILO>();
    auto kern = attn_bwd_dq_tile_kernel<D, HILO>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    const long long ctas = (long long)p.B * p.Hkv * ((p.G + 15) / 16) * ((p.Tq + DQ_WARPS - 1) / DQ_WARPS);
    if (ctas == 0) return SA_OK;
    if (ctas > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "attn_bwd_dq: %lld CTAs", ctas);
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)ctas, DQ_WARPS * 32, smem, st, p);
    SA_CHECK_LAUNCH("attn_bwd_dq_tile_kernel");
    return SA_OK;
}

// dq of a range branch on the tensor cores (head dim 128, at most 16 heads
// per KV head); SA_NSA_BWD_DQ=mma selects the mma.sync kernel instead.
static bool dq_tc_allowed(const BwdParams &p, int d) {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_NSA_BWD_DQ");
        v = (e && std::strcmp(e, "mma") == 0) ? 0 : 1;
    }
    return v && d == 128 && p.G <= 16 && (long long)p.B * p.Tq * p.Hq + 16 < INT_MAX &&
           (long long)p.B * std::max(p.L, 1) < INT_MAX;
}

template <int SRC>
static int launch_nsa_dq_tc(const BwdParams &bp, cudaStream_t st) {
    DqTcParams cp{};
    TileParams &t = cp.t;
    t.q = bp.q; t.k = bp.k; t.klo = SRC == TS_CMP ? bp.klo : bp.k; t.v = bp.v;
    t.B = bp.B; t.T = bp.Tq; t.Lk = std::max(bp.L, 1); t.Hq = bp.Hq; t.Hkv = bp.Hkv; t.G = bp.G;
    t.window = bp.window; t.cmp_len = bp.cmp_len; t.cmp_stride = bp.cmp_stride; t.scale_log2 = bp.scale_log2;
    cp.lse = bp.lse; cp.Dt = bp.Dt; cp.gate = bp.gate; cp.lse_stride = bp.lse_stride; cp.gate_stride = bp.gate_stride;
    cp.dq = bp.dq; cp.dq_accum = bp.dq_accum; cp.scale = bp.scale; cp.err = bp.err;
    const long long items = (long long)bp.B * bp.Hkv * ((bp.Tq + CT_Q - 1) / CT_Q);
    if (items == 0) return SA_OK;
    if (items > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "nsa_dq_tc: %lld items", items);
    cp.n_items = (int)items;
    CUtensorMap qm, dm, khm, klm, vm;
    int rc = bf16_tensor_map(&qm, bp.q, (long long)bp.B * bp.Tq * bp.Hq, 128, 16);
    if (!rc) rc = bf16_tensor_map(&dm, bp.dout, (long long)bp.B * bp.Tq * bp.Hq, 128, 16);
    if (!rc) rc = bf16_tensor_map_3d(&khm, t.k, 128, bp.Hkv, (long long)bp.B * t.Lk, DQ_KT);
    if (!rc) rc = bf16_tensor_map_3d(&klm, t.klo, 128, bp.Hkv, (long long)bp.B * t.Lk, DQ_KT);
    if (!rc) rc = bf16_tensor_map_3d(&vm, t.v, 128, bp.Hkv, (long long)bp.B * t.Lk, DQ_KT);
    if (rc) return rc;
    constexpr int smem = DqSmem::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = nsa_dq_tc_kernel<SRC>;
    rc = set_smem(kern, smem);
    if (rc) return rc;
    const int grid = (int)std::min<long long>(items, sm_count());
    launch_k(__PRETTY_FUNCTION__, kern, grid, DQ_THREADS, smem, st, qm, dm, khm, klm, vm, cp);
    SA_CHECK_LAUNCH("nsa_dq_tc_kernel");
    return SA_OK;
}

// Key-major dK / dV of a range branch on the tensor cores (head dim 128, at
// most 16 heads per KV head); SA_NSA_BWD_KV=mma selects the mma.sync kernel.
static bool kv_tc_allowed(const BwdParams &p, int d) {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_NSA_BWD_KV");
        v = (e && std::strcmp(e, "mma") == 0) ? 0 : 1;
    }
    return v && d == 128 && p.G <= 16 && p.Tq >= KV_QT && p.L >= 1 &&
           (long long)p.B * p.Tq * p.Hq + 16 < INT_MAX && (long long)p.B * p.L + 128 < INT_MAX;
}

template <int SRC>
static int launch_nsa_kv_tc(const BwdParams &bp, float4 *scal, cudaStream_t st) {
    const long long n_sc = (long long)bp.B * bp.Hkv * bp.Tq * 16;
    launch_k("nsa_kv_scalars_kernel", nsa_kv_scalars_kernel, (unsigned)((n_sc + 255) / 256), 256, 0, st,
             bp.lse, bp.lse_stride, (const float *)bp.Dt, bp.gate, bp.gate_stride, bp.B, bp.Tq, bp.Hq, bp.Hkv, bp.G,
             scal);
    SA_CHECK_LAUNCH("nsa_kv_scalars_kernel");
    KvTcParams cp{};
    TileParams &t = cp.t;
    t.q = bp.q; t.k = bp.k; t.klo = SRC == TS_CMP ? bp.klo : bp.k; t.v = bp.v;
    t.B = bp.B; t.T = bp.Tq; t.Lk = bp.L; t.Hq = bp.Hq; t.Hkv = bp.Hkv; t.G = bp.G;
    t.window = bp.window; t.cmp_len = bp.cmp_len; t.cmp_stride = bp.cmp_stride; t.scale_log2 = bp.scale_log2;
    cp.scal = scal; cp.dk = bp.dk; cp.dv = bp.dv; cp.scale = bp.scale; cp.err = bp.err;
    cp.n_kt = (bp.L + 127) / 128;
    const long long max_tiles = SRC == TS_CMP ? bp.Tq / KV_QT + 2 : (128 + (long long)bp.window) / KV_QT + 2;
    cp.n_split = (int)((max_tiles + KV_QSPLIT - 1) / KV_QSPLIT);
    const long long items = (long long)bp.B * bp.Hkv * cp.n_kt * cp.n_split;
    if (items == 0) return SA_OK;
    if (items > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "nsa_kv_tc: %lld items", items);
    cp.n_items = (int)items;
    CUtensorMap qm, dm, khm, klm, vm;
    int rc = bf16_tensor_map(&qm, bp.q, (long long)bp.B * bp.Tq * bp.Hq, 128, 16);
    if (!rc) rc = bf16_tensor_map(&dm, bp.dout, (long long)bp.B * bp.Tq * bp.Hq, 128, 16);
    if (!rc) rc = bf16_tensor_map_3d(&khm, t.k, 128, bp.Hkv, (long long)bp.B * bp.L, 128);
    if (!rc) rc = bf16_tensor_map_3d(&klm, t.klo, 128, bp.Hkv, (long long)bp.B * bp.L, 128);
    if (!rc) rc = bf16_tensor_map_3d(&vm, t.v, 128, bp.Hkv, (long long)bp.B * bp.L, 128);
    if (rc) return rc;
    constexpr int smem = KvSmem::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = nsa_kv_tc_kernel<SRC>;
    rc = set_smem(kern, smem);
    if (rc) return rc;
    const int grid = (int)std::min<long long>(items, sm_count());
    launch_k(__PRETTY_FUNCTION__, kern, grid, KV_THREADS, smem, st, qm, dm, khm, klm, vm, cp);
    SA_CHECK_LAUNCH("nsa_kv_tc_kernel");
    return SA_OK;
}

// Key-major dK / dV of a range branch (window, or compressed rows).
template <int D, bool HILO>
static int launch_bwd_kv(const BwdParams &p, cudaStream_t st) {
    if (p.L <= 0) return SA_OK;
    constexpr int smem = attn_bwd_kv_smem<D, HILO>();
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = attn_bwd_kv_kernel<D, HILO>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    constexpr int KB = 16 * KV_NWK;
    const int n_kb = (p.L + KB - 1) / KB;
    // queries per CTA: long ranges (compressed rows) in 512s, the window's in 256s
    const int q_split = p.window > 0 ? 256 : 512;
    const long long span = p.window > 0 ? (long long)KB - 1 + p.window : (long long)p.Tq;
    const int n_split = (int)std::max(1LL, (span + q_split - 1) / q_split);
    const long long ctas = (long long)p.B * p.Hkv * n_kb * n_split;
    if (ctas > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "attn_bwd_kv: %lld CTAs", ctas);
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)ctas, KV_NWK * 32, smem, st, p, n_kb, n_split, q_split,
             KvLists{});
    SA_CHECK_LAUNCH("attn_bwd_kv_kernel");
    return SA_OK;
}

// Key-major dK / dV of the selected branch over the inverse block lists.
template <int D>
static int launch_bwd_kv_lists(const BwdParams &p, const NsaBwdLayout &lay, char *ws, const int32_t *sel,
                               int sel_block, int sel_topk, cudaStream_t st) {
    int32_t *cnt = reinterpret_cast<int32_t *>(ws + lay.cnt_off);
    int32_t *qoff = reinterpret_cast<int32_t *>(ws + lay.qoff_off);
    int32_t *cur = reinterpret_cast<int32_t *>(ws + lay.cur_off);
    int2 *items = reinterpret_cast<int2 *>(ws + lay.items_off);
    int32_t *n_items = reinterpret_cast<int32_t *>(ws + lay.nitems_off);
    int32_t *qlist = reinterpret_cast<int32_t *>(ws + lay.qlist_off);
    if (lay.n_lists >= INT_MAX || lay.n_entries > INT_MAX || lay.max_items * 8 > INT_MAX)
        return fail(SA_ERR_UNSUPPORTED, "nsa_bwd: %lld block choices exceed the int32 lists", lay.n_entries);
    cudaError_t e = cudaMemsetAsync(cnt, 0, (size_t)lay.n_lists * 4, st);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "nsa_bwd memset: %s", cudaGetErrorString(e));
    const unsigned eg = (unsigned)((lay.n_entries + 255) / 256);
    launch_k("bwd_sel_count_kernel", bwd_sel_count_kernel, eg, 256, 0, st, sel, lay.n_entries, p.Tq, p.Hkv, sel_topk,
             lay.nb, cnt);
    SA_CHECK_LAUNCH("bwd_sel_count_kernel");
    launch_k("bwd_sel_scan_kernel", bwd_sel_scan_kernel, 1u, 1024, 0, st, (const int32_t *)cnt, (int)lay.n_lists,
             KV_SEL_SPLIT, qoff, cur, items, n_items);
    SA_CHECK_LAUNCH("bwd_sel_scan_kernel");
    launch_k("bwd_sel_fill_kernel", bwd_sel_fill_kernel, eg, 256, 0, st, sel, lay.n_entries, p.Tq, p.Hkv, sel_topk,
             lay.nb, cur, qlist);
    SA_CHECK_LAUNCH("bwd_sel_fill_kernel");
    if (D == 128 && kv_tc_allowed(p, D) && sel_block <= 128) {
        // tcgen05 key-major pass: each block in a 128-key tile, its list's queries in tiles of 4
        float4 *scal = reinterpret_cast<float4 *>(ws + lay.scal_off);
        const long long n_sc = (long long)p.B * p.Hkv * p.Tq * 16;
        launch_k("nsa_kv_scalars_kernel", nsa_kv_scalars_kernel, (unsigned)((n_sc + 255) / 256), 256, 0, st,
                 p.lse, p.lse_stride, (const float *)p.Dt, p.gate, p.gate_stride, p.B, p.Tq, p.Hq, p.Hkv, p.G, scal);
        SA_CHECK_LAUNCH("nsa_kv_scalars_kernel");
        KvTcParams cp{};
        TileParams &t = cp.t;
        t.q = p.q; t.k = p.k; t.klo = p.k; t.v = p.v;
        t.B = p.B; t.T = p.Tq; t.Lk = p.L; t.Hq = p.Hq; t.Hkv = p.Hkv; t.G = p.G; t.scale_log2 = p.scale_log2;
        cp.scal = scal; cp.dk = p.dk; cp.dv = p.dv; cp.scale = p.scale; cp.err = p.err;
        cp.qlist = qlist; cp.qoff = qoff; cp.items = items; cp.n_items_dev = n_items;
        cp.nb = lay.nb; cp.sel_block = sel_block; cp.list_split = KV_SEL_SPLIT;
        static_assert(KV_SEL_SPLIT == KV_QSPLIT * KV_QT, "list work items are KV_QSPLIT query tiles");
        CUtensorMap qm, dm, khm, vm;
        int rc = bf16_tensor_map(&qm, p.q, (long long)p.B * p.Tq * p.Hq, 128, 16);
        if (!rc) rc = bf16_tensor_map(&dm, p.dout, (long long)p.B * p.Tq * p.Hq, 128, 16);
        if (!rc) rc = bf16_tensor_map_3d(&khm, p.k, 128, p.Hkv, (long long)p.B * p.L, 128);
        if (!rc) rc = bf16_tensor_map_3d(&vm, p.v, 128, p.Hkv, (long long)p.B * p.L, 128);
        if (rc) return rc;
        constexpr int smem = KvSmem::ALLOC;
        auto kern = nsa_kv_tc_kernel<KV_LISTS>;
        rc = set_smem(kern, smem);
        if (rc) return rc;
        const int grid = (int)std::min<long long>(lay.max_items, sm_count());
        launch_k(__PRETTY_FUNCTION__, kern, grid, KV_THREADS, smem, st, qm, dm, khm, khm, vm, cp);
        SA_CHECK_LAUNCH("nsa_kv_tc_kernel");
        return SA_OK;
    }
    constexpr int smem = attn_bwd_kv_smem<D, false>();
    auto kern = attn_bwd_kv_kernel<D, false, true>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    constexpr int KB = 16 * KV_NWK;
    KvLists kl{qlist, qoff, items, n_items, lay.nb, sel_block, (sel_block + KB - 1) / KB};
    const long long ctas = lay.max_items * kl.n_kbpb;
    if (ctas > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "attn_bwd_kv: %lld CTAs", ctas);
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)ctas, KV_NWK * 32, smem, st, p, 0, 0, KV_SEL_SPLIT, kl);
    SA_CHECK_LAUNCH("attn_bwd_kv_kernel");
    return SA_OK;
}

template <int D>
static int nsa_bwd_branches(const BwdParams &base, const float *gates, const float *lse3, long long rows,
                            float *Dt, const NsaBwdLayout &lay, char *ws, const __nv_bfloat16 *kc,
                            const __nv_bfloat16 *klo, const __nv_bfloat16 *vc, float *dkc, float *dvc,
                            const int32_t *sel, int sel_block, int sel_topk, int window, int cmp_len,
                            int cmp_stride, cudaStream_t st) {
    float4 *scal = reinterpret_cast<float4 *>(ws + lay.scal_off);
    // compressed branch: keys Kc (hi/lo), gradients into dKc / dVc; writes dq
    BwdParams p = base;
    p.k = kc; p.klo = klo; p.v = vc; p.L = std::max(lay.nc, 1);
    p.lse = lse3; p.gate = gates; p.Dt = Dt;
    p.window = 0; p.cmp_len = cmp_len; p.cmp_stride = cmp_stride;
    p.dk = dkc; p.dv = dvc; p.dq_accum = 0;
    if (lay.nc == 0) p.L = 0;       // no compressed row is visible to any query
    int rc = dq_tc_allowed(p, D) ? launch_nsa_dq_tc<TS_CMP>(p, st)   // dq
                                 : launch_bwd_dq_tile<D, true>(p, st);
    if (rc) return rc;
    rc = kv_tc_allowed(p, D) ? launch_nsa_kv_tc<TS_CMP>(p, scal, st)   // dKc, dVc
                             : launch_bwd_kv<D, true>(p, st);
    if (rc) return rc;
    // selected branch: keys of the chosen blocks
    p = base;
    p.lse = lse3 + 1; p.gate = gates + 1; p.Dt = Dt + rows;
    p.idx = sel; p.idx_heads = base.Hkv; p.K = sel_topk; p.block = sel_block;
    p.block_shift = (sel_block & (sel_block - 1)) == 0 ? __builtin_ctz((unsigned)sel_block) : -1;
    p.dq_accum = 1;
    rc = launch_bwd_dq_blocks<D>(p, st);                                // dq
    if (rc) return rc;
    rc = launch_bwd_kv_lists<D>(p, lay, ws, sel, sel_block, sel_topk, st);   // dk, dv
    if (rc) return rc;
    // window branch
    p = base;
    p.lse = lse3 + 2; p.gate = gates + 2; p.Dt = Dt + 2 * rows;
    p.window = window; p.dq_accum = 1;
    rc = dq_tc_allowed(p, D) ? launch_nsa_dq_tc<TS_WINDOW>(p, st)       // dq
                             : launch_bwd_dq_tile<D, false>(p, st);
    if (rc) return rc;
    return kv_tc_allowed(p, D) ? launch_nsa_kv_tc<TS_WINDOW>(p, scal, st)   // dk, dv
                               : launch_bwd_kv<D, false>(p, st);
}

int sa_nsa_bwd(const void *q, const void *k, const void *v, const float *gates, const void *dout,
               const float *o_branches, const float *lse_branches, const int32_t *sel_idx, int B, int T, int Hq,
               int Hkv, int d, int cmp_len, int cmp_stride, int sel_block, int sel_topk, int window, float scale,
               float *dq, float *dk, float *dv, float *dgates, void *workspace, size_t workspace_bytes,
               void *stream) {
    SA_TRACE("sa_nsa_bwd");
    if (B <= 0 || T < 0 || Hq <= 0 || Hkv <= 0 || cmp_len <= 0 || cmp_stride <= 0 || sel_block <= 0 ||
        sel_topk <= 0 || window <= 0)
        return fail(SA_ERR_INVALID_ARG, "nsa_bwd: bad sizes");
    if (Hq % Hkv) return fail(SA_ERR_INVALID_ARG, "nsa_bwd: Hq %% Hkv != 0");
    if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "nsa_bwd: head dim %d", d);
    if (!q || !k || !v || !gates || !dout || !o_branches || !lse_branches || !sel_idx || !dq || !dk || !dv ||
        !dgates || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(gates) || !aligned16(dout) ||
        !aligned16(o_branches) || !aligned4(lse_branches) || !aligned4(sel_idx) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned4(dgates))
        return fail(SA_ERR_INVALID_ARG, "nsa_bwd: null or misaligned pointer");
    if (!std::isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "nsa_bwd: scale");
    if (T == 0) return SA_OK;
    if ((long long)sel_topk * sel_block > INT_MAX / 2) return fail(SA_ERR_UNSUPPORTED, "nsa_bwd: selection size");
    const NsaBwdLayout lay = nsa_bwd_layout(B, T, Hq, Hkv, d, cmp_len, cmp_stride, sel_block, sel_topk);
    if (!workspace || workspace_bytes < lay.total)
        return fail(SA_ERR_WORKSPACE, "nsa_bwd: workspace %zu < %zu", workspace_bytes, lay.total);
    if (!aligned16(workspace)) return fail(SA_ERR_INVALID_ARG, "nsa_bwd: workspace alignment");
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    cudaStream_t st = as_stream(stream);
    char *ws = static_cast<char *>(workspace);
    __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(ws + lay.kc_off);
    __nv_bfloat16 *klo = reinterpret_cast<__nv_bfloat16 *>(ws + lay.klo_off);
    __nv_bfloat16 *vc = reinterpret_cast<__nv_bfloat16 *>(ws + lay.vc_off);
    float *dkc = reinterpret_cast<float *>(ws + lay.dkc_off);
    float *dvc = reinterpret_cast<float *>(ws + lay.dvc_off);
    float *Dt = reinterpret_cast<float *>(ws + lay.dt_off);
    const long long rows = (long long)B * T * Hq;
    const size_t kv_bytes = (size_t)B * T * Hkv * d * 4;
    const size_t ckv_bytes = (size_t)B * std::max(lay.nc, 1) * Hkv * d * 4;
    cudaError_t e = cudaMemsetAsync(dk, 0, kv_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dkc, 0, ckv_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dvc, 0, ckv_bytes, st);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "nsa_bwd memset: %s", cudaGetErrorString(e));
    // 1. compressed rows, as in the forward
    if (lay.nc > 0) {
        const long long n2 = (long long)B * lay.nc * Hkv * (d / 2);
        launch_k("nsa_compress_kernel", nsa_compress_kernel, (unsigned)((n2 + 255) / 256), 256, 0, st,
            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, B, T, Hkv, d, lay.nc, cmp_len, cmp_stride, kc, klo,
            vc);
        SA_CHECK_LAUNCH("nsa_compress_kernel");
    }
    // 2. r_b = dO . O_b per row and branch (the D terms and the gate gradients)
    if (d == 64)
        launch_k("nsa_bwd_prep_kernel<64>", nsa_bwd_prep_kernel<64>, (unsigned)((rows + 7) / 8), 256, 0, st,
            (const __nv_bfloat16 *)dout, o_branches, rows, Dt, dgates);
    else
        launch_k("nsa_bwd_prep_kernel<128>", nsa_bwd_prep_kernel<128>, (unsigned)((rows + 7) / 8), 256, 0, st,
            (const __nv_bfloat16 *)dout, o_branches, rows, Dt, dgates);
    SA_CHECK_LAUNCH("nsa_bwd_prep_kernel");
    // 3. the three branches' backward (dq accumulates over them)
    BwdParams base{};
    base.q = static_cast<const __nv_bfloat16 *>(q); base.k = static_cast<const __nv_bfloat16 *>(k);
    base.v = static_cast<const __nv_bfloat16 *>(v); base.dout = static_cast<const __nv_bfloat16 *>(dout);
    base.B = B; base.Tq = T; base.L = T; base.Hq = Hq; base.Hkv = Hkv; base.G = Hq / Hkv; base.idx_heads = 1;
    base.q_pos0 = 0; base.scale = scale; base.scale_log2 = scale * kLog2e;
    base.lse_stride = 3; base.gate_stride = 3;
    base.dq = dq; base.dk = dk; base.dv = dv; base.err = ew;
    rc = d == 64 ? nsa_bwd_branches<64>(base, gates, lse_branches, rows, Dt, lay, ws, kc, klo, vc, dkc, dvc,
                                        sel_idx, sel_block, sel_topk, window, cmp_len, cmp_stride, st)
                 : nsa_bwd_branches<128>(base, gates, lse_branches, rows, Dt, lay, ws, kc, klo, vc, dkc, dvc,
                                         sel_idx, sel_block, sel_topk, window, cmp_len, cmp_stride, st);
    if (rc) return rc;
    // 4. compressed-row gradients back to the rows they average
    if (lay.nc > 0) {
        const long long n4 = (long long)B * T * Hkv * (d / 4);
        launch_k("nsa_pool_bwd_kernel", nsa_pool_bwd_kernel, (unsigned)((n4 + 255) / 256), 256, 0, st,
            (const float *)dkc, (const float *)dvc, dk, dv, B, T, Hkv, d, lay.nc, cmp_len, cmp_stride);
        SA_CHECK_LAUNCH("nsa_pool_bwd_kernel");
    }
    return SA_OK;
}

// ------------------------------------- full-attention exact indexer --
// Query rows per score/select chunk: the chunk's dense scores stay under
// 1 GiB.
static int full_chunk_rows(int B, int T) {
    const long long stride = (T + 3) / 4 * 4;
    const long long r = (1LL << 28) / ((long long)B * stride);
    return (int)std::max(1LL, std::min<long long>(r, T));
}

struct FullLayout {
    int rows_chunk;
    long long stride;
    size_t of32_off, lse_off, dense_off, total;
};

static FullLayout full_layout(int B, int T, int Hq, int d) {
    FullLayout lay{};
    lay.rows_chunk = full_chunk_rows(B, T);
    lay.stride = (T + 3) / 4 * 4;
    const size_t rows = (size_t)B * T * Hq;
    size_t off = 0;
    lay.of32_off = off; off += round_up(rows * d * 4, 256);
    lay.lse_off = off; off += round_up(rows * 4, 256);
    lay.dense_off = off; off += round_up((size_t)B * lay.rows_chunk * lay.stride * 4, 256);
    lay.total = off;
    return lay;
}

size_t sa_full_attn_topk_workspace_size(int B, int T, int Hq, int Hkv, int d, int topk, int window) {
    (void)Hkv; (void)topk; (void)window;
    if (B <= 0 || T <= 0 || Hq <= 0 || d <= 0) return 0;
    return full_layout(B, T, Hq, d).total;
}

template <int D>
static int launch_full_score(const FullScoreParams &p, cudaStream_t st) {
    constexpr int smem = full_score_smem<D>();
    auto kern = full_score_kernel<D>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    const long long ctas = (long long)p.B * ((p.Rt + FS_WARPS - 1) / FS_WARPS);
    if (ctas == 0) return SA_OK;
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)ctas, FS_WARPS * 32, smem, st, p);
    SA_CHECK_LAUNCH("full_score_kernel");
    return SA_OK;
}

// The score pass on the tensor cores (head dim 128, 16 query heads per KV
// head); SA_FULL_SCORE=mma selects the mma.sync kernel.
static bool full_score_tc_allowed(const FullScoreParams &p, int d) {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("SA_FULL_SCORE");
        v = (e && std::strcmp(e, "mma") == 0) ? 0 : 1;
    }
    return v && d == 128 && p.G == 16 && aligned16(p.lse) && (long long)p.B * p.T * p.Hq + 16 < INT_MAX &&
           (long long)p.B * p.T + FX_KT < INT_MAX;
}

static int launch_full_score_tc(const FullScoreParams &fp, unsigned *ew, cudaStream_t st) {
    FxParams cp{};
    cp.f = fp;
    cp.err = ew;
    cp.nqb = (fp.Rt + FX_QB - 1) / FX_QB;
    const long long t_last = (long long)fp.t0 + fp.Rt - 1;
    const long long n_max = std::max(0LL, fp.window > 0 ? t_last - fp.window + 1 : t_last + 1);
    const long long n_piece = ((n_max + FX_KT - 1) / FX_KT + FX_PIECE - 1) / FX_PIECE;
    const long long items = n_piece * fp.B * cp.nqb;
    if (items == 0) return SA_OK;
    if (items > INT_MAX) return fail(SA_ERR_UNSUPPORTED, "full_score_tc: %lld items", items);
    cp.n_items = (int)items;
    CUtensorMap qm, km;
    int rc = bf16_tensor_map(&qm, fp.q, (long long)fp.B * fp.T * fp.Hq, 128, 16);
    if (!rc) rc = bf16_tensor_map_3d(&km, fp.k, 128, fp.Hkv, (long long)fp.B * fp.T, FX_KT);
    if (rc) return rc;
    constexpr int smem = FxSmem::ALLOC;
    static_assert(smem <= 227 * 1024, "shared memory");
    rc = set_smem(full_score_tc_kernel, smem);
    if (rc) return rc;
    const int grid = (int)std::min<long long>(items, sm_count());
    launch_k("full_score_tc_kernel", full_score_tc_kernel, grid, FX_THREADS, smem, st, qm, km, cp);
    SA_CHECK_LAUNCH("full_score_tc_kernel");
    return SA_OK;
}

template <int NT>
static int launch_select_dense(const IdxParams &p, int words, cudaStream_t st) {
    const int smem = select_smem_staged<64>(words, 0);
    auto kern = topk_select_kernel<64, NT, true>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    launch_k(__PRETTY_FUNCTION__, kern, dim3(1u, (unsigned)p.Rt, (unsigned)p.B), NT, smem, st, p);
    SA_CHECK_LAUNCH("topk_select_kernel");
    return SA_OK;
}

int sa_full_attn_topk(const void *q, const void *k, const void *v, int B, int T, int Hq, int Hkv, int d,
                      float scale, int topk, int window, void *out, float *lse, int32_t *out_idx,
                      void *workspace, size_t workspace_bytes, void *stream) {
    SA_TRACE("sa_full_attn_topk");
    if (B <= 0 || T < 0 || Hq <= 0 || Hkv <= 0 || topk < 0 || window < 0 || topk + window < 1)
        return fail(SA_ERR_INVALID_ARG, "full_attn_topk: bad sizes");
    if (Hq % Hkv) return fail(SA_ERR_INVALID_ARG, "full_attn_topk: Hq %% Hkv != 0");
    if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "full_attn_topk: head dim %d", d);
    if (!q || !k || !v || !out_idx || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(out_idx) ||
        (out && !aligned16(out)) || (lse && !aligned4(lse)))
        return fail(SA_ERR_INVALID_ARG, "full_attn_topk: null or misaligned pointer");
    if (!std::isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "full_attn_topk: scale");
    if (T == 0) return SA_OK;
    const FullLayout lay = full_layout(B, T, Hq, d);
    if (!workspace || workspace_bytes < lay.total)
        return fail(SA_ERR_WORKSPACE, "full_attn_topk: workspace %zu < %zu", workspace_bytes, lay.total);
    if (!aligned16(workspace)) return fail(SA_ERR_INVALID_ARG, "full_attn_topk: workspace alignment");
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    cudaStream_t st = as_stream(stream);
    char *ws = static_cast<char *>(workspace);
    float *of32 = reinterpret_cast<float *>(ws + lay.of32_off);
    float *lse_ = lse ? lse : reinterpret_cast<float *>(ws + lay.lse_off);
    int32_t *dense = reinterpret_cast<int32_t *>(ws + lay.dense_off);
    const int G = Hq / Hkv;
    const long long rows = (long long)B * T * Hq;
    // 1. the full layer: causal attention over every earlier key (a window
    //    as long as the sequence)
    {
        TileParams p{};
        p.q = static_cast<const __nv_bfloat16 *>(q); p.k = static_cast<const __nv_bfloat16 *>(k);
        p.v = static_cast<const __nv_bfloat16 *>(v);
        p.B = B; p.T = T; p.Lk = T; p.Hq = Hq; p.Hkv = Hkv; p.G = G;
        p.window = T; p.scale_log2 = scale * kLog2e;
        p.out_f32 = of32; p.lse = lse_;
        rc = (G <= 16 && cmp_tc_applies(p, d)) ? launch_nsa_tc<TS_WINDOW>(p, ew, st)
                                                 : launch_tile(p, d, TS_WINDOW, st);
        if (rc) return rc;
        if (out) {
            const long long n2 = rows * d / 2;
            launch_k("f32_to_bf16_kernel", f32_to_bf16_kernel, (unsigned)((n2 + 255) / 256), 256, 0, st,
                (const float *)of32, n2, (__nv_bfloat16 *)out);
            SA_CHECK_LAUNCH("f32_to_bf16_kernel");
        }
    }
    // 2 + 3. per chunk of query rows: exact scores, then the exact top-k
    for (int t0 = 0; t0 < T; t0 += lay.rows_chunk) {
        const int Rt = std::min(lay.rows_chunk, T - t0);
        FullScoreParams fp{};
        fp.q = static_cast<const __nv_bfloat16 *>(q); fp.k = static_cast<const __nv_bfloat16 *>(k);
        fp.lse = lse_;
        fp.B = B; fp.T = T; fp.Hq = Hq; fp.Hkv = Hkv; fp.G = G;
        fp.t0 = t0; fp.Rt = Rt; fp.window = window; fp.scale_log2 = scale * kLog2e;
        fp.dense = dense; fp.stride = lay.stride;
        rc = full_score_tc_allowed(fp, d) ? launch_full_score_tc(fp, ew, st)
             : d == 64                    ? launch_full_score<64>(fp, st)
                                          : launch_full_score<128>(fp, st);
        if (rc) return rc;
        IdxParams ip{};
        ip.B = B; ip.Tq = T; ip.L = T; ip.q_pos0 = 0; ip.window = window; ip.topk = topk;
        ip.Kout = topk + window; ip.t0 = t0; ip.Rt = Rt;
        ip.out_idx = out_idx; ip.out_count = nullptr; ip.err = ew;
        ip.dense = dense; ip.dense_stride = lay.stride;
        const long long ncand = window > 0 ? (long long)t0 + Rt - window : (long long)t0 + Rt;
        const int words = (int)((std::max(ncand, 1LL) + 31) / 32);
        rc = ((long long)B * Rt <= sm_count()) ? launch_select_dense<1024>(ip, words, st)
                                                : launch_select_dense<SEL_THREADS>(ip, words, st);
        if (rc) return rc;
    }
    return SA_OK;
}

// ------------------------------------------------------ IndexCache driver --
size_t sa_dsa_decode_layers_workspace_size(int B, int Tq, int L, int Hq, int d, int Hi, int di,
                                           int topk, int window, int n_split) {
    const size_t a = sa_indexer_topk_workspace_size(B, Tq, L, Hi, di, topk, window);
    const size_t b = sa_sparse_attn_workspace_size(B, Tq, Hq, d, n_split);
    const size_t idx = round_up((size_t)B * Tq * (topk + window) * 4, 256);
    return round_up(std::max(a, b), 256) + idx;
}

int sa_dsa_decode_layers(const char *pattern, int n_layers, const sa_dsa_layer *layers, int B, int Tq,
                         int L, int Hq, int Hkv, int d, int Hi, int di, int64_t q_pos0, int topk,
                         int window, float scale, int n_split, int32_t *idx_cache, void *workspace,
                         size_t workspace_bytes, void *stream) {
    SA_TRACE("sa_dsa_decode_layers");
    if (!pattern || !layers || n_layers <= 0 || (int)strlen(pattern) < n_layers)
        return fail(SA_ERR_INVALID_ARG, "dsa_layers: pattern/layers");
    if (pattern[0] != 'F') return fail(SA_ERR_INVALID_ARG, "dsa_layers: the first layer must be 'F'");
    for (int i = 0; i < n_layers; ++i)
        if (pattern[i] != 'F' && pattern[i] != 'S')
            return fail(SA_ERR_INVALID_ARG, "dsa_layers: pattern char %d is '%c'", i, pattern[i]);
    const size_t need = sa_dsa_decode_layers_workspace_size(B, Tq, L, Hq, d, Hi, di, topk, window, n_split);
    if (!workspace || workspace_bytes < need)
        return fail(SA_ERR_WORKSPACE, "dsa_layers: workspace %zu < %zu", workspace_bytes, need);
    if (!aligned16(workspace)) return fail(SA_ERR_INVALID_ARG, "dsa_layers: workspace alignment");
    const size_t a = sa_indexer_topk_workspace_size(B, Tq, L, Hi, di, topk, window);
    const size_t b = sa_sparse_attn_workspace_size(B, Tq, Hq, d, n_split);
    const size_t scratch = round_up(std::max(a, b), 256);
    int32_t *cache = idx_cache ? idx_cache : reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + scratch);
    const int K = topk + window;
    for (int i = 0; i < n_layers; ++i) {
        const sa_dsa_layer &ly = layers[i];
        if (pattern[i] == 'F') {
            int rc = sa_indexer_topk(ly.q_idx, ly.k_idx, ly.w, B, Tq, L, Hi, di, q_pos0, topk, window, cache,
                                     nullptr, workspace, scratch, stream);
            if (rc) return rc;
        }
        int rc = sa_sparse_attn_fwd(ly.q, ly.k, ly.v, B, Tq, L, Hq, Hkv, d, q_pos0, cache, 1, K, nullptr,
                                    nullptr, nullptr, nullptr, scale, n_split, ly.out, ly.lse, nullptr, nullptr,
                                    workspace, scratch, stream);
        if (rc) return rc;
    }
    return SA_OK;
}


// -------------------------------------------------- gather ceiling probe --
template <int MODE, int STAGES>
static int launch_probe(const ProbeParams &p, int ctas, int smem, cudaStream_t st) {
    auto kern = probe_gather_kernel<MODE, STAGES>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    launch_k(__PRETTY_FUNCTION__, kern, ctas, p.warps * 32, smem, st, p);
    SA_CHECK_LAUNCH("probe_gather_kernel");
    return SA_OK;
}

int sa_probe_gather(const void *buf, int64_t n_rows, int mode, int warps, int stages, int iters,
                    int ctas_per_sm, unsigned *sink, void *stream) {
    SA_TRACE("sa_probe_gather");
    if (!buf || !sink || !aligned16(buf) || !aligned4(sink) || n_rows < 1 || n_rows > UINT_MAX)
        return fail(SA_ERR_INVALID_ARG, "probe_gather: buffer/sink/rows");
    if (mode < 0 || mode > 2) return fail(SA_ERR_INVALID_ARG, "probe_gather: mode %d", mode);
    if (mode == 2 && n_rows < PROBE_BLOCK / PROBE_ROW) return fail(SA_ERR_INVALID_ARG, "probe_gather: rows < one block");
    if (warps < 1 || warps > 16 || iters < 1 || ctas_per_sm < 1 || ctas_per_sm > 8)
        return fail(SA_ERR_INVALID_ARG, "probe_gather: warps %d iters %d ctas/SM %d", warps, iters, ctas_per_sm);
    if (mode == 0 ? !(stages == 2 || stages == 4 || stages == 8) : (stages < 2 || stages > 16))
        return fail(SA_ERR_INVALID_ARG, "probe_gather: stages %d", stages);
    const int smem = probe_smem_bytes(warps, stages, mode);
    if ((long long)smem * ctas_per_sm > 227LL * 1024)
        return fail(SA_ERR_INVALID_ARG, "probe_gather: %d bytes of shared memory x %d CTAs per SM", smem, ctas_per_sm);
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    ProbeParams p{static_cast<const unsigned char *>(buf), (unsigned)n_rows, warps, stages, iters, sink, ew};
    const int ctas = sm_count() * ctas_per_sm;
    cudaStream_t st = as_stream(stream);
    if (mode == 1) return launch_probe<1, 2>(p, ctas, smem, st);
    if (mode == 2) return launch_probe<2, 2>(p, ctas, smem, st);
    if (stages == 2) return launch_probe<0, 2>(p, ctas, smem, st);
    if (stages == 4) return launch_probe<0, 4>(p, ctas, smem, st);
    return launch_probe<0, 8>(p, ctas, smem, st);
}

// ------------------------------------------------------------- backward --
size_t sa_sparse_attn_bwd_workspace_size(int B, int Tq, int Hq) {
    if (B <= 0 || Tq <= 0 || Hq <= 0) return 0;
    return round_up((size_t)B * Tq * Hq * 4, 256);
}

template <int D>
static int launch_bwd(const BwdParams &p, long long rows, cudaStream_t st) {
    constexpr int NW = 8;
    launch_k("attn_bwd_prep_kernel<D>", attn_bwd_prep_kernel<D>, (unsigned)((rows + 7) / 8), 256, 0, st, p, rows);
    SA_CHECK_LAUNCH("attn_bwd_prep_kernel");
    constexpr int smem = attn_bwd_smem_bytes<D, NW>();
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = attn_bwd_kernel<D, NW>;
    int rc = set_smem(kern, smem);
    if (rc) return rc;
    const long long items = (long long)p.B * p.Tq * p.Hkv * ((p.G + 15) / 16);
    if (items == 0) return SA_OK;
    launch_k(__PRETTY_FUNCTION__, kern, (unsigned)((items + NW - 1) / NW), NW * 32, smem, st, p);
    SA_CHECK_LAUNCH("attn_bwd_kernel");
    return SA_OK;
}

int sa_sparse_attn_bwd(const void *q, const void *k, const void *v, const void *out, const float *lse,
                       const void *dout, int B, int Tq, int L, int Hq, int Hkv, int d, int64_t q_pos0,
                       const int32_t *idx, int idx_heads, int K, float scale, float *dq, float *dk, float *dv,
                       void *workspace, size_t workspace_bytes, void *stream) {
    SA_TRACE("sa_sparse_attn_bwd");
    if (B <= 0 || Tq < 0 || L <= 0 || Hq <= 0 || Hkv <= 0 || K < 0 || Hq % Hkv)
        return fail(SA_ERR_INVALID_ARG, "attn_bwd: bad sizes B=%d Tq=%d L=%d Hq=%d Hkv=%d K=%d", B, Tq, L, Hq, Hkv, K);
    if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "attn_bwd: head dim %d", d);
    if (q_pos0 < 0 || q_pos0 + Tq > L)
        return fail(SA_ERR_INVALID_ARG, "attn_bwd: query positions outside [0, L)");
    if (!(idx_heads == 1 || idx_heads == Hkv)) return fail(SA_ERR_INVALID_ARG, "attn_bwd: idx_heads");
    if (!q || !k || !v || !out || !lse || !dout || !idx || !dq || !dk || !dv || !aligned16(q) || !aligned16(k) ||
        !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned4(lse) || !aligned4(idx) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return fail(SA_ERR_INVALID_ARG, "attn_bwd: null or misaligned pointer");
    if (!std::isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "attn_bwd: scale");
    if (Tq == 0) return SA_OK;
    const size_t need = sa_sparse_attn_bwd_workspace_size(B, Tq, Hq);
    if (!workspace || workspace_bytes < need)
        return fail(SA_ERR_WORKSPACE, "attn_bwd: workspace %zu < %zu", workspace_bytes, need);
    if (!aligned16(workspace)) return fail(SA_ERR_INVALID_ARG, "attn_bwd: workspace alignment");
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    cudaStream_t st = as_stream(stream);
    const size_t kv_bytes = (size_t)B * L * Hkv * d * 4;
    cudaError_t e = cudaMemsetAsync(dk, 0, kv_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, st);
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "attn_bwd memset: %s", cudaGetErrorString(e));
    BwdParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q); p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v); p.o = static_cast<const __nv_bfloat16 *>(out);
    p.dout = static_cast<const __nv_bfloat16 *>(dout); p.lse = lse; p.idx = idx;
    p.B = B; p.Tq = Tq; p.L = L; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv; p.idx_heads = idx_heads; p.K = K;
    p.q_pos0 = q_pos0; p.scale = scale; p.scale_log2 = scale * kLog2e;
    p.lse_stride = 1; p.gate = nullptr; p.dq_accum = 0;
    p.Dt = static_cast<float *>(workspace); p.dq = dq; p.dk = dk; p.dv = dv; p.err = ew;
    const long long rows = (long long)B * Tq * Hq;
    return d == 64 ? launch_bwd<64>(p, rows, st) : launch_bwd<128>(p, rows, st);
}

// ------------------------------------------------- sequence split (Star) --
int sa_indexer_scores_at(const int8_t *q_idx, const int8_t *k_idx, const int32_t *w, int B, int Tq, int L, int Hi,
                         int di, const int32_t *idx, int K, int32_t *out_score, void *stream) {
    SA_TRACE("sa_indexer_scores_at");
    if (B <= 0 || Tq < 0 || L <= 0 || K < 0) return fail(SA_ERR_INVALID_ARG, "scores_at: bad sizes");
    if (!indexer_shape_ok(Hi, di)) return fail(SA_ERR_UNSUPPORTED, "scores_at: Hi=%d di=%d", Hi, di);
    if (!q_idx || !k_idx || !w || !idx || !out_score || !aligned16(q_idx) || !aligned16(k_idx) || !aligned4(w) ||
        !aligned4(idx) || !aligned4(out_score))
        return fail(SA_ERR_INVALID_ARG, "scores_at: null or misaligned pointer");
    if (Tq == 0 || K == 0) return SA_OK;
    unsigned *ew = nullptr;
    int rc = device_error_word(&ew);
    if (rc) return rc;
    const unsigned blocks = (unsigned)((long long)B * Tq);
    cudaStream_t st = as_stream(stream);
    if (di == 32) launch_k("idx_scores_at_kernel<32>", idx_scores_at_kernel<32>, blocks, 128, 0, st, q_idx, k_idx, w,
        B, Tq, L, Hi, idx, K, out_score, ew);
    else if (di == 64) launch_k("idx_scores_at_kernel<64>", idx_scores_at_kernel<64>, blocks, 128, 0, st, q_idx,
        k_idx, w, B, Tq, L, Hi, idx, K, out_score, ew);
    else launch_k("idx_scores_at_kernel<128>", idx_scores_at_kernel<128>, blocks, 128, 0, st, q_idx, k_idx, w, B, Tq,
        L, Hi, idx, K, out_score, ew);
    SA_CHECK_LAUNCH("idx_scores_at_kernel");
    return SA_OK;
}

int sa_topk_merge(const int32_t *cand_score, const int32_t *cand_idx, const int64_t *part_off, int n_parts,
                  int64_t rows, int kc, int topk, int window, int64_t q_pos, int32_t *out_idx, int32_t *out_count,
                  void *stream) {
    SA_TRACE("sa_topk_merge");
    if (n_parts < 1 || n_parts > TM_MAX_PARTS || rows < 0 || kc < 0 || topk < 0 || window < 0 || q_pos < 0)
        return fail(SA_ERR_INVALID_ARG, "topk_merge: bad sizes (n_parts 1..%d)", TM_MAX_PARTS);
    if (topk > TM_MAX_K || (long long)n_parts * kc > TM_MAX_CAND)
        return fail(SA_ERR_UNSUPPORTED, "topk_merge: topk %d (max %d) or %lld candidates per row (max %d)", topk,
                    TM_MAX_K, (long long)n_parts * kc, TM_MAX_CAND);
    if (!cand_score || !cand_idx || !part_off || !out_idx || !aligned4(cand_score) || !aligned4(cand_idx) ||
        !aligned4(out_idx) || (out_count && !aligned4(out_count)))
        return fail(SA_ERR_INVALID_ARG, "topk_merge: null or misaligned pointer");
    if (rows == 0) return SA_OK;
    MergeOffsets mo{};
    for (int i = 0; i < n_parts; ++i) {
        if (part_off[i] < 0) return fail(SA_ERR_INVALID_ARG, "topk_merge: negative part offset");
        mo.off[i] = part_off[i];
    }
    const int smem = topk_merge_smem_bytes(n_parts * kc);
    int rc = set_smem(topk_merge_kernel, smem);
    if (rc) return rc;
    launch_k("topk_merge_kernel", topk_merge_kernel, (unsigned)rows, TM_THREADS, smem, as_stream(stream), cand_score,
        cand_idx, mo, n_parts, rows, kc, topk, window, q_pos, out_idx, out_count);
    SA_CHECK_LAUNCH("topk_merge_kernel");
    return SA_OK;
}

int sa_index_shard(const int32_t *idx, int64_t n, int64_t key_lo, int64_t key_hi, int32_t *out, void *stream) {
    SA_TRACE("sa_index_shard");
    if (n < 0 || key_lo < 0 || key_hi < key_lo || !idx || !out || !aligned4(idx) || !aligned4(out))
        return fail(SA_ERR_INVALID_ARG, "index_shard: bad arguments");
    if (n == 0) return SA_OK;
    const unsigned blocks = (unsigned)((n + 255) / 256);
    launch_k("index_shard_kernel", index_shard_kernel, blocks, 256, 0, as_stream(stream), idx, n, key_lo, key_hi, out);
    SA_CHECK_LAUNCH("index_shard_kernel");
    return SA_OK;
}
