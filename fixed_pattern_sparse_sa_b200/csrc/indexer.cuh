// indexer.cuh -- lightweight-indexer scores and exact causal top-k.
//
// IndexCache page ("IndexCache: inferencia 82% mas rapida ...", body): a
// lightweight indexer scores every earlier token and each query keeps a small
// top-scoring subset.  Score of query t for key j:
//   I(t, j) = sum_h w[t,h] * max(0, q_idx[t,h,:] . k_idx[j,:])   (exact int32)
//
// Stage 1 (idx_score_kernel): int8 tensor-core products (mma.sync
// m16n8k32 s8 -> s32, exact).  Keys form the M side of the tile and the
// (query, head) pairs the N side, so the head sum of one query is a sum over
// the columns a thread (or its quad) already holds.  The contraction index is
// permuted identically on both operands so each lane loads its A and B
// fragments as contiguous 4..32-byte runs straight from global memory.
// Scores of a chunk of query rows land in a row-major int32 buffer.
//
// Stage 2 (topk_select_kernel): one thread-block cluster per query row.  The
// row is cut into one segment per CTA; min/max, radix histograms (12-bit
// digits over score - min) and the final counts are merged across the
// cluster through distributed shared memory, so the exact k-th largest score
// is found in at most three digit passes.  Keys above it are kept, and keys
// equal to it are kept in ascending index order until k are chosen (ties go
// to the lower index).  Output is written in ascending position order, then
// the forced recent window.
#pragma once

#include <cooperative_groups.h>

#include "sa_common.cuh"
#include "tc_common.cuh"

namespace sa {

namespace cg = cooperative_groups;

struct IdxScoreParams {
    const int8_t *q;       // [B, Tq, Hi, DI]
    const int8_t *k;       // [B, L, DI]
    const int32_t *w;      // [B, Tq, Hi]
    int B, Tq, L;
    long long q_pos0;
    int window;
    int t0, Rt;            // chunk: query rows t0 .. t0+Rt-1 of every batch element
    long long ld;          // row stride of the score buffer (elements)
    int32_t *scores;       // [B, Rt, ld]
    unsigned *err;         // device error word
};

// Number of selectable (non-window) candidates of a query at position p.
__device__ __forceinline__ long long n_candidates(long long p, int window) {
    long long n = window > 0 ? p - window + 1 : p + 1;
    return n > 0 ? n : 0;
}

// CTA tile: SC_KEYS keys (8 warps x SC_MT m-tiles of 16) x 128 (query, head)
// columns (QT = 128 / HI queries).  Each lane keeps the B fragments of all 128
// columns in registers; each warp walks its keys one m-tile at a time.
constexpr int SC_WARPS = 8;
constexpr int SC_MT = 8;                                   // m-tiles per warp
constexpr int SC_KEYS = SC_WARPS * SC_MT * 16;             // 1024 keys per CTA

template <int HI, int DI>
__global__ void __launch_bounds__(SC_WARPS * 32) idx_score_kernel(const IdxScoreParams p) {
    constexpr int COLS = 128;                // (query, head) columns per CTA
    constexpr int QT = COLS / HI;            // queries per CTA
    constexpr int NT = COLS / 8;             // n-tiles
    constexpr int REG = DI / 16;             // u32 registers per lane per row
    constexpr int KSTEPS = DI / 32;
    static_assert(HI == 1 || HI == 2 || HI == 4 || HI == 8 || HI == 16, "HI");
    static_assert(DI == 32 || DI == 64 || DI == 128, "DI");

    __shared__ int ws[COLS];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, qc = lane & 3;
    const int b = blockIdx.z;
    const int tq0 = p.t0 + blockIdx.y * QT;               // first query of the tile
    const int t_last = min(p.t0 + p.Rt, p.Tq) - 1;
    const int tq_last = min(tq0 + QT - 1, t_last);
    if (tq0 > t_last) return;
    const long long ncand_last = n_candidates(p.q_pos0 + tq_last, p.window);
    const int j_cta = blockIdx.x * SC_KEYS;
    if ((long long)j_cta >= ncand_last) return;           // above the diagonal

    for (int i = threadIdx.x; i < COLS; i += blockDim.x) {
        const int tq = tq0 + i / HI;
        ws[i] = tq <= tq_last ? __ldg(p.w + ((long long)b * p.Tq + tq) * HI + i % HI) : 0;
    }
    // B fragments (query side), all n-tiles, kept in registers
    unsigned bq[NT][REG];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + gr;
        const int tq = tq0 + col / HI, h = col % HI;
        const unsigned *src = reinterpret_cast<const unsigned *>(
            p.q + (((long long)b * p.Tq + tq) * HI + h) * DI + qc * (DI / 4));
#pragma unroll
        for (int r = 0; r < REG; ++r) bq[nt][r] = tq <= tq_last ? __ldg(src + r) : 0u;
    }
    __syncthreads();

    const int j_warp = j_cta + warp * SC_MT * 16;
    // A fragments of the next m-tile are fetched one step ahead
    unsigned a_nx[2][REG];
    auto load_a = [&](int mt, unsigned (&a)[2][REG]) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int j = j_warp + mt * 16 + gr + hr * 8;
            const unsigned *src = reinterpret_cast<const unsigned *>(
                p.k + ((long long)b * p.L + j) * DI + qc * (DI / 4));
#pragma unroll
            for (int r = 0; r < REG; ++r) a[hr][r] = j < p.L ? __ldg(src + r) : 0u;
        }
    };
    if ((long long)j_warp < ncand_last) load_a(0, a_nx);

#pragma unroll 1
    for (int mt = 0; mt < SC_MT; ++mt) {
        const int jm = j_warp + mt * 16;
        if ((long long)jm >= ncand_last) break;           // the rest is above the diagonal
        unsigned a[2][REG];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr)
#pragma unroll
            for (int r = 0; r < REG; ++r) a[hr][r] = a_nx[hr][r];
        if (mt + 1 < SC_MT && (long long)(jm + 16) < ncand_last) load_a(mt + 1, a_nx);

#pragma unroll
        for (int ng = 0; ng < NT / 4; ++ng) {
            int acc[4][4];
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks)
                    mma_s8_16832(acc[n], a[0][2 * ks], a[1][2 * ks], a[0][2 * ks + 1], a[1][2 * ks + 1],
                                 bq[ng * 4 + n][2 * ks], bq[ng * 4 + n][2 * ks + 1]);
            }
            // epilogue: w * relu, sum over the heads of each query, store
            int pr0 = 0, pr1 = 0;                             // HI == 16: even n-tile's half
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int nt = ng * 4 + n;
                const int c0 = nt * 8 + 2 * qc;               // columns c0, c0+1 of this thread
                const int w0 = ws[c0], w1 = ws[c0 + 1];
                const int s0 = w0 * max(acc[n][0], 0), s1 = w1 * max(acc[n][1], 0);   // key gr
                const int s2 = w0 * max(acc[n][2], 0), s3 = w1 * max(acc[n][3], 0);   // key gr+8
                if constexpr (HI == 1) {
                    // every column is its own query
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int qi = c0 + (e & 1);
                        const int key = jm + gr + (e >> 1) * 8;
                        const int tq = tq0 + qi;
                        const int v = e == 0 ? s0 : e == 1 ? s1 : e == 2 ? s2 : s3;
                        if (tq <= tq_last && key < n_candidates(p.q_pos0 + tq, p.window))
                            p.scores[((long long)b * p.Rt + (tq - p.t0)) * p.ld + key] = v;
                    }
                } else {
                    int r0 = s0 + s1, r1 = s2 + s3;
                    if constexpr (HI >= 4) {
                        r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
                        r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
                    }
                    if constexpr (HI >= 8) {
                        r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
                        r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
                    }
                    bool ready = true;
                    if constexpr (HI == 16) {                  // n-tiles 2m, 2m+1 = one query
                        if ((n & 1) == 0) { pr0 = r0; pr1 = r1; ready = false; }
                        else { r0 += pr0; r1 += pr1; }
                    }
                    constexpr int LEAD = HI >= 8 ? 4 : (HI == 4 ? 2 : 1);
                    const int tq = tq0 + c0 / HI;
                    if (ready && (qc % LEAD) == 0 && tq <= tq_last) {
                        const long long nc = n_candidates(p.q_pos0 + tq, p.window);
                        int32_t *dst = p.scores + ((long long)b * p.Rt + (tq - p.t0)) * p.ld;
                        if (jm + gr < nc) dst[jm + gr] = r0;
                        if (jm + gr + 8 < nc) dst[jm + gr + 8] = r1;
                    }
                }
            }
        }
    }
}

// ------------------------------------------------- tcgen05 score kernel --
// Tensor-core (tcgen05, kind::i8) version of the score GEMM.  CTA tile:
// M = 128 keys (TMEM lanes) x N = 256 (query, head) columns (256/HI queries)
// x K = DI; the accumulator lives in 256 TMEM columns.  Operands are staged
// with cp.async in the K-major no-swizzle core-matrix layout: 8-row group r8
// at r8 * 8*DI bytes, inside it the DI/16 core matrices (8 rows x 16 B)
// back to back, so LBO = 128 B (next core along K) and SBO = 8*DI (next
// 8-row group).  Thread i of warp w owns key row 32w+i: it reads that TMEM
// lane and forms sum_h w*relu(s_h) for every query of the tile.
constexpr int TC_KT = 8;                 // 128-key tiles per CTA
constexpr int TC_SMEM = 80 * 1024;       // > 227/3 KB: at most 2 CTAs (2 x 256 TMEM columns) per SM
constexpr long long TC_WAIT_CYCLES = 4000000000LL;   // ~2 s: bounded wait on the MMA barrier

__device__ __forceinline__ int tc_core_off(int row, int chunk, int di) {
    return (row >> 3) * (8 * di) + chunk * 128 + (row & 7) * 16;
}

template <int HI, int DI>
__global__ void __launch_bounds__(128) idx_score_tc_kernel(const IdxScoreParams p) {
    constexpr int NCOL = 256;                // N: (query, head) columns
    constexpr int NQ = NCOL / HI;            // queries per CTA
    constexpr int CH = DI / 16;              // 16-byte chunks per row
    constexpr int A_BYTES = 128 * DI;
    constexpr int B_BYTES = NCOL * DI;
    static_assert(2 * A_BYTES + B_BYTES + NCOL * 4 + 64 <= TC_SMEM, "smem");
    constexpr uint32_t IDESC = tc::make_idesc(2 /*s32*/, 1 /*s8*/, 128, NCOL);

    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *a_s = smem;                               // 2 x A tile
    unsigned char *b_s = smem + 2 * A_BYTES;                 // B tile
    int *w_s = reinterpret_cast<int *>(b_s + B_BYTES);       // [NCOL]
    uint64_t *bar = reinterpret_cast<uint64_t *>(w_s + NCOL);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z;
    const int tq0 = p.t0 + blockIdx.y * NQ;
    const int t_last = min(p.t0 + p.Rt, p.Tq) - 1;
    const int tq_last = min(tq0 + NQ - 1, t_last);
    if (tq0 > t_last) return;
    const long long ncand_last = n_candidates(p.q_pos0 + tq_last, p.window);
    const int j_cta = blockIdx.x * TC_KT * 128;
    if ((long long)j_cta >= ncand_last) return;              // above the diagonal (uniform)
    const int n_tiles = (int)min((long long)TC_KT, (ncand_last - j_cta + 127) / 128);

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, NCOL);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_fence_init();
    }
    // B tile: rows (q, h) of q_idx are contiguous in memory
    {
        const int8_t *src = p.q + (((long long)b * p.Tq + tq0) * HI) * DI;
        const int nrows_valid = (tq_last - tq0 + 1) * HI;
        for (int i = tid; i < NCOL * CH; i += 128) {
            const int row = i / CH, c = i % CH;
            const bool ok = row < nrows_valid;
            cp_async16(b_s + tc_core_off(row, c, DI), ok ? src + (long long)row * DI + c * 16 : src, ok ? 16 : 0);
        }
        for (int i = tid; i < NCOL; i += 128) {
            const int tq = tq0 + i / HI;
            w_s[i] = tq <= tq_last ? __ldg(p.w + ((long long)b * p.Tq + tq) * HI + i % HI) : 0;
        }
    }
    auto load_a = [&](int kt) {
        unsigned char *dst = a_s + (kt & 1) * A_BYTES;
        const int j0 = j_cta + kt * 128;
        const int8_t *src = p.k + ((long long)b * p.L) * DI;
        for (int i = tid; i < 128 * CH; i += 128) {
            const int row = i / CH, c = i % CH;
            const int j = j0 + row;
            const bool ok = j < p.L;
            cp_async16(dst + tc_core_off(row, c, DI), ok ? src + (long long)j * DI + c * 16 : src, ok ? 16 : 0);
        }
        cp_async_commit();
    };
    load_a(0);
    cp_async_wait<0>();
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    bool timed_out = false;
    uint32_t pending = 0;   // parity of the MMA batch in flight
    for (int kt = 0; kt < n_tiles; ++kt) {
        pending = kt & 1;
        if (tid == 0) {
            const uint32_t a_addr = tc::smem_u32(a_s + (kt & 1) * A_BYTES);
            const uint32_t b_addr = tc::smem_u32(b_s);
#pragma unroll
            for (int kk = 0; kk < DI / 32; ++kk) {
                // K = 32 bytes per MMA = two core matrices along K
                const uint64_t ad = tc::desc_noswizzle(a_addr + kk * 256, 128, 8 * DI);
                const uint64_t bd = tc::desc_noswizzle(b_addr + kk * 256, 128, 8 * DI);
                tc::mma_i8(tmem, ad, bd, IDESC, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(bar);
        }
        if (kt + 1 < n_tiles) load_a(kt + 1);                  // other buffer: its MMA is done
        if (!tc::mbar_wait_bounded(bar, kt & 1, TC_WAIT_CYCLES)) {
            timed_out = true;
            raise_error(p.err, ERR_TIMEOUT);
            break;
        }
        tc::fence_after_sync();

        // epilogue: this thread's key row, every query of the tile
        const int j = j_cta + kt * 128 + warp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < NCOL; c0 += 16) {
            uint32_t r[16];
            tc::tmem_ld16(trow + c0, r);
            tc::tmem_ld_wait();
            if constexpr (HI >= 16) {
                // one query spans HI/16 loads: accumulate into the first
                int sc = 0;
#pragma unroll
                for (int u = 0; u < 16; ++u) sc += w_s[c0 + u] * max((int)r[u], 0);
                const int q = c0 / HI;
                const int tq = tq0 + q;
                // HI == 16: exactly one load per query
                if (tq <= tq_last && (long long)j < n_candidates(p.q_pos0 + tq, p.window))
                    p.scores[((long long)b * p.Rt + (tq - p.t0)) * p.ld + j] = sc;
            } else {
#pragma unroll
                for (int qq = 0; qq < 16 / HI; ++qq) {
                    int sc = 0;
#pragma unroll
                    for (int h = 0; h < HI; ++h) sc += w_s[c0 + qq * HI + h] * max((int)r[qq * HI + h], 0);
                    const int tq = tq0 + (c0 / HI) + qq;
                    if (tq <= tq_last && (long long)j < n_candidates(p.q_pos0 + tq, p.window))
                        p.scores[((long long)b * p.Rt + (tq - p.t0)) * p.ld + j] = sc;
                }
            }
        }
        // the next MMA overwrites the accumulator and reads the other A buffer
        tc::fence_before_sync();
        cp_async_wait<0>();
        tc::fence_proxy_async_smem();
        __syncthreads();
        tc::fence_after_sync();
    }
    if (timed_out) {
        cp_async_wait<0>();
        // give the tensor core a bounded chance to finish before freeing TMEM
        tc::mbar_wait_bounded(bar, pending, TC_WAIT_CYCLES / 4);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, NCOL);
}

// ------------------------------------------------------------- top-k select --
struct SelectParams {
    const int32_t *scores;   // [B, Rt, ld]
    long long ld;
    int B, Tq, t0, Rt;
    long long q_pos0;
    int topk, window, Kout;
    int seg_cap;             // bitmap words per row buffer (>= ceil(n/32) for every row)
    int32_t *out_idx;        // [B, Tq, Kout]
    int32_t *out_count;      // [B, Tq] nullable
};

constexpr int SEL_THREADS = 256;
constexpr int SEL_BITS = 12;
constexpr int SEL_BINS = 1 << SEL_BITS;
constexpr int SEL_TIE_CAP = 2048;        // boundary-bin entries resolved from a list
constexpr int SEL_MAX_N = 1 << 20;       // candidates per row (bitmaps of n/8 bytes each)

// Inclusive block scan (sum) of one int per thread; `tmp` holds 32 ints.
__device__ __forceinline__ int block_incl_scan(int v, int *tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) tmp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (int)(blockDim.x >> 5) ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        tmp[lane] = w;
    }
    __syncthreads();
    const int add = warp > 0 ? tmp[warp - 1] : 0;
    __syncthreads();
    return v + add;
}

__device__ __forceinline__ int block_sum(int v, int *tmp) {
    v = warp_sum_int(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) tmp[warp] = v;
    __syncthreads();
    int t = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += tmp[i];
    return t;
}

// Streams the row [0, n) from global memory (L2) with 16-byte loads, U
// vectors in flight per thread; f(value, index) is called for every element.
template <typename F>
__device__ __forceinline__ void stream_row(const int32_t *row, int n, F f) {
    constexpr int U = 4;
    const int n4 = n / 4;
    const int4 *r4 = reinterpret_cast<const int4 *>(row);
    for (int b4 = threadIdx.x; b4 < n4; b4 += SEL_THREADS * U) {
        int4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = b4 + u * SEL_THREADS;
            if (i < n4) v[u] = __ldg(r4 + i);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = b4 + u * SEL_THREADS;
            if (i < n4) {
                f(v[u].x, 4 * i); f(v[u].y, 4 * i + 1); f(v[u].z, 4 * i + 2); f(v[u].w, 4 * i + 3);
            }
        }
    }
    for (int i = n4 * 4 + (int)threadIdx.x; i < n; i += SEL_THREADS) f(__ldg(row + i), i);
}

// Exact top-k of one row, one CTA.  Keys are u = score - row_min (32-bit,
// unsigned order = score order).  The boundary key is found by histogram
// passes over the row: a 4096-bin histogram of u >> shift; the bin holding
// the k-th largest key is refined until its width is 1 or it holds at most
// SEL_TIE_CAP elements, which are then resolved exactly in shared memory.
// Keys above the threshold go to a "greater" bitmap, keys equal to it to an
// "equal" bitmap; the output takes every greater key and the lowest-index
// equal keys, in ascending position order.
__global__ void __launch_bounds__(SEL_THREADS) topk_select_kernel(const SelectParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    int *hist = reinterpret_cast<int *>(smem);                        // [SEL_BINS]
    unsigned *tie_key = reinterpret_cast<unsigned *>(hist + SEL_BINS);  // [SEL_TIE_CAP]
    int *tie_idx = reinterpret_cast<int *>(tie_key + SEL_TIE_CAP);     // [SEL_TIE_CAP]
    unsigned *gt_bm = reinterpret_cast<unsigned *>(tie_idx + SEL_TIE_CAP);  // [words]
    const int words_cap = p.seg_cap;                                     // bitmap words
    unsigned *eq_bm = gt_bm + words_cap;
    __shared__ int scan_tmp[32];
    __shared__ int bcast[4];
    __shared__ int tie_n;

    const int b = blockIdx.z, tr = blockIdx.y, t = p.t0 + tr;
    if (t >= p.Tq || tr >= p.Rt) return;
    const long long pos = p.q_pos0 + t;
    const int n = (int)n_candidates(pos, p.window);
    const int wc = p.window > 0 ? (int)(pos + 1 < p.window ? pos + 1 : p.window) : 0;
    const int k_eff = n < p.topk ? n : p.topk;
    int32_t *orow = p.out_idx + ((long long)b * p.Tq + t) * p.Kout;
    const int32_t *srow = p.scores + ((long long)b * p.Rt + tr) * p.ld;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // window entries, padding and count
    for (int i = tid; i < p.Kout - k_eff; i += SEL_THREADS)
        orow[k_eff + i] = i < wc ? (int)(pos - wc + 1 + i) : -1;
    if (tid == 0 && p.out_count) p.out_count[(long long)b * p.Tq + t] = k_eff + wc;
    if (k_eff == n) {                                 // every candidate is kept
        for (int j = tid; j < n; j += SEL_THREADS) orow[j] = j;
        return;
    }
    if (k_eff == 0) return;

    // 1. row min / max
    int vmin = INT_MAX, vmax = INT_MIN;
    stream_row(srow, n, [&](int v, int) { vmin = min(vmin, v); vmax = max(vmax, v); });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
        vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (tid == 0) { bcast[0] = INT_MAX; bcast[1] = INT_MIN; }
    __syncthreads();
    if (lane == 0) { atomicMin(&bcast[0], vmin); atomicMax(&bcast[1], vmax); }
    __syncthreads();
    const int gmin = bcast[0];
    const unsigned range = (unsigned)bcast[1] - (unsigned)gmin;
    const int nbits = range == 0 ? 0 : 32 - __clz(range);

    // 2. histogram refinement: [lo_key, lo_key + 2^width) holds the k-th key
    unsigned lo_key = 0;
    int width = nbits;                // bits still undetermined
    int k_rem = k_eff;                // keys to take at or below lo_key's bin
    int bin_count = n;                // elements inside the current bin
    while (width > 0 && (width > SEL_BITS || bin_count > SEL_TIE_CAP)) {
        const int shift = width > SEL_BITS ? width - SEL_BITS : 0;
        for (int i = tid; i < SEL_BINS; i += SEL_THREADS) hist[i] = 0;
        __syncthreads();
        const unsigned hi_key = lo_key + (width >= 32 ? 0xffffffffu : ((1u << width) - 1u));
        stream_row(srow, n, [&](int v, int) {
            const unsigned key = (unsigned)v - (unsigned)gmin;
            if (key >= lo_key && key <= hi_key) atomicAdd(&hist[(key - lo_key) >> shift], 1);
        });
        __syncthreads();
        constexpr int per = SEL_BINS / SEL_THREADS;   // bins per thread, highest first
        int cntb[per];
        int local = 0;
#pragma unroll
        for (int u = 0; u < per; ++u) {
            cntb[u] = hist[SEL_BINS - 1 - (tid * per + u)];
            local += cntb[u];
        }
        const int incl = block_incl_scan(local, scan_tmp);
        int above = incl - local;
#pragma unroll
        for (int u = 0; u < per; ++u) {
            const int bin = SEL_BINS - 1 - (tid * per + u);
            if (above < k_rem && above + cntb[u] >= k_rem) {
                bcast[2] = bin;
                bcast[3] = above;
            }
            above += cntb[u];
        }
        __syncthreads();
        const int bin = bcast[2];
        k_rem -= bcast[3];
        bin_count = hist[bin];
        lo_key += (unsigned)bin << shift;
        width = shift;
        __syncthreads();
    }

    // 3. filter pass: bitmaps of keys above the bin; the bin's own elements
    //    go to the equal bitmap (width 0) or to the tie list
    const int words = (n + 31) / 32;
    for (int i = tid; i < words; i += SEL_THREADS) { gt_bm[i] = 0u; eq_bm[i] = 0u; }
    if (tid == 0) tie_n = 0;
    __syncthreads();
    const unsigned bin_hi = lo_key + (width >= 32 ? 0xffffffffu : ((1u << width) - 1u));
    stream_row(srow, n, [&](int v, int j) {
        const unsigned key = (unsigned)v - (unsigned)gmin;
        if (key > bin_hi) {
            atomicOr(&gt_bm[j >> 5], 1u << (j & 31));
        } else if (key >= lo_key) {
            if (width == 0) {
                atomicOr(&eq_bm[j >> 5], 1u << (j & 31));
            } else {
                const int slot = atomicAdd(&tie_n, 1);
                if (slot < SEL_TIE_CAP) { tie_key[slot] = key - lo_key; tie_idx[slot] = j; }
            }
        }
    });
    __syncthreads();
    // 4. resolve the tie list: exact threshold inside the bin (width <= 12 bits)
    if (width > 0) {
        const int m = min(tie_n, SEL_TIE_CAP);
        for (int i = tid; i < SEL_BINS; i += SEL_THREADS) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < m; i += SEL_THREADS) atomicAdd(&hist[tie_key[i]], 1);
        __syncthreads();
        constexpr int per = SEL_BINS / SEL_THREADS;
        int cntb[per];
        int local = 0;
#pragma unroll
        for (int u = 0; u < per; ++u) {
            cntb[u] = hist[SEL_BINS - 1 - (tid * per + u)];
            local += cntb[u];
        }
        const int incl = block_incl_scan(local, scan_tmp);
        int above = incl - local;
#pragma unroll
        for (int u = 0; u < per; ++u) {
            const int bin = SEL_BINS - 1 - (tid * per + u);
            if (above < k_rem && above + cntb[u] >= k_rem) {
                bcast[2] = bin;
                bcast[3] = above;
            }
            above += cntb[u];
        }
        __syncthreads();
        const unsigned thr_off = (unsigned)bcast[2];
        k_rem -= bcast[3];
        for (int i = tid; i < m; i += SEL_THREADS) {
            const int j = tie_idx[i];
            if (tie_key[i] > thr_off) atomicOr(&gt_bm[j >> 5], 1u << (j & 31));
            else if (tie_key[i] == thr_off) atomicOr(&eq_bm[j >> 5], 1u << (j & 31));
        }
        __syncthreads();
    }

    // 5. ordered output: warps own contiguous word ranges
    constexpr int NW = SEL_THREADS / 32;
    const int wpw = (words + NW - 1) / NW;
    const int w_lo = min(warp * wpw, words), w_hi = min(w_lo + wpw, words);
    int gcnt = 0, ecnt = 0;
    for (int i = w_lo + lane; i < w_hi; i += 32) { gcnt += __popc(gt_bm[i]); ecnt += __popc(eq_bm[i]); }
    gcnt = warp_sum_int(gcnt);
    ecnt = warp_sum_int(ecnt);
    __shared__ int wg[NW], we[NW];
    if (lane == 0) { wg[warp] = gcnt; we[warp] = ecnt; }
    __syncthreads();
    int g_before = 0, e_before = 0;
    for (int i = 0; i < warp; ++i) { g_before += wg[i]; e_before += we[i]; }
    int out_base = g_before + min(e_before, k_rem);
    const unsigned lt = (1u << lane) - 1u;
    for (int i0 = w_lo; i0 < w_hi; i0 += 32) {
        const int i = i0 + lane;
        const unsigned gw = i < w_hi ? gt_bm[i] : 0u;
        const unsigned ew = i < w_hi ? eq_bm[i] : 0u;
        // equal keys are taken in index order until k_rem are used
        const int ec = __popc(ew);
        int e_incl = ec;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, e_incl, o);
            if (lane >= o) e_incl += x;
        }
        const int e_pre = e_before + e_incl - ec;           // equal keys before this word
        int take = k_rem - e_pre;
        take = take < 0 ? 0 : (take > ec ? ec : take);
        unsigned em = 0u, rest = ew;
        for (int c = 0; c < take; ++c) { const unsigned lowbit = rest & (~rest + 1u); em |= lowbit; rest ^= lowbit; }
        const unsigned sw = gw | em;
        const int sc = __popc(sw);
        int s_incl = sc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, s_incl, o);
            if (lane >= o) s_incl += x;
        }
        int slot = out_base + s_incl - sc;
        unsigned bits = sw;
        while (bits) {
            const int bpos = __ffs(bits) - 1;
            bits &= bits - 1u;
            if (slot < k_eff) orow[slot] = i * 32 + bpos;   // slot < k_eff by construction
            ++slot;
        }
        out_base += __shfl_sync(0xffffffffu, s_incl, 31);
        e_before += __shfl_sync(0xffffffffu, e_incl, 31);
    }
    (void)lt;
}

}  // namespace sa
