// indexer.cuh -- lightweight-indexer scores and exact causal top-k.
//
// IndexCache page ("IndexCache: inferencia 82% mas rapida ...", body): a
// lightweight indexer scores every earlier token and each query keeps a small
// top-scoring subset.  HySparse2 page ("Xiaomi presenta HySparse2 ...",
// section "Mas precision con menos memoria"): the most recent tokens are
// forced into the set.  Score of query t for key j:
//   I(t, j) = sum_h w[t,h] * max(0, q_idx[t,h,:] . k_idx[j,:])   (exact int32)
// Selection: the top-k candidates j (non-window, j <= position) by
// (I desc, j asc), output in ascending position order, then the window.
//
// Pipeline (per chunk of query rows):
//  1. idx_score_tc_kernel<SAMPLE>: tcgen05 int8 scores of every query against
//     a strided subset of its candidates (about SAMPLE_TARGET keys; all of
//     them when the row is short).
//  2. idx_threshold_kernel: per row, a value tau from the sample chosen so
//     that about k + 4 sigma candidates are expected to reach it (the exact
//     k-th largest score when the sample is the whole row).
//  3. idx_score_tc_kernel<FILTER>: tcgen05 scores of every (query, candidate);
//     the epilogue appends (score, j) with score >= tau to the row's list.
//  4. topk_select_kernel: exact top-k of the list.  If the list holds fewer
//     than k entries or overflowed, the row is recomputed exactly on CUDA
//     cores inside the same kernel, so the result never depends on the
//     sample.  Ties at the k-th score go to the lowest positions.
#pragma once

#include <climits>

#include "sa_common.cuh"
#include "tc_common.cuh"

namespace sa {

constexpr int SAMPLE_TARGET = 2048;       // sampled keys per row (stride = n / target)
constexpr double SAMPLE_Z = 4.5;          // safety margin of the sampled threshold, in sigmas

struct IdxParams {
    const int8_t *q;       // [B, Tq, Hi, DI]
    const int8_t *k;       // [B, L, DI]
    const int32_t *w;      // [B, Tq, Hi]
    int B, Tq, L, Hi, di;
    long long q_pos0;
    int window, topk, Kout;
    int t0, Rt;            // chunk: query rows t0 .. t0+Rt-1 of every batch element
    int nq_block;          // queries per score CTA (fixes the sample stride of a block)
    int m_cap;             // sample buffer row width
    int32_t *sample;       // [B, Rt, m_cap]
    int32_t *tau;          // [B, Rt]
    int cand_cap;          // candidate list capacity per row
    int2 *cand;            // [B, Rt, cand_cap] (score, key position) pairs
    int32_t *cand_cnt;     // [B, Rt]  (zeroed before the filter pass)
    int32_t *out_idx;      // [B, Tq, Kout]
    int32_t *out_count;    // [B, Tq] nullable
    unsigned *err;         // device error word
    const int32_t *dense;  // select's dense mode: [B, Rt, dense_stride] scores (non-negative)
    long long dense_stride;
};

// Number of selectable (non-window) candidates of a query at position p.
__device__ __forceinline__ long long n_candidates(long long p, int window) {
    long long n = window > 0 ? p - window + 1 : p + 1;
    return n > 0 ? n : 0;
}

// Sample stride shared by the query block that starts at row tq0.
__device__ __forceinline__ int sample_stride(const IdxParams &p, int tq0) {
    const long long n0 = n_candidates(p.q_pos0 + tq0, p.window);
    const long long s = n0 / SAMPLE_TARGET;
    return s < 1 ? 1 : (int)min(s, (long long)INT_MAX);
}

// ------------------------------------------------- tcgen05 score kernel --
// Tensor-core (tcgen05, kind::i8) score GEMM.  CTA tile: M = 128 keys (TMEM
// lanes) x N = NCOL (query, head) columns (NCOL/HI queries) x K = DI; the
// accumulator lives in max(NCOL, 32) TMEM columns.  Operands are staged in
// the K-major no-swizzle core-matrix layout: 8-row group r8 at r8 * 8*DI
// bytes, inside it the DI/16 core matrices (8 rows x 16 B) back to back, so
// LBO = 128 B (next core along K) and SBO = 8*DI (next 8-row group).
// 16 warps (8 when NCOL < 64): warp w reads TMEM lane quadrant w % 4 (one key
// row per thread) over part w / 4 of the columns.
// When every head weight of the tile is >= 0 and every w*q fits int8, the
// weights are folded into the query operand (w*relu(x) = relu(w*x)), so the
// epilogue is a plain sum of ReLUs; otherwise it multiplies by w itself.
constexpr int TC_KT = 16;                // 128-key tiles per CTA (amortises the query-tile setup)
// threads of a score CTA: 4 column parts of 4 warps, or 2 parts when the
// tile has fewer than 64 columns
__host__ __device__ constexpr int tc_threads(int ncol) { return ncol >= 64 ? 512 : 256; }
constexpr long long TC_WAIT_CYCLES = 4000000000LL;   // ~2 s: drain wait for the MMA in flight
enum : int { MODE_SAMPLE = 0, MODE_FILTER = 1 };

__device__ __forceinline__ int tc_core_off(int row, int chunk, int di) {
    return (row >> 3) * (8 * di) + chunk * 128 + (row & 7) * 16;
}

// Key tiles are staged through a ring of TC_AS buffers (TC_AS - 1 in flight).
constexpr int TC_AS = 4;

// Filter pass with at most TC_LIST_NQ queries per CTA: the kept (score, key)
// pairs of a tile go to per-query lists in shared memory (double-buffered,
// TC_LCAP = 128 entries = one tile's keys, so they cannot overflow) and are
// copied to the global lists one tile later, with one global atomic per
// (query, tile) whose latency hides behind the next tile's epilogue.
constexpr int TC_LIST_NQ = 32;
constexpr int TC_LCAP = 128;
template <int HI, int NCOL, int MODE>
__host__ __device__ constexpr bool tc_lists() {
    return MODE == 1 && NCOL / HI <= TC_LIST_NQ;
}
template <int HI, int NCOL>
__host__ __device__ constexpr int tc_list_bytes() {
    return (3 * (NCOL / HI) * 4 + 2 * (NCOL / HI) * TC_LCAP * 5 + 15) / 16 * 16;
}

// Shared memory of one score CTA; at least 80 KB for NCOL = 256 so that at
// most two CTAs (2 x 256 TMEM columns) share an SM.
template <int HI, int DI, int NCOL, int MODE>
__host__ __device__ constexpr int tc_smem_bytes() {
    return (NCOL >= 256 &&
            TC_AS * 128 * DI + NCOL * DI + NCOL * 8 + 64 + (tc_lists<HI, NCOL, MODE>() ? tc_list_bytes<HI, NCOL>() : 0) <
                80 * 1024)
               ? 80 * 1024
               : TC_AS * 128 * DI + NCOL * DI + NCOL * 8 + 64 +
                     (tc_lists<HI, NCOL, MODE>() ? tc_list_bytes<HI, NCOL>() : 0);
}

// S + max(x, 0) as one add-then-max: max(S + x, S).
__device__ __forceinline__ int add_relu(int S, int x) { return __viaddmax_s32(S, x, S); }

template <int HI, int DI, int NCOL, int MODE>
__global__ void __launch_bounds__(tc_threads(NCOL), NCOL >= 64 ? 2 : 4) idx_score_tc_kernel(const IdxParams p) {
    grid_dependency_sync();
    constexpr int TC_THREADS = tc_threads(NCOL);
    constexpr int PARTS = TC_THREADS / 128;  // column parts (4 warps each)
    constexpr int NQ = NCOL / HI;            // queries per CTA
    constexpr int CH = DI / 16;              // 16-byte chunks per row
    constexpr int A_BYTES = 128 * DI;
    constexpr int B_BYTES = NCOL * DI;
    constexpr int TCOLS = NCOL < 32 ? 32 : NCOL;
    constexpr int HALF = NCOL / PARTS;       // columns per warp
    constexpr int STEP = HALF < 16 ? HALF : 16;
    static_assert(NCOL % 16 == 0 && NCOL >= 16 && NCOL <= 256 && NCOL % HI == 0, "NCOL");
    static_assert(HI <= STEP, "the heads of a query must lie within one step of one warp");
    static_assert(HALF >= 16 || PARTS == 2, "16-column tiles use two column parts");
    constexpr bool LISTS = tc_lists<HI, NCOL, MODE>();
    static_assert(TC_AS * A_BYTES + B_BYTES + NCOL * 8 + 64 + (LISTS ? tc_list_bytes<HI, NCOL>() : 0) <=
                      tc_smem_bytes<HI, DI, NCOL, MODE>(), "smem");
    constexpr int NWARPS = TC_THREADS / 32;
    constexpr uint32_t IDESC = tc::make_idesc(2 /*s32*/, 1 /*s8*/, 128, NCOL);

    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *a_s = smem;                               // TC_AS x A tile
    unsigned char *b_s = smem + TC_AS * A_BYTES;             // B tile
    int *w_s = reinterpret_cast<int *>(b_s + B_BYTES);       // [NCOL]
    int *tau_s = w_s + NCOL;                                 // [NQ] (filter mode)
    uint64_t *bar = reinterpret_cast<uint64_t *>(tau_s + NCOL);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
    int *fold_bad = reinterpret_cast<int *>(tmem_slot + 1);
    int *wait_ok = fold_bad + 1;
    // per-query tile lists (filter pass): counts [2][NQ], global bases [NQ],
    // scores [2][NQ][TC_LCAP], key offsets within the tile [2][NQ][TC_LCAP]
    int *lcnt_s = reinterpret_cast<int *>(smem + TC_AS * A_BYTES + B_BYTES + NCOL * 8 + 64);
    int *lbase_s = lcnt_s + 2 * NQ;
    int *lval_s = lbase_s + NQ;
    uint8_t *loff_s = reinterpret_cast<uint8_t *>(lval_s + 2 * NQ * TC_LCAP);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z;
    const int tq0 = p.t0 + blockIdx.y * NQ;
    const int t_last = min(p.t0 + p.Rt, p.Tq) - 1;
    const int tq_last = min(tq0 + NQ - 1, t_last);
    if (tq0 > t_last) return;
    const long long ncand_last = n_candidates(p.q_pos0 + tq_last, p.window);
    // key position of tile row r: j = stride * (j_cta + r)
    const int stride = MODE == MODE_SAMPLE ? sample_stride(p, tq0) : 1;
    const long long n_keys = MODE == MODE_SAMPLE ? (ncand_last + stride - 1) / stride : ncand_last;
    const int j_cta = blockIdx.x * TC_KT * 128;
    if ((long long)j_cta >= n_keys) return;                  // nothing left for this block (uniform)
    const int n_tiles = (int)min((long long)TC_KT, (n_keys - j_cta + 127) / 128);

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TCOLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_fence_init();
        *fold_bad = 0;
    }
    for (int i = tid; i < NCOL; i += TC_THREADS) {
        const int tq = tq0 + i / HI;
        w_s[i] = tq <= tq_last ? __ldg(p.w + ((long long)b * p.Tq + tq) * HI + i % HI) : 0;
    }
    if (MODE == MODE_FILTER) {
        for (int i = tid; i < NQ; i += TC_THREADS) {
            const int tq = tq0 + i;
            tau_s[i] = tq <= tq_last ? p.tau[(long long)b * p.Rt + (tq - p.t0)] : INT_MAX;
        }
    }
    if constexpr (LISTS) {
        for (int i = tid; i < 2 * NQ; i += TC_THREADS) lcnt_s[i] = 0;
    }
    __syncthreads();
    // B tile (rows (q, h) of q_idx are contiguous in memory), weights folded in
    // when that is exact
    const int8_t *qsrc = p.q + (((long long)b * p.Tq + tq0) * HI) * DI;
    const int nrows_valid = (tq_last - tq0 + 1) * HI;
    for (int i = tid; i < NCOL * CH; i += TC_THREADS) {
        const int row = i / CH, c = i % CH;
        int4 v = make_int4(0, 0, 0, 0);
        if (row < nrows_valid) v = __ldg(reinterpret_cast<const int4 *>(qsrc + (long long)row * DI + c * 16));
        const int wv = w_s[row];
        int bad = wv < 0;
        int words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            unsigned packed = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int x = (int)(signed char)((words[u] >> (8 * e)) & 0xff) * wv;
                bad |= (x < -128) | (x > 127);
                packed |= ((unsigned)x & 0xffu) << (8 * e);
            }
            words[u] = (int)packed;
        }
        if (bad) atomicOr(fold_bad, 1);
        *reinterpret_cast<int4 *>(b_s + tc_core_off(row, c, DI)) = make_int4(words[0], words[1], words[2], words[3]);
    }
    __syncthreads();
    const bool fold = *fold_bad == 0;
    if (!fold) {   // exact path: plain q, weights applied in the epilogue
        for (int i = tid; i < NCOL * CH; i += TC_THREADS) {
            const int row = i / CH, c = i % CH;
            int4 v = make_int4(0, 0, 0, 0);
            if (row < nrows_valid) v = __ldg(reinterpret_cast<const int4 *>(qsrc + (long long)row * DI + c * 16));
            *reinterpret_cast<int4 *>(b_s + tc_core_off(row, c, DI)) = v;
        }
    }
    auto load_a = [&](int kt) {   // always commits a group (empty past the last tile)
        if (kt < n_tiles) {
            unsigned char *dst = a_s + (kt % TC_AS) * A_BYTES;
            const int i0 = j_cta + kt * 128;
            const int8_t *src = p.k + ((long long)b * p.L) * DI;
            for (int i = tid; i < 128 * CH; i += TC_THREADS) {
                const int row = i / CH, c = i % CH;
                const long long j = (long long)stride * (i0 + row);
                const bool ok = j < p.L;
                cp_async16(dst + tc_core_off(row, c, DI), ok ? src + j * DI + c * 16 : src, ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int s = 0; s < TC_AS - 1; ++s) load_a(s);
    cp_async_wait<TC_AS - 2>();                              // tile 0 has landed
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const int quad = warp & 3;                     // TMEM lane quadrant of this warp
    const int c_begin = (warp >> 2) * HALF;        // this warp's part of the columns
    // per-query constants of this warp's queries, held in registers: the
    // number of candidates (keys j < nt_q are scored) and the threshold
    constexpr int NQH = HALF / HI;                 // queries in this warp's half
    constexpr int GQ = NQH < 32 ? NQH : 32;        // queries per append group
    int nt_r[GQ], tau_r[GQ];
    auto load_query_consts = [&](int g0) {
#pragma unroll
        for (int q = 0; q < GQ; ++q) {
            const int tq = tq0 + c_begin / HI + g0 + q;
            const long long nt = tq <= tq_last ? n_candidates(p.q_pos0 + tq, p.window) : 0;
            nt_r[q] = (int)min(nt, (long long)INT_MAX);
            tau_r[q] = MODE == MODE_FILTER ? tau_s[c_begin / HI + g0 + q] : 0;
        }
    };
    if (NQH == GQ) load_query_consts(0);
    // Filter-pass lists: global row of CTA query q, and the copy of tile kt's
    // shared list (buffer kt & 1) to the global list at the base reserved
    // for it; each query's list is copied and then cleared by warp q % NWARPS.
    auto list_row = [&](int q) -> long long { return (long long)b * p.Rt + (tq0 + q - p.t0); };
    auto copy_lists = [&](int kt_done) {
        const int buf = kt_done & 1;
        const int key0 = j_cta + kt_done * 128;
        for (int q = warp; q < NQ; q += NWARPS) {
            const int n = lcnt_s[buf * NQ + q];
            if (n == 0) continue;                              // warp-uniform
            const int base = lbase_s[q];
            const long long roff = list_row(q) * p.cand_cap;
            for (int e = lane; e < n; e += 32) {
                const int slot = base + e;
                if (slot < p.cand_cap) {
                    p.cand[roff + slot] = make_int2(lval_s[(buf * NQ + q) * TC_LCAP + e],
                                                    key0 + loff_s[(buf * NQ + q) * TC_LCAP + e]);
                }
            }
            __syncwarp();
            if (lane == 0) lcnt_s[buf * NQ + q] = 0;
        }
    };
    // one global atomic per (query, tile): lane q of warp 0 reserves room for
    // tile kt_done's list of query q and returns the base
    auto reserve_lists = [&](int kt_done) -> int {
        int base = 0;
        if (lane < NQ) {
            const int n = lcnt_s[(kt_done & 1) * NQ + lane];
            if (n > 0) base = atomicAdd(p.cand_cnt + list_row(lane), n);
        }
        return base;
    };

    bool timed_out = false;
    uint32_t pending = 0;   // parity of the MMA batch in flight
    for (int kt = 0; kt < n_tiles; ++kt) {
        pending = kt & 1;
        if (tid == 0) {
            const uint32_t a_addr = tc::smem_u32(a_s + (kt % TC_AS) * A_BYTES);
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
        int list_base = 0;                                     // warp 0: bases for tile kt-1
        if (LISTS && warp == 0 && kt > 0) list_base = reserve_lists(kt - 1);
        load_a(kt + TC_AS - 1);                                // buffer of tile kt-1: its MMA is done
        // one thread waits (bounded) and the whole CTA follows its verdict
        if (tid == 0) *wait_ok = tc::mbar_wait_bounded(bar, kt & 1, spin_limit()) ? 1 : 0;
        __syncthreads();
        if (*wait_ok == 0) {
            timed_out = true;
            if (tid == 0) raise_error(p.err, ERR_TIMEOUT);
            break;
        }
        tc::fence_after_sync();

        // epilogue: this thread's key row, the queries of its column half,
        // in groups of up to 32 queries so that the list appends of a whole
        // group go out as one warp-wide atomic (one lane per query)
        const int i_key = j_cta + kt * 128 + quad * 32 + lane;       // tile row -> key index
        const long long j = (long long)stride * i_key;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        constexpr int QPL = HI >= STEP ? 1 : STEP / HI;  // queries per TMEM load
        constexpr int HPL = HI >= STEP ? STEP : HI;      // heads of a query in a load
#pragma unroll 1
        for (int g0 = 0; g0 < NQH; g0 += GQ) {
            if (NQH != GQ) load_query_consts(g0);
            int sc[GQ];
#pragma unroll
            for (int c = 0; c < GQ * HI; c += STEP) {
                uint32_t r[16];
                // a load covers 16 columns; with NCOL == 16 both halves read the
                // same load and keep their own 8 columns
                tc::tmem_ld16(trow + (HALF >= 16 ? c_begin + g0 * HI + c : 0), r);
                tc::tmem_ld_wait();
                if constexpr (HALF < 16) {
                    if (warp >> 2) {
#pragma unroll
                        for (int h = 0; h < HALF; ++h) r[h] = r[HALF + h];
                    }
                }
#pragma unroll
                for (int qq = 0; qq < QPL; ++qq) {
                    int v = 0;
                    if (fold) {
#pragma unroll
                        for (int h = 0; h < HPL; ++h) v = add_relu(v, (int)r[qq * HPL + h]);
                    } else {
                        const int cw = c_begin + g0 * HI + c + qq * HPL;
#pragma unroll
                        for (int h = 0; h < HPL; ++h) v += w_s[cw + h] * max((int)r[qq * HPL + h], 0);
                    }
                    sc[c / HI + qq] = v;
                }
            }
            const int q_first = c_begin / HI + g0;      // query index (within the CTA) of sc[0]
            const int row0 = b * p.Rt + (tq0 + q_first - p.t0);   // list row of sc[0]
            const int jj = (int)min(j, (long long)INT_MAX);
            if constexpr (MODE == MODE_SAMPLE) {
#pragma unroll
                for (int q = 0; q < GQ; ++q)
                    if (jj < nt_r[q]) p.sample[(long long)(row0 + q) * p.m_cap + i_key] = sc[q];
            } else if constexpr (LISTS) {
                // kept pairs go to this tile's shared list of their query
                const int buf = kt & 1;
                // causal test j < n_candidates(position of query q) as dd < q;
                // queries past the chunk have tau = INT_MAX
                const long long ddl = j + (p.window > 0 ? p.window : 0) - 1 - (p.q_pos0 + tq0 + q_first);
                const int dd = (int)max(min(ddl, (long long)GQ), -1LL);
#pragma unroll
                for (int q = 0; q < GQ; ++q) {
                    if ((dd < q) & (sc[q] >= tau_r[q])) {
                        const int lq = buf * NQ + q_first + q;
                        const int slot = atomicAdd(lcnt_s + lq, 1);
                        lval_s[lq * TC_LCAP + slot] = sc[q];
                        loff_s[lq * TC_LCAP + slot] = (uint8_t)(quad * 32 + lane);
                    }
                }
            } else {
                unsigned ball[GQ];
                unsigned keepm = 0u;
                int mycnt = 0;
#pragma unroll
                for (int q = 0; q < GQ; ++q) {
                    const bool keep = (jj < nt_r[q]) & (sc[q] >= tau_r[q]);
                    keepm |= keep ? (1u << q) : 0u;
                    ball[q] = __ballot_sync(0xffffffffu, keep);
                    mycnt = lane == q ? __popc(ball[q]) : mycnt;
                }
                int base = 0;
                if (mycnt > 0) base = atomicAdd(p.cand_cnt + row0 + lane, mycnt);   // lane q < GQ
                const unsigned lt = (1u << lane) - 1u;
#pragma unroll
                for (int q = 0; q < GQ; ++q) {
                    if (ball[q] == 0u) continue;                           // warp-uniform
                    const int slot = __shfl_sync(0xffffffffu, base, q) + __popc(ball[q] & lt);
                    if (((keepm >> q) & 1u) && slot < p.cand_cap) {
                        const long long off = (long long)(row0 + q) * p.cand_cap + slot;
                        p.cand[off] = make_int2(sc[q], jj);
                    }
                }
            }
        }
        if (LISTS && warp == 0 && kt > 0 && lane < NQ) lbase_s[lane] = list_base;
        // the next MMA overwrites the accumulator and reads tile kt+1's buffer
        tc::fence_before_sync();
        cp_async_wait<TC_AS - 2>();
        tc::fence_proxy_async_smem();
        __syncthreads();
        tc::fence_after_sync();
        if (LISTS && kt > 0) copy_lists(kt - 1);
    }
    if (LISTS && !timed_out) {                                 // the last tile's lists
        const int base = warp == 0 ? reserve_lists(n_tiles - 1) : 0;
        __syncthreads();                                       // tile n_tiles-2's copies are done
        if (warp == 0 && lane < NQ) lbase_s[lane] = base;
        __syncthreads();
        copy_lists(n_tiles - 1);
    }
    if (timed_out) {
        cp_async_wait<0>();
        // give the tensor core a bounded chance to finish before freeing TMEM
        if (tid == 0) tc::mbar_wait_bounded(bar, pending, TC_WAIT_CYCLES / 4);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, TCOLS);
}

// ----------------------------------------------- decode-shaped scores --
// With one or two queries per sequence the score pass is a memory-bound
// matrix-vector product; it runs on CUDA cores (dp4a) so the keys stream at
// HBM bandwidth.  CTA = (b, query row, DEC_KEYS keys); thread = key.
constexpr int DEC_THREADS = 256;
constexpr int DEC_KEYS = 2048;

template <int DI, int MODE>
__global__ void __launch_bounds__(DEC_THREADS) idx_score_dp4a_kernel(const IdxParams p) {
    grid_dependency_sync();
    __shared__ __align__(16) int8_t q_s[16 * DI];
    __shared__ int w_s[16];
    const int b = blockIdx.z, tr = blockIdx.y, t = p.t0 + tr;
    if (t >= p.Tq || tr >= p.Rt) return;
    const long long nt = n_candidates(p.q_pos0 + t, p.window);
    const int stride = MODE == MODE_SAMPLE ? sample_stride(p, t) : 1;     // query blocks of one
    const long long n_keys = MODE == MODE_SAMPLE ? (nt + stride - 1) / stride : nt;
    const long long i0 = (long long)blockIdx.x * DEC_KEYS;
    if (i0 >= n_keys) return;
    const int tid = threadIdx.x, lane = tid & 31;
    const long long row = (long long)b * p.Rt + tr;
    const int8_t *qsrc = p.q + ((long long)b * p.Tq + t) * p.Hi * DI;
    for (int i = tid; i < p.Hi * DI / 16; i += DEC_THREADS)
        reinterpret_cast<int4 *>(q_s)[i] = __ldg(reinterpret_cast<const int4 *>(qsrc) + i);
    if (tid < p.Hi) w_s[tid] = __ldg(p.w + ((long long)b * p.Tq + t) * p.Hi + tid);
    const int tau = MODE == MODE_FILTER ? p.tau[row] : 0;
    __syncthreads();
    const int8_t *kb = p.k + (long long)b * p.L * DI;
    constexpr int U = 2;                                    // keys per thread in flight
    for (long long base = i0 + tid; base < i0 + DEC_KEYS; base += (long long)DEC_THREADS * U) {
        int4 kv[U][DI / 16];
        long long jj[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = base + (long long)u * DEC_THREADS;
            jj[u] = (long long)stride * i;
            const bool ok = i < n_keys && i < i0 + DEC_KEYS && jj[u] < p.L;
#pragma unroll
            for (int c = 0; c < DI / 16; ++c)
                kv[u][c] = ok ? __ldg(reinterpret_cast<const int4 *>(kb + jj[u] * DI) + c) : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = base + (long long)u * DEC_THREADS;
            const bool ok = i < n_keys && i < i0 + DEC_KEYS && jj[u] < nt;
            int total = 0;
            for (int h = 0; h < p.Hi; ++h) {
                const int4 *qv = reinterpret_cast<const int4 *>(q_s + h * DI);
                int dot = 0;
#pragma unroll
                for (int c = 0; c < DI / 16; ++c) {
                    const int4 a = qv[c];
                    dot = __dp4a(a.x, kv[u][c].x, dot);
                    dot = __dp4a(a.y, kv[u][c].y, dot);
                    dot = __dp4a(a.z, kv[u][c].z, dot);
                    dot = __dp4a(a.w, kv[u][c].w, dot);
                }
                total += w_s[h] * max(dot, 0);
            }
            if constexpr (MODE == MODE_SAMPLE) {
                if (ok) p.sample[row * p.m_cap + i] = total;
            } else {
                const bool keep = ok && total >= tau;
                const unsigned ballot = __ballot_sync(0xffffffffu, keep);
                if (ballot) {
                    int slot0 = 0;
                    if (lane == 0) slot0 = atomicAdd(p.cand_cnt + row, __popc(ballot));
                    const int slot = __shfl_sync(0xffffffffu, slot0, 0) + __popc(ballot & ((1u << lane) - 1u));
                    if (keep && slot < p.cand_cap) {
                        p.cand[row * p.cand_cap + slot] = make_int2(total, (int)jj[u]);
                    }
                }
            }
        }
    }
}

// ------------------------------------- decode-shaped scores, tensor cores --
// One query row and 8 indexer heads of width 64: per 16 keys, two
// mma.sync m16n8k32 (s8 x s8 -> s32) give the 16 x 8 head scores.  The
// contraction index is permuted identically on both operands (a dot product
// does not depend on the order of its terms) so that every thread's share of
// a key row is one contiguous 16-byte load: logical byte s*32 + h*16 + 4c + e
// (MMA slice s, fragment half h, thread quad c) lives at physical byte
// 16c + 8s + 4h + e of the 64-byte row.  A warp's loads cover 8 whole rows
// per instruction.  Kept (score, key) pairs collect in a per-CTA shared list
// and reach the global list with one atomic per CTA.
constexpr int DMMA_THREADS = 256;
constexpr int DMMA_KEYS = 4096;                 // keys per CTA in the filter pass (512 per warp)
constexpr int DMMA_KEYS_SAMPLE = 512;           // sampled keys per CTA (the sample is short)
constexpr int DMMA_U = 4;                       // 16-key groups per warp in flight
__host__ __device__ constexpr int dmma_keys(int mode) { return mode == 0 ? DMMA_KEYS_SAMPLE : DMMA_KEYS; }

template <int MODE>
__global__ void __launch_bounds__(DMMA_THREADS) idx_score_dec_mma_kernel(const IdxParams p) {
    grid_dependency_sync();
    constexpr int DI = 64, HI = 8;
    __shared__ int lcnt_s, lbase_s;
    __shared__ int lval_s[MODE == MODE_FILTER ? DMMA_KEYS : 1];
    __shared__ int lidx_s[MODE == MODE_FILTER ? DMMA_KEYS : 1];
    const int b = blockIdx.z, tr = blockIdx.y, t = p.t0 + tr;
    if (t >= p.Tq || tr >= p.Rt) return;
    const long long nt = n_candidates(p.q_pos0 + t, p.window);
    const int stride = MODE == MODE_SAMPLE ? sample_stride(p, t) : 1;
    const long long n_keys = MODE == MODE_SAMPLE ? (nt + stride - 1) / stride : nt;
    constexpr int KPC = dmma_keys(MODE);
    const long long i0 = (long long)blockIdx.x * KPC;
    if (i0 >= n_keys) return;                                       // uniform
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const long long row = (long long)b * p.Rt + tr;
    if (MODE == MODE_FILTER && tid == 0) lcnt_s = 0;

    // B operand: head n = g, this thread's 16 permuted bytes of q
    const int8_t *qrow = p.q + (((long long)b * p.Tq + t) * HI + g) * DI;
    int4 qv = __ldg(reinterpret_cast<const int4 *>(qrow) + c);
    const int wn = __ldg(p.w + ((long long)b * p.Tq + t) * HI + g);   // weight of head g
    // weights of the two heads whose scores this thread holds (2c, 2c+1)
    const int w0 = __shfl_sync(0xffffffffu, wn, (2 * c) << 2);
    const int w1 = __shfl_sync(0xffffffffu, wn, (2 * c + 1) << 2);
    bool fold_ok = wn >= 0;
    {
        int words[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            unsigned packed = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int x = (int)(signed char)((words[u] >> (8 * e)) & 0xff) * wn;
                fold_ok &= (x >= -128) & (x <= 127);
                packed |= ((unsigned)x & 0xffu) << (8 * e);
            }
            words[u] = (int)packed;
        }
        if (__all_sync(0xffffffffu, fold_ok)) qv = make_int4(words[0], words[1], words[2], words[3]);
        else fold_ok = false;
    }
    const bool fold = __all_sync(0xffffffffu, fold_ok);
    const int tau = MODE == MODE_FILTER ? p.tau[row] : 0;
    if (MODE == MODE_FILTER) __syncthreads();                       // lcnt_s initialised

    const int8_t *kb = p.k + (long long)b * p.L * DI;
    const long long wbeg = i0 + (long long)warp * (KPC / 8);
    const long long wend = min(wbeg + KPC / 8, n_keys);
    for (long long gb = wbeg; gb < wend; gb += 16 * DMMA_U) {
        int4 ka[DMMA_U], kc8[DMMA_U];                               // rows g and g + 8 of each group
#pragma unroll
        for (int u = 0; u < DMMA_U; ++u) {
            const long long ia = gb + 16 * u + g, ib = ia + 8;
            const long long ja = (long long)stride * ia, jb = (long long)stride * ib;
            ka[u] = (ia < wend && ja < p.L) ? __ldg(reinterpret_cast<const int4 *>(kb + ja * DI) + c) : make_int4(0, 0, 0, 0);
            kc8[u] = (ib < wend && jb < p.L) ? __ldg(reinterpret_cast<const int4 *>(kb + jb * DI) + c) : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < DMMA_U; ++u) {
            int acc[4] = {0, 0, 0, 0};
            mma_s8_16832(acc, (unsigned)ka[u].x, (unsigned)kc8[u].x, (unsigned)ka[u].y, (unsigned)kc8[u].y,
                         (unsigned)qv.x, (unsigned)qv.y);
            mma_s8_16832(acc, (unsigned)ka[u].z, (unsigned)kc8[u].z, (unsigned)ka[u].w, (unsigned)kc8[u].w,
                         (unsigned)qv.z, (unsigned)qv.w);
            // acc: (key g, heads 2c, 2c+1), (key g+8, heads 2c, 2c+1)
            int va, vb;
            if (fold) {
                va = max(acc[0], 0) + max(acc[1], 0);
                vb = max(acc[2], 0) + max(acc[3], 0);
            } else {
                va = w0 * max(acc[0], 0) + w1 * max(acc[1], 0);
                vb = w0 * max(acc[2], 0) + w1 * max(acc[3], 0);
            }
            va += __shfl_xor_sync(0xffffffffu, va, 1);
            va += __shfl_xor_sync(0xffffffffu, va, 2);
            vb += __shfl_xor_sync(0xffffffffu, vb, 1);
            vb += __shfl_xor_sync(0xffffffffu, vb, 2);
            const long long ia = gb + 16 * u + g, ib = ia + 8;
            if (c == 0) {
                if constexpr (MODE == MODE_SAMPLE) {
                    if (ia < wend) p.sample[row * p.m_cap + ia] = va;
                    if (ib < wend) p.sample[row * p.m_cap + ib] = vb;
                } else {
                    if (ia < wend && va >= tau) {
                        const int sl = atomicAdd(&lcnt_s, 1);
                        lval_s[sl] = va;
                        lidx_s[sl] = (int)ia;
                    }
                    if (ib < wend && vb >= tau) {
                        const int sl = atomicAdd(&lcnt_s, 1);
                        lval_s[sl] = vb;
                        lidx_s[sl] = (int)ib;
                    }
                }
            }
        }
    }
    if constexpr (MODE == MODE_FILTER) {
        __syncthreads();
        const int n = lcnt_s;
        if (tid == 0) lbase_s = n > 0 ? atomicAdd(p.cand_cnt + row, n) : 0;
        __syncthreads();
        const int base = lbase_s;
        for (int e = tid; e < n; e += DMMA_THREADS) {
            const int slot = base + e;
            if (slot < p.cand_cap) {
                p.cand[row * p.cand_cap + slot] = make_int2(lval_s[e], lidx_s[e]);
            }
        }
    }
}

// ----------------------------------------------------- block helpers --
constexpr int SEL_THREADS = 256;
constexpr int SEL_BITS = 8;
constexpr int SEL_BINS = 1 << SEL_BITS;
constexpr int SEL_TIE_CAP = 2048;        // boundary-bin entries resolved from a list
constexpr int SEL_FINE_BINS = 2 * SEL_TIE_CAP;   // exact-histogram bins (they reuse the tie arrays)
constexpr int SEL_MAX_N = 768 * 1024;    // candidates per row (two bitmaps of n/8 bytes in shared memory)

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

// Radix state of a top-k search over 32-bit keys u = value - vmin: the k-th
// largest key lies in [lo_key, lo_key + 2^width), and k_rem keys still have
// to be taken at or below that bin.
struct RadixState {
    unsigned lo_key;
    int width, k_rem, bin_count;
};

// One histogram refinement step over the keys of the current bin.
// `for_each(f)` calls f(value, position) for every element of the row.
// Block-uniform result.
template <int NT = SEL_THREADS, typename ForEach>
__device__ void radix_refine(RadixState &st, int gmin, int *hist, int *scan_tmp, int *bcast, ForEach for_each) {
    const int tid = threadIdx.x;
    const int shift = st.width > SEL_BITS ? st.width - SEL_BITS : 0;
    for (int i = tid; i < SEL_BINS; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const unsigned lo = st.lo_key;
    const unsigned hi = lo + (st.width >= 32 ? 0xffffffffu : ((1u << st.width) - 1u));
    for_each([&](int v, int) {
        const unsigned key = (unsigned)v - (unsigned)gmin;
        if (key >= lo && key <= hi) atomicAdd(&hist[(key - lo) >> shift], 1);
    });
    __syncthreads();
    constexpr int per = NT >= SEL_BINS ? 1 : SEL_BINS / NT;   // bins per thread, highest first
    int cntb[per];
    int local = 0;
#pragma unroll
    for (int u = 0; u < per; ++u) {
        cntb[u] = tid * per + u < SEL_BINS ? hist[SEL_BINS - 1 - (tid * per + u)] : 0;
        local += cntb[u];
    }
    const int incl = block_incl_scan(local, scan_tmp);
    int above = incl - local;
#pragma unroll
    for (int u = 0; u < per; ++u) {
        const int bin = SEL_BINS - 1 - (tid * per + u);
        if (tid * per + u < SEL_BINS && above < st.k_rem && above + cntb[u] >= st.k_rem) {
            bcast[2] = bin;
            bcast[3] = above;
        }
        above += cntb[u];
    }
    __syncthreads();
    const int bin = bcast[2];
    st.k_rem -= bcast[3];
    st.bin_count = hist[bin];
    st.lo_key += (unsigned)bin << shift;
    st.width = shift;
    __syncthreads();
}

// Block min/max of per-thread partial minima and maxima.
__device__ __forceinline__ void block_minmax_reduce(int vmin, int vmax, int &gmin, int &gmax, int *bcast) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
        vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (threadIdx.x == 0) { bcast[0] = INT_MAX; bcast[1] = INT_MIN; }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) { atomicMin(&bcast[0], vmin); atomicMax(&bcast[1], vmax); }
    __syncthreads();
    gmin = bcast[0];
    gmax = bcast[1];
    __syncthreads();
}

// Block min/max of the values produced by for_each.
template <typename ForEach>
__device__ void block_minmax(int &gmin, int &gmax, int *bcast, ForEach for_each) {
    int vmin = INT_MAX, vmax = INT_MIN;
    for_each([&](int v, int) { vmin = min(vmin, v); vmax = max(vmax, v); });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
        vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (threadIdx.x == 0) { bcast[0] = INT_MAX; bcast[1] = INT_MIN; }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) { atomicMin(&bcast[0], vmin); atomicMax(&bcast[1], vmax); }
    __syncthreads();
    gmin = bcast[0];
    gmax = bcast[1];
    __syncthreads();
}

// Exact k-th largest when every value lies in [gmin, gmin + SEL_FINE_BINS):
// one histogram with a bin per value (fh: SEL_FINE_BINS ints of shared
// memory).  Returns, block-uniform, the k-th largest value's offset from
// gmin and the number of values above it.
// Second half of fine_kth: the k-th largest bin of a filled histogram.
template <int NT>
__device__ void fine_scan(int k, const int *fh, int *scan_tmp, int *bcast, int &bin, int &above_bin) {
    const int tid = threadIdx.x;
    constexpr int PER = SEL_FINE_BINS / NT;               // bins per thread, highest first
    int cb[PER], local = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) { cb[u] = fh[SEL_FINE_BINS - 1 - (tid * PER + u)]; local += cb[u]; }
    const int incl = block_incl_scan(local, scan_tmp);
    int above = incl - local;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        if (above < k && above + cb[u] >= k) {
            bcast[2] = SEL_FINE_BINS - 1 - (tid * PER + u);
            bcast[3] = above;
        }
        above += cb[u];
    }
    __syncthreads();
    bin = bcast[2];
    above_bin = bcast[3];
    __syncthreads();
}
template <int NT, typename ForEach>
__device__ void fine_kth(int k, int gmin, int *fh, int *scan_tmp, int *bcast, ForEach for_each, int &bin,
                         int &above_bin) {
    for (int i = threadIdx.x; i < SEL_FINE_BINS; i += NT) fh[i] = 0;
    __syncthreads();
    for_each([&](int v, int) { atomicAdd(&fh[(unsigned)v - (unsigned)gmin], 1); });
    __syncthreads();
    fine_scan<NT>(k, fh, scan_tmp, bcast, bin, above_bin);
}

// Streams int32 values [0, n) from global memory with 16-byte loads, U vectors
// in flight per thread; f(value, index).  `vals` must be 16-byte aligned.
template <typename F>
__device__ __forceinline__ void stream_values(const int32_t *vals, int n, F f) {
    constexpr int U = 8;
    const int n4 = n / 4;
    const int4 *r4 = reinterpret_cast<const int4 *>(vals);
    for (int b4 = threadIdx.x; b4 < n4; b4 += blockDim.x * U) {
        int4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = b4 + u * blockDim.x;
            if (i < n4) v[u] = __ldg(r4 + i);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = b4 + u * blockDim.x;
            if (i < n4) {
                f(v[u].x, 4 * i); f(v[u].y, 4 * i + 1); f(v[u].z, 4 * i + 2); f(v[u].w, 4 * i + 3);
            }
        }
    }
    for (int i = n4 * 4 + (int)threadIdx.x; i < n; i += blockDim.x) f(__ldg(vals + i), i);
}

// -------------------------------------------------------------- threshold --
// tau of one row from its sample: the r-th largest sampled score, with r
// chosen so that r/m of the n candidates (plus four standard deviations of a
// sampling count) reach it.  A sample that is the whole row gives the exact
// k-th largest score.  Rows whose every candidate is kept get INT_MIN.
__global__ void __launch_bounds__(SEL_THREADS, 4) idx_threshold_kernel(const IdxParams p) {
    grid_dependency_sync();
    __shared__ int hist[SEL_BINS];
    __shared__ int fine[SEL_FINE_BINS];
    __shared__ int scan_tmp[32];
    __shared__ int bcast[4];
    const int b = blockIdx.z, tr = blockIdx.y, t = p.t0 + tr;
    if (t >= p.Tq || tr >= p.Rt) return;
    const long long row = (long long)b * p.Rt + tr;
    if (threadIdx.x == 0) p.cand_cnt[row] = 0;                // the filter pass appends from zero
    const int n = (int)n_candidates(p.q_pos0 + t, p.window);
    const int k_eff = n < p.topk ? n : p.topk;
    if (k_eff == n || k_eff == 0) {
        if (threadIdx.x == 0) p.tau[row] = k_eff == 0 ? INT_MAX : INT_MIN;
        return;
    }
    const int tq0 = p.t0 + ((t - p.t0) / p.nq_block) * p.nq_block;
    const int s = sample_stride(p, tq0);
    const int m = (n + s - 1) / s;                           // sampled keys of this row
    int r;
    if (s == 1) {
        r = k_eff;
    } else {
        // The count of candidates at or above the sample's r-th value is about
        // s*r with a standard deviation of about s*sqrt(r); r = e + z*sqrt(r)
        // keeps it z sigmas above k (e = k/s, the sample rank of the k-th key).
        const double e = (double)k_eff * m / n;
        double rr = e + SAMPLE_Z * sqrt(e) + 2.0;
        rr = e + SAMPLE_Z * sqrt(rr) + 2.0;
        rr = e + SAMPLE_Z * sqrt(rr) + 2.0;
        r = (int)ceil(rr);
        r = min(r, m);
    }
    const int32_t *vals = p.sample + row * p.m_cap;
    auto for_each = [&](auto f) { stream_values(vals, m, f); };
    int gmin, gmax;
    block_minmax(gmin, gmax, bcast, for_each);
    const unsigned range = (unsigned)gmax - (unsigned)gmin;
    if (range < (unsigned)SEL_FINE_BINS) {
        // narrow range: the r-th largest sampled value from one exact histogram
        int bin, above;
        fine_kth<SEL_THREADS>(r, gmin, fine, scan_tmp, bcast, for_each, bin, above);
        if (threadIdx.x == 0) p.tau[row] = (int)((unsigned)gmin + (unsigned)bin);
        return;
    }
    RadixState st{0u, range == 0 ? 0 : 32 - __clz(range), r, m};
    while (st.width > 0) radix_refine(st, gmin, hist, scan_tmp, bcast, for_each);
    if (threadIdx.x == 0) p.tau[row] = (int)((unsigned)gmin + st.lo_key);
}

// Warp-per-row form of idx_threshold_kernel (the default): 8 rows per CTA,
// each warp streams its row's sample from L2 with 16-byte loads, takes the
// range with shuffles, then the r-th largest value by 8-bit radix digits
// from the top (a 256-bin histogram per warp in shared memory, the bin found
// by a suffix scan over the lanes' 8 bins each).  No block barriers, so the
// rows of a CTA proceed independently.
constexpr int THW_WARPS = 8;
__global__ void __launch_bounds__(THW_WARPS * 32) idx_threshold_warp_kernel(const IdxParams p) {
    grid_dependency_sync();
    __shared__ int hist_all[THW_WARPS][SEL_BINS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * THW_WARPS + warp;
    if (row >= (long long)p.B * p.Rt) return;
    const int tr = (int)(row % p.Rt), t = p.t0 + tr;
    if (t >= p.Tq) return;
    int *hist = hist_all[warp];
    if (lane == 0) p.cand_cnt[row] = 0;                       // the filter pass appends from zero
    const int n = (int)n_candidates(p.q_pos0 + t, p.window);
    const int k_eff = n < p.topk ? n : p.topk;
    if (k_eff == n || k_eff == 0) {
        if (lane == 0) p.tau[row] = k_eff == 0 ? INT_MAX : INT_MIN;
        return;
    }
    const int tq0 = p.t0 + ((t - p.t0) / p.nq_block) * p.nq_block;
    const int s = sample_stride(p, tq0);
    const int m = (n + s - 1) / s;
    int r;
    if (s == 1) {
        r = k_eff;
    } else {
        // the same rank rule as idx_threshold_kernel
        const double e = (double)k_eff * m / n;
        double rr = e + SAMPLE_Z * sqrt(e) + 2.0;
        rr = e + SAMPLE_Z * sqrt(rr) + 2.0;
        rr = e + SAMPLE_Z * sqrt(rr) + 2.0;
        r = (int)ceil(rr);
        r = min(r, m);
    }
    const int32_t *vals = p.sample + row * p.m_cap;           // 16-byte aligned rows (m_cap % 4 == 0)
    const int m4 = m / 4;
    auto for_each = [&](auto f) {
        const int4 *v4 = reinterpret_cast<const int4 *>(vals);
        constexpr int U = 4;
        for (int b0 = lane; b0 < m4; b0 += 32 * U) {
            int4 x[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (b0 + 32 * u < m4) x[u] = __ldcg(v4 + b0 + 32 * u);
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (b0 + 32 * u < m4) { f(x[u].x); f(x[u].y); f(x[u].z); f(x[u].w); }
        }
        for (int i = 4 * m4 + lane; i < m; i += 32) f(__ldcg(vals + i));
    };
    int vmin = INT_MAX, vmax = INT_MIN;
    for_each([&](int v) { vmin = min(vmin, v); vmax = max(vmax, v); });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
        vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    const unsigned range = (unsigned)vmax - (unsigned)vmin;
    int width = range == 0 ? 0 : 32 - __clz(range);
    unsigned lo_key = 0u;                                     // digits chosen so far, in place
    int r_rem = r;
    while (width > 0) {
        const int shift = width > SEL_BITS ? width - SEL_BITS : 0;
        const unsigned hi_mask = ~((width >= 32) ? 0u : ((1u << width) - 1u));   // bits already fixed
#pragma unroll
        for (int i = 0; i < SEL_BINS / 32; ++i) hist[lane * (SEL_BINS / 32) + i] = 0;
        __syncwarp();
        for_each([&](int v) {
            const unsigned key = (unsigned)v - (unsigned)vmin;
            if ((key & hi_mask) == lo_key) atomicAdd(&hist[(key >> shift) & (SEL_BINS - 1)], 1);
        });
        __syncwarp();
        // lane l holds bins 8l .. 8l+7; counts above each bin from the top
        int cb[SEL_BINS / 32], local = 0;
#pragma unroll
        for (int i = 0; i < SEL_BINS / 32; ++i) { cb[i] = hist[lane * (SEL_BINS / 32) + i]; local += cb[i]; }
        int suf = local;                                      // inclusive suffix over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += x;
        }
        int above = suf - local;                              // values in higher lanes' bins
        int sel_bin = -1, sel_above = 0;
#pragma unroll
        for (int i = SEL_BINS / 32 - 1; i >= 0; --i) {
            if (sel_bin < 0 && above < r_rem && above + cb[i] >= r_rem) { sel_bin = lane * (SEL_BINS / 32) + i; sel_above = above; }
            above += cb[i];
        }
        const unsigned who = __ballot_sync(0xffffffffu, sel_bin >= 0);
        if (who == 0u) break;                                 // cannot happen (r <= m); keeps the lower bound
        const int src = __ffs(who) - 1;                       // exactly one lane holds the bin
        sel_bin = __shfl_sync(0xffffffffu, sel_bin, src);
        sel_above = __shfl_sync(0xffffffffu, sel_above, src);
        r_rem -= sel_above;
        lo_key |= (unsigned)sel_bin << shift;
        width = shift;
        __syncwarp();
    }
    if (lane == 0) p.tau[row] = (int)((unsigned)vmin + lo_key);
}

// ----------------------------------------------------------- final select --
// Rows whose top-k was taken by the exact-recompute path (the candidate list
// was short or overflowed), counted per device; read and cleared by
// sa_debug_exact_recompute_rows().
__device__ unsigned long long g_sa_recompute_rows = 0ull;

// Exact score of one (query, key) on CUDA cores (fallback path).
template <int DI>
__device__ __forceinline__ int exact_score(const int8_t *qrow_s, const int *w_s, int Hi, const int8_t *krow) {
    int4 kv[DI / 16];
#pragma unroll
    for (int c = 0; c < DI / 16; ++c) kv[c] = __ldg(reinterpret_cast<const int4 *>(krow) + c);
    int total = 0;
    for (int h = 0; h < Hi; ++h) {
        const int4 *qv = reinterpret_cast<const int4 *>(qrow_s + h * DI);
        int dot = 0;
#pragma unroll
        for (int c = 0; c < DI / 16; ++c) {
            const int4 a = qv[c];
            dot = __dp4a(a.x, kv[c].x, dot);
            dot = __dp4a(a.y, kv[c].y, dot);
            dot = __dp4a(a.z, kv[c].z, dot);
            dot = __dp4a(a.w, kv[c].w, dot);
        }
        total += w_s[h] * max(dot, 0);
    }
    return total;
}

template <int DI>
__host__ __device__ constexpr int select_smem_bytes(int words) {
    return (SEL_BINS + 2 * SEL_TIE_CAP) * 4 + 16 * DI + 16 * 4 + 2 * words * 4;
}
// The candidate list of a row (scores and positions, cap entries each) is
// staged in shared memory after the bitmaps when it fits: the select passes
// then re-read shared memory instead of L2.
constexpr int SEL_STAGE_MAX = 8192;      // list entries staged in shared memory
template <int DI>
__host__ __device__ constexpr int select_stage_off(int words) {
    return (select_smem_bytes<DI>(words) + 15) / 16 * 16;
}
template <int DI>
__host__ __device__ constexpr int select_smem_staged(int words, int cap) {
    return select_stage_off<DI>(words) + (cap <= SEL_STAGE_MAX ? 2 * cap * 4 : 0);
}

// Exact top-k of one row from its candidate list (or, when the list is
// unusable, from scores recomputed on CUDA cores).  Keys above the
// threshold go to a "greater" bitmap over positions, keys equal to it to an
// "equal" bitmap; the output takes every greater key and the lowest-position
// equal keys, in ascending position order.
// DENSE: the row's scores are read from p.dense (every candidate j < n),
// not from a candidate list or recomputed from the indexer vectors.
template <int DI, int NT = SEL_THREADS, bool DENSE = false>
__global__ void __launch_bounds__(NT, NT <= 256 ? 3 : 1) topk_select_kernel(const IdxParams p) {
    grid_dependency_sync();
    extern __shared__ __align__(1024) unsigned char smem[];
    int *hist = reinterpret_cast<int *>(smem);                          // [SEL_BINS]
    unsigned *tie_key = reinterpret_cast<unsigned *>(hist + SEL_BINS);  // [SEL_TIE_CAP]
    int *tie_idx = reinterpret_cast<int *>(tie_key + SEL_TIE_CAP);     // [SEL_TIE_CAP]
    int8_t *qrow_s = reinterpret_cast<int8_t *>(tie_idx + SEL_TIE_CAP);  // [16 * DI]
    int *w_s = reinterpret_cast<int *>(qrow_s + 16 * DI);                // [16]
    unsigned *gt_bm = reinterpret_cast<unsigned *>(w_s + 16);           // [words]
    __shared__ int scan_tmp[32];
    __shared__ int bcast[4];
    __shared__ int tie_n;
    constexpr int NW = NT / 32;
    __shared__ int wg[NW], we[NW];

    const int b = blockIdx.z, tr = blockIdx.y, t = p.t0 + tr;
    if (t >= p.Tq || tr >= p.Rt) return;
    const long long row = (long long)b * p.Rt + tr;
    const long long pos = p.q_pos0 + t;
    const int n = (int)n_candidates(pos, p.window);
    const int wc = p.window > 0 ? (int)(pos + 1 < p.window ? pos + 1 : p.window) : 0;
    const int k_eff = n < p.topk ? n : p.topk;
    int32_t *orow = p.out_idx + ((long long)b * p.Tq + t) * p.Kout;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int words = (n + 31) / 32;
    unsigned *eq_bm = gt_bm + words;

    // window entries, padding and count
    for (int i = tid; i < p.Kout - k_eff; i += NT)
        orow[k_eff + i] = i < wc ? (int)(pos - wc + 1 + i) : -1;
    if (tid == 0 && p.out_count) p.out_count[(long long)b * p.Tq + t] = k_eff + wc;
    if (k_eff == n) {                                 // every candidate is kept
        for (int j = tid; j < n; j += NT) orow[j] = j;
        return;
    }
    if (k_eff == 0) return;

    const int cnt = DENSE ? 0 : p.cand_cnt[row];
    const bool use_list = !DENSE && cnt >= k_eff && cnt <= p.cand_cap;
    if (!DENSE && !use_list && tid == 0) atomicAdd(&g_sa_recompute_rows, 1ull);
    const int2 *cl = DENSE ? nullptr : p.cand + row * p.cand_cap;
    const int8_t *kb = DENSE ? nullptr : p.k + (long long)b * p.L * DI;
    if (!DENSE && !use_list) {
        // exact recompute: stage this query's indexer vectors and weights
        const int8_t *qsrc = p.q + ((long long)b * p.Tq + t) * p.Hi * DI;
        for (int i = tid; i < p.Hi * DI / 16; i += NT)
            reinterpret_cast<int4 *>(qrow_s)[i] = __ldg(reinterpret_cast<const int4 *>(qsrc) + i);
        for (int i = tid; i < p.Hi; i += NT) w_s[i] = __ldg(p.w + ((long long)b * p.Tq + t) * p.Hi + i);
        __syncthreads();
    }
    // the bitmaps are cleared first, while the list loads below are in flight
    for (int i = tid; i < words; i += NT) { gt_bm[i] = 0u; eq_bm[i] = 0u; }
    if (tid == 0) tie_n = 0;
    // stage the list in shared memory (one pass over L2, 16-byte loads, U in
    // flight per thread) and take the score range on the way
    const bool staged = use_list && p.cand_cap <= SEL_STAGE_MAX;
    int *lv_s = reinterpret_cast<int *>(smem + select_stage_off<DI>(words));
    int *li_s = lv_s + p.cand_cap;
    int smin = INT_MAX, smax = INT_MIN;
    // Every listed score is >= the row's threshold tau (the filter kept
    // exactly those), so a histogram with bin = score - tau can be filled
    // while staging; when every score falls within SEL_FINE_BINS of tau it
    // gives the k-th largest score without another pass.
    int *fh = reinterpret_cast<int *>(tie_key);               // the tie arrays serve as its bins
    const int tau_b = staged ? p.tau[row] : 0;
    bool wide = false;
    if (staged) {
        for (int i = tid; i < SEL_FINE_BINS; i += NT) fh[i] = 0;
        __syncthreads();
    }
    if (staged) {
        constexpr int U = 4;
        const int n2 = (cnt + 1) / 2;                 // rows are 16-byte aligned (cap % 64 == 0)
        for (int b0 = tid; b0 < n2; b0 += NT * U) {
            int4 e[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (b0 + u * NT < n2) e[u] = __ldg(reinterpret_cast<const int4 *>(cl) + b0 + u * NT);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = b0 + u * NT;             // pairs 2i and 2i + 1
                if (i < n2) {
                    reinterpret_cast<int2 *>(lv_s)[i] = make_int2(e[u].x, e[u].z);
                    reinterpret_cast<int2 *>(li_s)[i] = make_int2(e[u].y, e[u].w);
                    smin = min(smin, e[u].x);
                    smax = max(smax, e[u].x);
                    unsigned bin = (unsigned)e[u].x - (unsigned)tau_b;
                    if (bin < (unsigned)SEL_FINE_BINS) atomicAdd(&fh[bin], 1); else wide = true;
                    if (2 * i + 1 < cnt) {
                        smin = min(smin, e[u].z);
                        smax = max(smax, e[u].z);
                        bin = (unsigned)e[u].z - (unsigned)tau_b;
                        if (bin < (unsigned)SEL_FINE_BINS) atomicAdd(&fh[bin], 1); else wide = true;
                    }
                }
            }
        }
    }
    // every element of the row: (score, position)
    auto for_each = [&](auto f) {
        if (staged) {
            for (int i = tid; i < cnt; i += NT) f(lv_s[i], li_s[i]);
        } else if (use_list) {
            constexpr int U = 4;
            for (int b0 = tid; b0 < cnt; b0 += NT * U) {
                int2 e[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = b0 + u * NT;
                    if (i < cnt) e[u] = __ldg(cl + i);
                }
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (b0 + u * NT < cnt) f(e[u].x, e[u].y);
            }
        } else if constexpr (DENSE) {
            const int32_t *dr = p.dense + row * p.dense_stride;
            for (int j = tid; j < n; j += NT) f(__ldg(dr + j), j);
        } else {
            for (int j = tid; j < n; j += NT) f(exact_score<DI>(qrow_s, w_s, p.Hi, kb + (long long)j * DI), j);
        }
    };

    // the barrier publishes the staged list and its histogram
    const bool any_wide = staged ? __syncthreads_or(wide) != 0 : true;
    int gmin, gmax;
    RadixState st{0u, 0, k_eff, use_list ? cnt : n};
    if (!any_wide) {
        // every score within SEL_FINE_BINS of tau: the k-th largest from the
        // histogram filled while staging (keys below are relative to tau)
        int bin, above;
        fine_scan<NT>(k_eff, fh, scan_tmp, bcast, bin, above);
        gmin = tau_b;
        st.lo_key = (unsigned)bin;
        st.k_rem = k_eff - above;
    } else {
        if (staged) block_minmax_reduce(smin, smax, gmin, gmax, bcast);
        else block_minmax(gmin, gmax, bcast, for_each);
        const unsigned range = (unsigned)gmax - (unsigned)gmin;
        st.width = range == 0 ? 0 : 32 - __clz(range);
        if (use_list && range < (unsigned)SEL_FINE_BINS) {
            // narrow score range: one exact histogram (bin = score - min) gives
            // the k-th largest score directly; the tie arrays serve as its bins
            int bin, above;
            fine_kth<NT>(k_eff, gmin, fh, scan_tmp, bcast, for_each, bin, above);
            st.lo_key = (unsigned)bin;
            st.width = 0;
            st.k_rem = k_eff - above;
        }
    }
    while (st.width > 0 && (st.width > SEL_BITS || st.bin_count > SEL_TIE_CAP))
        radix_refine<NT>(st, gmin, hist, scan_tmp, bcast, for_each);

    // filter: bitmaps of keys above the bin; the bin's own elements go to the
    // equal bitmap (width 0) or to the tie list
    const unsigned lo_key = st.lo_key;
    const unsigned bin_hi = lo_key + (st.width >= 32 ? 0xffffffffu : ((1u << st.width) - 1u));
    const int width = st.width;
    for_each([&](int v, int j) {
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
    int k_rem = st.k_rem;
    if (width > 0) {   // resolve the tie list: exact threshold inside the bin (<= SEL_BITS bits)
        const int m = min(tie_n, SEL_TIE_CAP);
        RadixState ts{0u, width, k_rem, m};
        auto tie_each = [&](auto f) {
            for (int i = tid; i < m; i += NT) f((int)tie_key[i], tie_idx[i]);
        };
        radix_refine<NT>(ts, 0, hist, scan_tmp, bcast, tie_each);   // width <= 12: one step is exact
        const unsigned thr_off = ts.lo_key;
        k_rem = ts.k_rem;
        for (int i = tid; i < m; i += NT) {
            const int j = tie_idx[i];
            if (tie_key[i] > thr_off) atomicOr(&gt_bm[j >> 5], 1u << (j & 31));
            else if (tie_key[i] == thr_off) atomicOr(&eq_bm[j >> 5], 1u << (j & 31));
        }
        __syncthreads();
    }

    // ordered output: warps own contiguous word ranges, and inside a warp
    // each lane a contiguous run of words, so one prefix over the lanes
    // (not one per 32 words) places every lane's keys
    const int wpw = (words + NW - 1) / NW;
    const int w_lo = min(warp * wpw, words), w_hi = min(w_lo + wpw, words);
    const int wpl = (w_hi - w_lo + 31) / 32;                 // words per lane
    const int l_lo = min(w_lo + lane * wpl, w_hi), l_hi = min(l_lo + wpl, w_hi);
    int gl = 0, el = 0;
    for (int i = l_lo; i < l_hi; ++i) { gl += __popc(gt_bm[i]); el += __popc(eq_bm[i]); }
    int g_incl = gl, e_incl = el;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int xg = __shfl_up_sync(0xffffffffu, g_incl, o);
        const int xe = __shfl_up_sync(0xffffffffu, e_incl, o);
        if (lane >= o) { g_incl += xg; e_incl += xe; }
    }
    if (lane == 31) { wg[warp] = g_incl; we[warp] = e_incl; }
    __syncthreads();
    int g_before = 0, e_before = 0;
    for (int i = 0; i < warp; ++i) { g_before += wg[i]; e_before += we[i]; }
    // equal keys are taken in position order until k_rem are used
    const int e_pre = e_before + e_incl - el;                 // equal keys before this lane's run
    int take = k_rem - e_pre;
    take = take < 0 ? 0 : (take > el ? el : take);
    int slot = g_before + (g_incl - gl) + min(e_pre, k_rem);
    for (int i = l_lo; i < l_hi; ++i) {
        const unsigned ew = eq_bm[i];
        unsigned em = 0u;
        if (take >= __popc(ew)) {
            em = ew;
        } else {
            unsigned rest = ew;
            for (int c = 0; c < take; ++c) { const unsigned lowbit = rest & (~rest + 1u); em |= lowbit; rest ^= lowbit; }
        }
        take -= __popc(em);
        unsigned bits = gt_bm[i] | em;
        while (bits) {
            const int bpos = __ffs(bits) - 1;
            bits &= bits - 1u;
            if (slot < k_eff) orow[slot] = i * 32 + bpos;   // slot < k_eff by construction
            ++slot;
        }
    }
}

}  // namespace sa
