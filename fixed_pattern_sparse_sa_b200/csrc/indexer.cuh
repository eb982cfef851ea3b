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
};

// Number of selectable (non-window) candidates of a query at position p.
__device__ __forceinline__ long long n_candidates(long long p, int window) {
    long long n = window > 0 ? p - window + 1 : p + 1;
    return n > 0 ? n : 0;
}

// Tile: 128 keys (4 warps x 2 m-tiles of 16) x 128 (query, head) columns.
template <int HI, int DI>
__global__ void __launch_bounds__(128) idx_score_kernel(const IdxScoreParams p) {
    constexpr int KT = 128;                  // keys per CTA
    constexpr int COLS = 128;                // (query, head) columns per CTA
    constexpr int QT = COLS / HI;            // queries per CTA
    constexpr int NT = COLS / 8;             // n-tiles
    constexpr int REG = DI / 16;             // u32 registers per lane per row
    constexpr int KSTEPS = DI / 32;
    constexpr int NG = 4;                    // n-tiles per accumulator group
    static_assert(HI == 1 || HI == 2 || HI == 4 || HI == 8 || HI == 16, "HI");
    static_assert(DI == 32 || DI == 64 || DI == 128, "DI");

    extern __shared__ __align__(1024) unsigned char smem[];
    int *tile = reinterpret_cast<int *>(smem);           // [QT][KT]
    int *ws = tile + QT * KT;                             // [QT*HI]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, qc = lane & 3;
    const int b = blockIdx.z;
    const int tq0 = p.t0 + blockIdx.y * QT;               // first query of the tile
    const int j0 = blockIdx.x * KT;
    const int t_last = min(p.t0 + p.Rt, p.Tq) - 1;
    const int tq_last = min(tq0 + QT - 1, t_last);
    if (tq0 > t_last) return;
    if ((long long)j0 >= n_candidates(p.q_pos0 + tq_last, p.window)) return;   // above the diagonal

    for (int i = threadIdx.x; i < QT * HI; i += blockDim.x) {
        const int tq = tq0 + i / HI;
        ws[i] = tq <= tq_last ? __ldg(p.w + ((long long)b * p.Tq + tq) * HI + i % HI) : 0;
    }

    // A fragments: this warp's 32 keys (2 m-tiles), rows gr and gr+8.
    unsigned a[2][2][REG];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int j = j0 + warp * 32 + mt * 16 + gr + hr * 8;
            const unsigned *src = reinterpret_cast<const unsigned *>(
                p.k + ((long long)b * p.L + j) * DI + qc * (DI / 4));
#pragma unroll
            for (int r = 0; r < REG; ++r) a[mt][hr][r] = j < p.L ? __ldg(src + r) : 0u;
        }
    __syncthreads();

#pragma unroll 1
    for (int ng = 0; ng < NT / NG; ++ng) {
        int acc[2][NG][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int n = 0; n < NG; ++n) acc[mt][n][0] = acc[mt][n][1] = acc[mt][n][2] = acc[mt][n][3] = 0;
#pragma unroll
        for (int n = 0; n < NG; ++n) {
            const int nt = ng * NG + n;
            const int col = nt * 8 + gr;                      // B column held by this lane
            const int tq = tq0 + col / HI, h = col % HI;
            unsigned bq[REG];
            const unsigned *src = reinterpret_cast<const unsigned *>(
                p.q + (((long long)b * p.Tq + tq) * HI + h) * DI + qc * (DI / 4));
#pragma unroll
            for (int r = 0; r < REG; ++r) bq[r] = tq <= tq_last ? __ldg(src + r) : 0u;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks)
                    mma_s8_16832(acc[mt][n], a[mt][0][2 * ks], a[mt][1][2 * ks], a[mt][0][2 * ks + 1],
                                 a[mt][1][2 * ks + 1], bq[2 * ks], bq[2 * ks + 1]);
        }
        // epilogue: w * relu, sum over the heads of each query, stage to smem
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int n = 0; n < NG; ++n) {
                const int nt = ng * NG + n;
                const int c0 = nt * 8 + 2 * qc, c1 = c0 + 1;  // columns of this thread
                const int w0 = ws[c0], w1 = ws[c1];
                const int r0a = w0 * max(acc[mt][n][0], 0), r0b = w1 * max(acc[mt][n][1], 0);
                const int r1a = w0 * max(acc[mt][n][2], 0), r1b = w1 * max(acc[mt][n][3], 0);
                const int kr0 = warp * 32 + mt * 16 + gr, kr1 = kr0 + 8;
                if constexpr (HI == 1) {
                    tile[(c0)*KT + kr0] = r0a; tile[(c1)*KT + kr0] = r0b;
                    tile[(c0)*KT + kr1] = r1a; tile[(c1)*KT + kr1] = r1b;
                } else {
                    int s0 = r0a + r0b, s1 = r1a + r1b;
                    if constexpr (HI >= 4) {
                        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
                        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                    }
                    if constexpr (HI >= 8) {
                        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
                        s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                    }
                    const int qi = c0 / HI;                   // query of this column pair
                    constexpr int LEAD = HI >= 8 ? 4 : (HI == 4 ? 2 : 1);
                    if ((qc % LEAD) == 0) {
                        if constexpr (HI == 16) {
                            // a query spans two n-tiles: accumulate both halves
                            if ((nt & 1) == 0) {
                                tile[qi * KT + kr0] = s0; tile[qi * KT + kr1] = s1;
                            } else {
                                tile[qi * KT + kr0] += s0; tile[qi * KT + kr1] += s1;
                            }
                        } else {
                            tile[qi * KT + kr0] = s0; tile[qi * KT + kr1] = s1;
                        }
                    }
                }
            }
        __syncwarp();
    }
    __syncthreads();

    // coalesced write-out of the [QT][KT] tile
    const bool vec = (p.ld % 4) == 0;
    for (int i = threadIdx.x; i < QT * (KT / 4); i += blockDim.x) {
        const int qi = i / (KT / 4), k4 = (i % (KT / 4)) * 4;
        const int tq = tq0 + qi;
        if (tq > tq_last) continue;
        const long long ncand = n_candidates(p.q_pos0 + tq, p.window);
        const int j = j0 + k4;
        if (j >= ncand) continue;
        int32_t *dst = p.scores + ((long long)b * p.Rt + (tq - p.t0)) * p.ld + j;
        const int *src = tile + qi * KT + k4;
        if (vec && j + 3 < ncand) {
            *reinterpret_cast<int4 *>(dst) = *reinterpret_cast<const int4 *>(src);
        } else {
            for (int u = 0; u < 4 && j + u < ncand; ++u) dst[u] = src[u];
        }
    }
}

// ------------------------------------------------------------- top-k select --
struct SelectParams {
    const int32_t *scores;   // [B, Rt, ld]
    long long ld;
    int B, Tq, t0, Rt;
    long long q_pos0;
    int topk, window, Kout;
    int32_t *out_idx;        // [B, Tq, Kout]
    int32_t *out_count;      // [B, Tq] nullable
};

constexpr int SEL_THREADS = 512;
constexpr int SEL_BITS = 12;
constexpr int SEL_BINS = 1 << SEL_BITS;

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

__global__ void __launch_bounds__(SEL_THREADS) topk_select_kernel(const SelectParams p) {
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();

    __shared__ int hist[2][SEL_BINS];
    __shared__ int red[4];            // local min, max, n_gt, n_eq
    __shared__ int wcnt[2][SEL_THREADS / 32];
    __shared__ int scan_tmp[32];
    __shared__ int bcast[4];

    const int b = blockIdx.z, tr = blockIdx.y, t = p.t0 + tr;
    if (t >= p.Tq || tr >= p.Rt) return;     // uniform for the whole cluster
    const long long pos = p.q_pos0 + t;
    const long long n = n_candidates(pos, p.window);
    const int wc = p.window > 0 ? (int)(pos + 1 < p.window ? pos + 1 : p.window) : 0;
    const int k_eff = (int)(n < p.topk ? n : p.topk);
    int32_t *orow = p.out_idx + ((long long)b * p.Tq + t) * p.Kout;
    const int32_t *srow = p.scores + ((long long)b * p.Rt + tr) * p.ld;
    const int tid = threadIdx.x;

    // window entries, padding and count (rank 0 only)
    if (rank == 0) {
        for (int i = tid; i < p.Kout - k_eff; i += blockDim.x) {
            const int o = k_eff + i;
            orow[o] = i < wc ? (int)(pos - wc + 1 + i) : -1;
        }
        if (tid == 0 && p.out_count) p.out_count[(long long)b * p.Tq + t] = k_eff + wc;
    }
    const long long seg = (n + C - 1) / C;
    const long long lo = rank * seg < n ? rank * seg : n;
    const long long hi = lo + seg < n ? lo + seg : n;

    if (k_eff == n) {                          // every candidate is kept
        for (long long j = lo + tid; j < hi; j += blockDim.x) orow[j] = (int)j;
        return;
    }
    if (k_eff == 0) return;

    // 1. min / max of the row
    int vmin = INT_MAX, vmax = INT_MIN;
    for (long long j = lo + tid; j < hi; j += blockDim.x) {
        const int v = __ldg(srow + j);
        vmin = min(vmin, v);
        vmax = max(vmax, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        vmin = min(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
        vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (tid == 0) { red[0] = INT_MAX; red[1] = INT_MIN; }
    __syncthreads();
    if ((tid & 31) == 0) { atomicMin(&red[0], vmin); atomicMax(&red[1], vmax); }
    cluster.sync();
    if (tid == 0) {
        int mn = INT_MAX, mx = INT_MIN;
        for (int r = 0; r < C; ++r) {
            const int *rr = cluster.map_shared_rank(red, r);
            mn = min(mn, rr[0]);
            mx = max(mx, rr[1]);
        }
        bcast[0] = mn; bcast[1] = mx;
    }
    __syncthreads();
    const int gmin = bcast[0], gmax = bcast[1];
    const unsigned range = (unsigned)((long long)gmax - (long long)gmin);
    const int nbits = range == 0 ? 0 : 32 - __clz(range);

    // 2. radix passes over u = v - gmin, 12-bit digits from the top
    unsigned long long prefix = 0;   // determined high bits of the threshold key
    int known = nbits;               // bits at and above `known` are determined (all zero above nbits)
    int k_rem = k_eff;               // how many still to take at/below the current prefix
    int pass = 0;
    while (known > 0) {
        const int shift = known > SEL_BITS ? known - SEL_BITS : 0;
        const int width = known - shift;
        int *h = hist[pass & 1];
        for (int i = tid; i < SEL_BINS; i += blockDim.x) h[i] = 0;
        __syncthreads();
        for (long long j = lo + tid; j < hi; j += blockDim.x) {
            const unsigned long long u = (unsigned long long)((long long)__ldg(srow + j) - gmin);
            if ((u >> known) == prefix) atomicAdd(&h[(u >> shift) & ((1u << width) - 1u)], 1);
        }
        cluster.sync();
        // total histogram, then the digit whose suffix count first reaches k_rem
        const int per = SEL_BINS / SEL_THREADS;   // bins per thread (8), highest bins first
        int cnt[SEL_BINS / SEL_THREADS];
        int local = 0;
#pragma unroll
        for (int u = 0; u < per; ++u) {
            const int bin = SEL_BINS - 1 - (tid * per + u);
            int c = 0;
            for (int r = 0; r < C; ++r) c += cluster.map_shared_rank(h, r)[bin];
            cnt[u] = c;
            local += c;
        }
        const int incl = block_incl_scan(local, scan_tmp);
        int above = incl - local;                 // count in strictly higher bins
#pragma unroll
        for (int u = 0; u < per; ++u) {
            const int bin = SEL_BINS - 1 - (tid * per + u);
            if (above < k_rem && above + cnt[u] >= k_rem) {
                bcast[2] = bin;
                bcast[3] = above;
            }
            above += cnt[u];
        }
        __syncthreads();
        const int digit = bcast[2];
        k_rem -= bcast[3];
        prefix = (prefix << width) | (unsigned long long)digit;
        known = shift;
        ++pass;
        __syncthreads();
    }
    const long long thr = (long long)gmin + (long long)prefix;   // exact k-th largest score

    // 3. per-warp counts of (> thr) and (== thr) over warp sub-segments
    const int nw = blockDim.x >> 5, warp = tid >> 5, lane = tid & 31;
    const long long wseg = ((hi - lo) + nw - 1) / nw;
    const long long wlo = lo + warp * wseg < hi ? lo + warp * wseg : hi;
    const long long whi = wlo + wseg < hi ? wlo + wseg : hi;
    int ngt = 0, neq = 0;
    for (long long j = wlo + lane; j < whi; j += 32) {
        const int v = __ldg(srow + j);
        ngt += v > thr;
        neq += v == thr;
    }
    ngt = warp_sum_int(ngt);
    neq = warp_sum_int(neq);
    if (lane == 0) { wcnt[0][warp] = ngt; wcnt[1][warp] = neq; }
    __syncthreads();
    if (tid == 0) {
        int a = 0, e = 0;
        for (int i = 0; i < nw; ++i) { a += wcnt[0][i]; e += wcnt[1][i]; }
        red[2] = a; red[3] = e;
    }
    cluster.sync();
    __shared__ long long base[2];
    if (tid == 0) {
        long long gb = 0, eb = 0;
        for (int r = 0; r < rank; ++r) {
            const int *rr = cluster.map_shared_rank(red, r);
            gb += rr[2];
            eb += rr[3];
        }
        base[0] = gb; base[1] = eb;
    }
    __syncthreads();
    long long gt_base = base[0], eq_base = base[1];
    for (int i = 0; i < warp; ++i) { gt_base += wcnt[0][i]; eq_base += wcnt[1][i]; }
    // output slot of the first selected key of this warp: all earlier > thr
    // keys, plus the earlier ties that are kept
    long long sel_base = gt_base + (eq_base < k_rem ? eq_base : k_rem);
    const unsigned lt = (1u << lane) - 1u;
    for (long long j0 = wlo; j0 < whi; j0 += 32) {
        const long long j = j0 + lane;
        const int v = j < whi ? __ldg(srow + j) : INT_MIN;
        const bool isg = j < whi && v > thr, ise = j < whi && v == thr;
        const unsigned me = __ballot_sync(0xffffffffu, ise);
        const long long erank = eq_base + __popc(me & lt);
        const bool sel = isg || (ise && erank < k_rem);
        const unsigned ms = __ballot_sync(0xffffffffu, sel);
        const long long slot = sel_base + __popc(ms & lt);
        if (sel && slot < k_eff) orow[slot] = (int)j;   // slot < k_eff by construction
        sel_base += __popc(ms);
        eq_base += __popc(me);
    }
    cluster.sync();   // keep shared memory alive until every remote read is done
}

}  // namespace sa
