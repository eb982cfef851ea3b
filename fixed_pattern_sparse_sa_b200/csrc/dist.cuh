// dist.cuh -- kernels of the sequence-split (multi-GPU) decode path.
//
// Star Attention page ("NVIDIA AI Research presenta Star Attention ...",
// body): the context is split across hosts, each host computes its part and
// the parts are merged by a distributed softmax, with little data crossing
// between hosts.  Applied to indexer-selected sparse attention with the keys
// of one sequence split by position over R ranks:
//   1. each rank takes the exact top-(k + window) of its own keys (with the
//      scores of the kept keys: idx_scores_at_kernel);
//   2. the ranks exchange these candidates (R x (k + window) pairs per query);
//   3. topk_merge_kernel picks the exact global top-k by (score desc, index
//      asc) among the non-window candidates and adds the window; the global
//      top-k of the non-window keys lies inside the union of the local
//      top-(k + window) sets, so the result equals the single-GPU selection;
//   4. each rank attends over the selected keys that it holds
//      (index_shard_kernel maps them to its rows) and the partial
//      (out, lse) of the ranks are merged by lse_combine.
#pragma once

#include "indexer.cuh"

namespace sa {

// Exact indexer scores of listed keys: one CTA per query row (b, t); entry
// idx[row, e] >= 0 gets I(t, idx), -1 gets INT_MIN.
template <int DI>
__global__ void __launch_bounds__(128) idx_scores_at_kernel(const int8_t *q, const int8_t *k, const int32_t *w,
                                                            int B, int Tq, int L, int Hi, const int32_t *idx, int K,
                                                            int32_t *out, unsigned *err) {
    grid_dependency_sync();
    __shared__ __align__(16) int8_t qrow_s[16 * DI];
    __shared__ int w_s[16];
    const long long row = blockIdx.x;                  // b * Tq + t
    if (row >= (long long)B * Tq) return;
    const int b = (int)(row / Tq);
    for (int i = threadIdx.x; i < Hi * DI / 16; i += blockDim.x)
        reinterpret_cast<int4 *>(qrow_s)[i] = __ldg(reinterpret_cast<const int4 *>(q + row * Hi * DI) + i);
    for (int i = threadIdx.x; i < Hi; i += blockDim.x) w_s[i] = __ldg(w + row * Hi + i);
    __syncthreads();
    for (int e = threadIdx.x; e < K; e += blockDim.x) {
        const int j = __ldg(idx + row * K + e);
        int s = INT_MIN;
        if (j >= 0 && j < L) s = exact_score<DI>(qrow_s, w_s, Hi, k + ((long long)b * L + j) * DI);
        else if (j >= L) raise_error(err, ERR_BAD_INDEX);
        out[row * K + e] = s;
    }
}

// Global top-k of gathered candidates, one CTA (TM_THREADS) per row.
// Candidates: n_parts blocks of kc (score, local index) pairs; part p's
// indices are shifted by part_off[p] to global positions (-1 = none).
// Positions in the forced window [q_pos - window + 1, q_pos] are left out of
// the ranking and appended; the output row is ascending, -1 padded.
constexpr int TM_THREADS = 512;
constexpr int TM_MAX_PARTS = 64;                     // ranks whose candidates one merge takes
struct MergeOffsets {
    long long off[TM_MAX_PARTS];                     // position of part p's local index 0
};
constexpr int TM_MAX_CAND = 24576;                   // candidates per row held in shared memory
constexpr int TM_MAX_K = 4096;                       // topk of the merge (power of two for the sort)

__host__ __device__ constexpr int topk_merge_smem_bytes(int n_cand) {
    return n_cand * 8 + TM_MAX_K * 4 + (SEL_BINS + 64) * 4;
}

__global__ void __launch_bounds__(TM_THREADS) topk_merge_kernel(const int32_t *cand_score, const int32_t *cand_idx,
                                                                 const MergeOffsets part_off, int n_parts, long long rows,
                                                                 int kc, int topk, int window, long long q_pos,
                                                                 int32_t *out_idx, int32_t *out_count) {
    grid_dependency_sync();
    extern __shared__ __align__(1024) unsigned char smem[];
    const int n = n_parts * kc;
    int *sv = reinterpret_cast<int *>(smem);                  // [n] scores
    int *sj = sv + n;                                         // [n] global positions (-1: none)
    int *sel = sj + n;                                        // [TM_MAX_K] chosen positions
    int *hist = sel + TM_MAX_K;                               // [SEL_BINS]
    int *scan_tmp = hist + SEL_BINS;                          // [32]
    int *bcast = scan_tmp + 32;                               // [4]
    int *n_sel = bcast + 4;
    const long long row = blockIdx.x;
    if (row >= rows) return;
    const int tid = threadIdx.x;
    const long long wlo = window > 0 ? q_pos - window + 1 : q_pos + 1;   // first window position
    int local_valid = 0;
    for (int i = tid; i < n; i += TM_THREADS) {
        const int p = i / kc, e = i % kc;
        const long long off = ((long long)p * rows + row) * kc + e;
        const int j = __ldg(cand_idx + off);
        const long long gj = j >= 0 ? (long long)j + part_off.off[p] : -1;
        const bool ok = gj >= 0 && gj < wlo;                  // window positions are forced, not ranked
        sv[i] = ok ? __ldg(cand_score + off) : INT_MIN;
        sj[i] = ok ? (int)gj : -1;
        local_valid += ok;
    }
    if (tid == 0) *n_sel = 0;
    const int m = block_incl_scan(local_valid, scan_tmp);    // last thread holds the total
    if (tid == TM_THREADS - 1) bcast[0] = m;
    __syncthreads();
    const int n_valid = bcast[0];
    __syncthreads();
    const int k_eff = min(topk, n_valid);
    auto each_valid = [&](auto f) {
        for (int i = tid; i < n; i += TM_THREADS)
            if (sj[i] >= 0) f(sv[i], i);
    };
    int thr_v = INT_MAX, thr_j = -1;                          // take score > thr_v, and == thr_v with j <= thr_j
    if (k_eff > 0) {
        int gmin, gmax;
        block_minmax(gmin, gmax, bcast, each_valid);
        const unsigned range = (unsigned)gmax - (unsigned)gmin;
        RadixState st{0u, range == 0 ? 0 : 32 - __clz(range), k_eff, n_valid};
        while (st.width > 0) radix_refine<TM_THREADS>(st, gmin, hist, scan_tmp, bcast, each_valid);
        thr_v = (int)((unsigned)gmin + st.lo_key);
        // ties at thr_v: the st.k_rem lowest positions (positions are unique)
        auto each_tie = [&](auto f) {
            for (int i = tid; i < n; i += TM_THREADS)
                if (sj[i] >= 0 && sv[i] == thr_v) f(INT_MAX - sj[i], i);
        };
        int tmin, tmax;
        block_minmax(tmin, tmax, bcast, each_tie);
        const unsigned r2 = (unsigned)tmax - (unsigned)tmin;
        RadixState s2{0u, r2 == 0 ? 0 : 32 - __clz(r2), st.k_rem, 0};
        while (s2.width > 0) radix_refine<TM_THREADS>(s2, tmin, hist, scan_tmp, bcast, each_tie);
        thr_j = INT_MAX - (int)((unsigned)tmin + s2.lo_key);
    }
    // chosen positions, then an ascending bitonic sort in shared memory
    for (int i = tid; i < n; i += TM_THREADS) {
        if (sj[i] >= 0 && (sv[i] > thr_v || (sv[i] == thr_v && sj[i] <= thr_j))) {
            const int slot = atomicAdd(n_sel, 1);
            if (slot < TM_MAX_K) sel[slot] = sj[i];
        }
    }
    __syncthreads();
    const int ns = min(*n_sel, TM_MAX_K);
    int np2 = 1;
    while (np2 < ns) np2 <<= 1;
    for (int i = ns + tid; i < np2; i += TM_THREADS) sel[i] = INT_MAX;
    __syncthreads();
    for (int size = 2; size <= np2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < np2; i += TM_THREADS) {
                const int pj = i ^ stride;
                if (pj > i) {
                    const bool up = (i & size) == 0;
                    const int a = sel[i], c = sel[pj];
                    if ((a > c) == up) { sel[i] = c; sel[pj] = a; }
                }
            }
            __syncthreads();
        }
    }
    const int wc = window > 0 ? (int)min((long long)window, q_pos + 1) : 0;
    const int kout = topk + window;
    int32_t *orow = out_idx + row * kout;
    for (int i = tid; i < kout; i += TM_THREADS) {
        int v = -1;
        if (i < ns) v = sel[i];
        else if (i < ns + wc) v = (int)(q_pos - wc + 1 + (i - ns));
        orow[i] = v;
    }
    if (tid == 0 && out_count) out_count[row] = ns + wc;
}

// Global positions -> rows of the shard [key_lo, key_hi) (other entries -1).
__global__ void index_shard_kernel(const int32_t *idx, long long n, long long key_lo, long long key_hi, int32_t *out) {
    grid_dependency_sync();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int j = idx[i];
    out[i] = (j >= key_lo && j < key_hi) ? (int)(j - key_lo) : -1;
}

}  // namespace sa
