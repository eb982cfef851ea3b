// indexer_filter.cuh -- the indexer's filter pass on tcgen05: exact int8
// scores of every (query, candidate key), kept when they reach the query's
// sampled threshold tau.
//
// IndexCache page ("IndexCache: inferencia 82% mas rapida ...", body): the
// lightweight indexer scores every earlier token of each query; its cost
// grows with the context.  Score of query t for key j (exact, int32):
//   I(t, j) = sum_h w[t,h] * max(0, q[t,h,:] . k[j,:])
// The pairs with I >= tau[t] go to the row's candidate list; the exact top-k
// is then taken from the list (topk_select_kernel in indexer.cuh).
//
// Design (one persistent CTA per SM):
//  * Work unit = one block of NQ = 224 / HI consecutive queries of one
//    sequence and ALL of their candidate keys, so a row's list is written by
//    one CTA only: list slots come from shared-memory counters, never from
//    global atomics.  Units are taken latest (heaviest) block first.
//  * MMA: D[128 keys x 224 (query, head) columns] = K_tile . Q_block^T
//    (tcgen05.mma kind::i8, s32 accumulators in TMEM), K = DI.  Two
//    accumulators (two 224-column regions of TMEM) let the MMA of tile k+1
//    run while the epilogue drains tile k.
//  * Operands arrive by TMA box loads into the K-major swizzled layout whose
//    swizzle width equals the row (DI bytes: 32B, 64B or 128B swizzle): key
//    tiles of 128 rows through a FT_STAGES-deep ring, the query block's
//    224 rows double-buffered by unit.
//  * Weights are folded into the query operand beforehand wherever that is
//    exact (w >= 0 and every w*q fits int8: w*relu(x) = relu(w*x)); a unit
//    whose weights all fold sums ReLUs with one DPX add-max per head,
//    starting from -tau so that the keep test is a sign test.
//  * Warps: 0 TMA producer (lane 0 issues; all lanes write the unit's
//    per-query constants), 1 MMA issuer and TMEM owner, 2..29 epilogue:
//    warp w reads TMEM lane quadrant w % 4 (one key row per thread) over 32
//    of the 224 columns.  224 columns (not 256) let 28 epilogue warps share
//    them evenly: the epilogue is bound by latency, and 30 warps per SM at
//    64 registers hide more of it than 18 warps at 96.
// Every wait is bounded (progress waits by the spin limit, drains by a fixed
// long limit); a timeout sets ERR_TIMEOUT, the roles stop together and the
// CTA drains its copies and MMAs before freeing TMEM.
#pragma once

#include <cuda.h>

#include "attn_tc.cuh"
#include "indexer.cuh"

namespace sa {

constexpr int FT_NCOL = 224;                      // (query, head) columns of a unit: 7 x 32
constexpr int FT_STAGES = 6;                      // key-tile ring depth
constexpr int FT_EPI_WARPS = 28;                  // 7 per TMEM lane quadrant, 32 columns each
constexpr int FT_THREADS = (2 + FT_EPI_WARPS) * 32;
constexpr int FT_CW = FT_NCOL / (FT_EPI_WARPS / 4);   // columns per epilogue warp (32)
constexpr int FT_ACC = 256;                       // TMEM column stride of the two accumulators
constexpr uint32_t FT_TM_COLS = 512;

template <int DI>
struct FtSmem {
    static constexpr int A_BYTES = 128 * DI;                  // one key tile
    static constexpr int B_BYTES = FT_NCOL * DI;              // one query block
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + FT_STAGES * A_BYTES;
    static constexpr int OFF_W = OFF_B + 2 * B_BYTES;         // int [2][256] weight per column (slow path)
    static constexpr int OFF_TAU = OFF_W + 2 * FT_NCOL * 4;   // int [2][256] threshold per query
    static constexpr int OFF_NC = OFF_TAU + 2 * FT_NCOL * 4;  // int [2][256] candidates per query
    static constexpr int OFF_CNT = OFF_NC + 2 * FT_NCOL * 4;  // int [2][256] list length per query
    static constexpr int OFF_FAST = OFF_CNT + 2 * FT_NCOL * 4;   // int [2]: every weight of the unit folded
    static constexpr int OFF_BAR = OFF_FAST + 16;
    // a_full[S], a_empty[S], b_full[2], b_empty[2], meta_full[2], meta_empty[2],
    // acc_full[2], acc_free[2], drain
    static constexpr int N_BAR = 2 * FT_STAGES + 10 + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;      // tmem slot, abort flag
    static constexpr int TOTAL = OFF_MISC + 16;
    // at least ~116 KB so that one CTA (and its 512 TMEM columns) holds an SM
    static constexpr int ALLOC = TOTAL + 1024 > 118 * 1024 ? TOTAL + 1024 : 118 * 1024;
};

struct FtParams {
    IdxParams p;             // shapes, chunk rows, thresholds, candidate lists
    const int32_t *wf;       // [B, Tq, Hi] weight left to apply (1 where folded into q)
    int n_units;             // B * ceil(Rt / NQ)
};

// Weight folding, one thread per (query row, head) of the whole call:
// qf = w*q and wf = 1 when w >= 0 and every product fits int8, else qf = q and
// wf = w.  Either way sum_h wf*relu(qf.k) equals the score.
template <int DI>
__global__ void __launch_bounds__(256) idx_fold_kernel(const int8_t *__restrict__ q, const int32_t *__restrict__ w,
                                                       int8_t *__restrict__ qf, int32_t *__restrict__ wf,
                                                       long long n_heads) {
    grid_dependency_sync();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_heads) return;
    const int wv = __ldg(w + i);
    const int4 *src = reinterpret_cast<const int4 *>(q + i * DI);
    int4 *dst = reinterpret_cast<int4 *>(qf + i * DI);
    int4 v[DI / 16];
    bool ok = wv >= 0;
#pragma unroll
    for (int c = 0; c < DI / 16; ++c) {
        v[c] = __ldg(src + c);
        int words[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            unsigned packed = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int x = (int)(signed char)((words[u] >> (8 * e)) & 0xff) * wv;
                ok &= (x >= -128) & (x <= 127);
                packed |= ((unsigned)x & 0xffu) << (8 * e);
            }
            words[u] = (int)packed;
        }
        if (ok) v[c] = make_int4(words[0], words[1], words[2], words[3]);
    }
    if (!ok) {
#pragma unroll
        for (int c = 0; c < DI / 16; ++c) v[c] = __ldg(src + c);
    }
#pragma unroll
    for (int c = 0; c < DI / 16; ++c) dst[c] = v[c];
    wf[i] = ok ? 1 : wv;
}

namespace ft {
// Shared-memory counter increment that returns the old value.
__device__ __forceinline__ int atom_add1_shared(uint32_t addr) {
    int old;
    asm volatile("atom.shared.add.u32 %0, [%1], 1;\n" : "=r"(old) : "r"(addr));
    return old;
}
// 32 lanes x 32 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// K-major shared-memory descriptor with the swizzle whose width is one DI-byte
// row (layout type 6 = 32B, 4 = 64B, 2 = 128B); 8-row groups 8*DI bytes apart.
template <int DI>
__device__ __forceinline__ uint64_t desc_row_swizzled(uint32_t saddr) {
    constexpr uint64_t layout = DI == 32 ? 6 : DI == 64 ? 4 : 2;
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                              // leading offset: unused in this layout
    d |= (uint64_t)(((8 * DI) >> 4) & 0x3FFFu) << 32;     // 8-row group stride
    d |= (uint64_t)1 << 46;
    d |= layout << 61;
    return d;
}
}  // namespace ft

// Start of the ReLU-sum chain on the folded path: the chain runs from -tau
// so that a pair is kept when the sum ends >= 0.  With every weight folded a
// score is below 2^25 (at most 16 heads x 128 x 128 x 128), so clamping tau
// to [0, 2^26] keeps the keep test exact (tau <= 0 keeps everything, tau
// above every score keeps nothing: tau = INT_MAX marks a row with nothing to
// keep or a query past the unit) while no partial sum can leave int32.
__device__ __forceinline__ int ft_fast_tau(int tau) { return min(max(tau, 0), 1 << 26); }

// Unit u -> (b, first query, last query); latest query blocks first.
__device__ __forceinline__ void ft_unit(const IdxParams &p, int nq, int u, int &b, int &tq0, int &tq_last) {
    const int nqb = (p.Rt + nq - 1) / nq;
    const int qb = nqb - 1 - u / p.B;
    b = u % p.B;
    tq0 = p.t0 + qb * nq;
    tq_last = min(tq0 + nq - 1, min(p.t0 + p.Rt, p.Tq) - 1);
}
__device__ __forceinline__ int ft_tiles(const IdxParams &p, int tq_last) {
    const long long n = n_candidates(p.q_pos0 + tq_last, p.window);
    return (int)((n + 127) / 128);
}

template <int HI, int DI>
__global__ void __launch_bounds__(FT_THREADS, 1)
    idx_filter_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                         const FtParams fp) {
    grid_dependency_sync();
    constexpr int NQ = FT_NCOL / HI;         // queries per unit
    constexpr int NQT = FT_CW / HI;          // queries per epilogue thread
    constexpr bool QREG = NQT <= 8;          // per-query constants held in registers
    using L = FtSmem<DI>;
    static_assert(FT_CW % HI == 0 && NQ <= FT_NCOL, "heads of a query within one warp's columns");
    constexpr uint32_t IDESC = tc::make_idesc(2 /*s32*/, 1 /*s8*/, 128, FT_NCOL);
    const IdxParams &p = fp.p;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *a_full = bars, *a_empty = bars + FT_STAGES;
    uint64_t *b_full = bars + 2 * FT_STAGES, *b_empty = b_full + 2;
    uint64_t *meta_full = b_empty + 2, *meta_empty = meta_full + 2;
    uint64_t *acc_full = meta_empty + 2, *acc_free = acc_full + 2, *drain = acc_free + 2;
    int *w_s = reinterpret_cast<int *>(smem + L::OFF_W);
    int *tau_s = reinterpret_cast<int *>(smem + L::OFF_TAU);
    int *nc_s = reinterpret_cast<int *>(smem + L::OFF_NC);
    int *cnt_s = reinterpret_cast<int *>(smem + L::OFF_CNT);
    int *fast_s = reinterpret_cast<int *>(smem + L::OFF_FAST);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, FT_TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < FT_STAGES; ++i) { tc::mbar_init(a_full + i, 1); tc::mbar_init(a_empty + i, 1); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(b_full + i, 1); tc::mbar_init(b_empty + i, 1);
            tc::mbar_init(meta_full + i, 32); tc::mbar_init(meta_empty + i, FT_EPI_WARPS * 32);
            tc::mbar_init(acc_full + i, 1); tc::mbar_init(acc_free + i, FT_EPI_WARPS);
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() {
        raise_error(p.err, ERR_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        bool ok = true;
        int un = 0, tile = 0, b_issued = 0;
        for (int u = blockIdx.x; u < fp.n_units && ok; u += gridDim.x) {
            int b, tq0, tq_last;
            ft_unit(p, NQ, u, b, tq0, tq_last);
            const int nt = ft_tiles(p, tq_last);
            if (nt == 0) continue;
            const int bb = un & 1, ph = (un >> 1) & 1;
            // per-query constants of the unit for the epilogue
            if (!__all_sync(0xffffffffu, atc::wait(meta_empty + bb, ph ^ 1, abort_flag))) { ok = false; break; }
            bool fast = true;
            for (int c = lane; c < FT_NCOL; c += 32) {
                const int tq = tq0 + c / HI;
                const int wv = tq <= tq_last ? __ldg(fp.wf + ((long long)b * p.Tq + tq) * HI + c % HI) : 1;
                w_s[bb * FT_NCOL + c] = wv;
                fast &= wv == 1;
            }
            for (int q = lane; q < NQ; q += 32) {
                const int tq = tq0 + q;
                const bool v = tq <= tq_last;
                tau_s[bb * FT_NCOL + q] = v ? p.tau[(long long)b * p.Rt + (tq - p.t0)] : INT_MAX;
                nc_s[bb * FT_NCOL + q] = v ? (int)min(n_candidates(p.q_pos0 + tq, p.window), (long long)INT_MAX) : 0;
                cnt_s[bb * FT_NCOL + q] = 0;
            }
            fast = __all_sync(0xffffffffu, fast);
            if (lane == 0) fast_s[bb] = fast ? 1 : 0;
            __syncwarp();
            atc::arrive(meta_full + bb);                 // each lane releases its own writes
            // query block (B operand)
            if (!__all_sync(0xffffffffu, atc::wait(b_empty + bb, ph ^ 1, abort_flag))) { ok = false; break; }
            if (lane == 0) {
                atc::expect_tx(b_full + bb, L::B_BYTES);
                atc::load_2d(smem + L::OFF_B + bb * L::B_BYTES, &bmap, 0, (b * p.Tq + tq0) * HI, b_full + bb);
            }
            ++b_issued;
            // key tiles (A operand)
            for (int k = 0; k < nt; ++k, ++tile) {
                const int st = tile % FT_STAGES;
                if (!__all_sync(0xffffffffu, atc::wait(a_empty + st, ((tile / FT_STAGES) & 1) ^ 1, abort_flag))) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    atc::expect_tx(a_full + st, L::A_BYTES);
                    atc::load_2d(smem + L::OFF_A + st * L::A_BYTES, &amap, 0, b * p.L + k * 128, a_full + st);
                }
            }
            if (ok) ++un;
        }
        if (!ok && lane == 0) fail();
        if (lane == 0) {
            // every issued copy lands before the CTA exits
            for (int i = 0; i < 2 && i < b_issued; ++i) {
                const int ui = b_issued - 1 - i;
                tc::mbar_wait_bounded(b_full + (ui & 1), (ui >> 1) & 1, kDefaultSpinCycles);
            }
            for (int i = 0; i < FT_STAGES && i < tile; ++i) {
                const int ti = tile - 1 - i;
                tc::mbar_wait_bounded(a_full + ti % FT_STAGES, (ti / FT_STAGES) & 1, kDefaultSpinCycles);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            bool ok = true;
            int un = 0, tile = 0;
            for (int u = blockIdx.x; u < fp.n_units && ok; u += gridDim.x) {
                int b, tq0, tq_last;
                ft_unit(p, NQ, u, b, tq0, tq_last);
                const int nt = ft_tiles(p, tq_last);
                if (nt == 0) continue;
                const int bb = un & 1;
                if (!atc::wait(b_full + bb, (un >> 1) & 1, abort_flag)) { ok = false; break; }
                const uint32_t b_addr = tc::smem_u32(smem + L::OFF_B + bb * L::B_BYTES);
                for (int k = 0; k < nt; ++k, ++tile) {
                    const int st = tile % FT_STAGES, ab = tile & 1;
                    if (!atc::wait(a_full + st, (tile / FT_STAGES) & 1, abort_flag) ||
                        !atc::wait(acc_free + ab, ((tile >> 1) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t a_addr = tc::smem_u32(smem + L::OFF_A + st * L::A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < DI / 32; ++kk)
                        tc::mma_i8(tmem + ab * FT_ACC, ft::desc_row_swizzled<DI>(a_addr + kk * 32),
                                   ft::desc_row_swizzled<DI>(b_addr + kk * 32), IDESC, kk > 0 ? 1u : 0u);
                    tc::mma_commit(a_empty + st);
                    tc::mma_commit(acc_full + ab);
                }
                if (!ok) break;
                tc::mma_commit(b_empty + bb);              // the unit's MMAs are done with its query block
                ++un;
            }
            if (!ok) fail();
            tc::mma_commit(drain);                         // every MMA issued here completes first
            tc::mbar_wait_bounded(drain, 0, kDefaultSpinCycles);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        const int ew = warp - 2;                           // 0..15
        const int quad = warp & 3;                         // TMEM lane quadrant
        const int c0 = (ew >> 2) * FT_CW;                  // this warp's columns
        const int q_lo = c0 / HI;                          // its first query (within the unit)
        const uint32_t lrow = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        int un = 0, tile = 0;
        for (int u = blockIdx.x; u < fp.n_units && ok; u += gridDim.x) {
            int b, tq0, tq_last;
            ft_unit(p, NQ, u, b, tq0, tq_last);
            const int nt = ft_tiles(p, tq_last);
            if (nt == 0) continue;
            const int bb = un & 1;
            bool bad = !atc::wait(meta_full + bb, (un >> 1) & 1, abort_flag);
            if (bad) fail();                               // the other roles stop at their next wait
            const bool fast = !bad && fast_s[bb] != 0;
            const int *tau_u = tau_s + bb * FT_NCOL + q_lo;
            const int *nc_u = nc_s + bb * FT_NCOL + q_lo;
            const int *w_u = w_s + bb * FT_NCOL + c0;
            int *cnt_u = cnt_s + bb * FT_NCOL + q_lo;
            const int nc_first = nc_s[bb * FT_NCOL];
            // thresholds in registers; the causal bounds are read from shared
            // memory on the diagonal tiles only
            int tau_r[QREG ? NQT : 1];
            if constexpr (QREG) {
#pragma unroll
                for (int q = 0; q < NQT; ++q) tau_r[q] = fast ? -ft_fast_tau(tau_u[q]) : tau_u[q];   // fast: -tau
            }
            const long long list0 = ((long long)b * p.Rt + (tq0 + q_lo - p.t0)) * p.cand_cap;
            int2 *const lbase = p.cand + list0;             // this warp's first query's list
            const int cap = p.cand_cap;
            const uint32_t cnt_a = tc::smem_u32(cnt_u);
            for (int k = 0; k < nt; ++k, ++tile) {
                const int ab = tile & 1;
                if (!bad && !atc::wait(acc_full + ab, (tile >> 1) & 1, abort_flag)) {
                    bad = true;
                    fail();
                }
                if (bad) continue;                         // stop with the others at the unit's end
                tc::fence_after_sync();
                const int j = k * 128 + quad * 32 + lane;  // this thread's key
                const bool full = (k + 1) * 128 <= nc_first;   // every key visible to every query
                // this warp's columns, 32 at a time (32 registers); the
                // accumulator is released once the last part is loaded
#pragma unroll
                for (int half = 0; half < FT_CW / 32; ++half) {
                    uint32_t x[32];
                    ft::tmem_ld32(tmem + lrow + ab * FT_ACC + c0 + half * 32, x);
                    tc::tmem_ld_wait();
                    if (half == FT_CW / 32 - 1) {
                        tc::fence_before_sync();
                        __syncwarp();
                        if (lane == 0) atc::arrive(acc_free + ab);
                    }
                    constexpr int NQH = 32 / HI;              // queries in a half
                    constexpr int NG = NQH < 8 ? NQH : 8;     // queries per group
                    // per group: the sums first (independent chains), a keep
                    // mask, then the kept pairs go to their queries' lists
#pragma unroll
                    for (int g0 = 0; g0 < NQH; g0 += NG) {
                        const int qb = half * NQH + g0;       // first query of the group (in this warp)
                        int sc[NG];
                        bool keep[NG];
                        if (fast) {
#pragma unroll
                            for (int qq = 0; qq < NG; ++qq) {
                                const int ntau = QREG ? tau_r[qb + qq] : -ft_fast_tau(tau_u[qb + qq]);
                                int sacc = ntau;
#pragma unroll
                                for (int h = 0; h < HI; ++h)
                                    sacc = __viaddmax_s32(sacc, (int)x[(g0 + qq) * HI + h], sacc);
                                sc[qq] = sacc - ntau;
                                keep[qq] = sacc >= 0;
                            }
                        } else {
#pragma unroll
                            for (int qq = 0; qq < NG; ++qq) {
                                int sacc = 0;
#pragma unroll
                                for (int h = 0; h < HI; ++h)
                                    sacc += w_u[(qb + qq) * HI + h] * max((int)x[(g0 + qq) * HI + h], 0);
                                sc[qq] = sacc;
                                keep[qq] = sacc >= (QREG ? tau_r[qb + qq] : tau_u[qb + qq]);
                            }
                        }
                        if (!full) {                           // diagonal tiles: causal bound per query
#pragma unroll
                            for (int qq = 0; qq < NG; ++qq) keep[qq] = keep[qq] && j < nc_u[qb + qq];
                        }
                        // every keeping lane takes its list slot with its own
                        // shared-memory atomic (one per kept pair, ~10% of the
                        // pairs: fewer instructions than reserving a warp's
                        // slots by ballot, shuffle and popcount) and stores
                        // the pair; 32-bit offsets from the unit's list base
#pragma unroll
                        for (int qq = 0; qq < NG; ++qq) {
                            if (keep[qq]) {
                                // past the capacity the row's count marks the list
                                // unusable (the select recomputes the row), so an
                                // overflowing pair may land on the last slot
                                const int slot = ft::atom_add1_shared(cnt_a + 4u * (uint32_t)(qb + qq));
                                lbase[(qb + qq) * cap + min(slot, cap - 1)] = make_int2(sc[qq], j);
                            }
                        }
                    }
                }
            }
            // unit end: every epilogue thread agrees (a failed wait anywhere
            // stops all of them here), then the list lengths go out
            if (!atc::agree(1, FT_EPI_WARPS * 32, !bad)) { ok = false; break; }
            const int e = tid - 64;
            if (e < NQ && tq0 + e <= tq_last)
                p.cand_cnt[(long long)b * p.Rt + (tq0 + e - p.t0)] = cnt_s[bb * FT_NCOL + e];
            atc::arrive(meta_empty + bb);
            ++un;
        }
        if (!ok) fail();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, FT_TM_COLS);
}

}  // namespace sa
