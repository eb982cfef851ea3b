// full_score.cuh -- a full-attention layer as an exact indexer for the
// sparse layers (HySparse2 page, "Xiaomi presenta HySparse2 ...", section
// "Que significa para la evolucion de la IA": a few full-attention layers
// compute exact scores and guide the selection of the sparse ones).
//
// The full layer's causal attention (out, lse) comes from the tile attention
// kernels with a window as long as the sequence.  The exact score of key j
// for query t is the probability mass the full layer puts on j, summed over
// all of its heads:
//   score(t, j) = sum_h exp2(scale_log2 * q_{t,h} . k_{j,g(h)} - lse2_{t,h})
// full_score_kernel writes it, as the bit pattern of the non-negative fp32
// value (which orders like the value), for every non-window candidate
// j < n_candidates(t) of a chunk of query rows; the exact radix select
// (topk_select_kernel in its dense mode) then takes the top-k by
// (score desc, j asc) and appends the forced window.
//
// One CTA = 8 consecutive queries, one warp each; the CTA stages chunks of
// 64 keys of one KV group by cp.async (two stages, XOR-swizzled 16-byte
// units) and every warp multiplies its query's 16-head tile by them
// (mma.sync m16n8k16, bf16 -> fp32).  P = exp2(S - lse2) and its column sums
// over the heads stay in fp32 (shuffles across the row groups of the
// fragment).  Groups are the outer loop; a group after the first adds to the
// scores the same lanes wrote for the previous one.
//
// full_score_tc_kernel is the same pass on the tcgen05 tensor cores for head
// dim 128 and 16 query heads per KV head, key-major: a 128-key tile of K is
// the M side and the 16 queries x 16 heads of a query block the N side,
//   S^T[128 keys x 256 (query, head)] = K_tile . Q_blk^T     (kind::f16)
// into one of two 256-column TMEM buffers.  A score thread owns one key (one
// TMEM lane) and eight queries, so the sum over the heads is a sum of the 16
// columns of a query in its own registers: no shuffles; a warp stores 128
// bytes of a dense row per query.  Warp roles (320 threads, one persistent
// CTA per SM): warp 0 loads the block's Q (TMA) and lse (bulk copies) and a
// 4-stage ring of K tiles; warp 1 issues the MMAs and owns the TMEM; warps
// 2-9 are the score warps (two per TMEM lane quadrant, queries 0-7 / 8-15).
// Work items are (batch element, 16-query block, piece of <= 32 key tiles),
// pieces the slowest index.  Every wait is bounded; on a timeout the kernel
// records ERR_TIMEOUT, stops issuing work, lets its own copies and MMAs
// finish (bounded) and frees its TMEM.
#pragma once

#include "attn_tc.cuh"
#include "sa_common.cuh"

namespace sa {

struct FullScoreParams {
    const __nv_bfloat16 *q, *k;   // q [B,T,Hq,D], k [B,T,Hkv,D]
    const float *lse;             // [B,T,Hq] natural log (the full layer's)
    int B, T, Hq, Hkv, G;
    int t0, Rt;                   // query rows t0 .. t0+Rt-1 of every batch element
    int window;                   // forced recent keys (not scored)
    float scale_log2;
    int32_t *dense;               // [B, Rt, stride]: fp32 bits of score(t, j), j < n_candidates(t)
    long long stride;
};

constexpr int FS_WARPS = 8;       // queries per CTA
constexpr int FS_NK = 64;         // keys per chunk

template <int D>
constexpr int full_score_smem() {
    return 2 * FS_NK * D * 2;
}

__device__ __forceinline__ long long fs_candidates(long long t, int window) {
    const long long n = window > 0 ? t - window + 1 : t + 1;
    return n > 0 ? n : 0;
}

template <int D>
__global__ void __launch_bounds__(FS_WARPS * 32, 2) full_score_kernel(const FullScoreParams p) {
    grid_dependency_sync();
    constexpr int ROWB = D * 2;
    constexpr int UNITS = ROWB / 16;
    constexpr int CH = FS_NK * ROWB;
    constexpr int KS_D = D / 16;
    constexpr int CP_ITERS = FS_NK * UNITS / (FS_WARPS * 32);
    static_assert(CP_ITERS * FS_WARPS * 32 == FS_NK * UNITS, "copy split");
    extern __shared__ __align__(1024) unsigned char smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, qc = lane & 3;
    const int nqb = (p.Rt + FS_WARPS - 1) / FS_WARPS;
    const int b = blockIdx.x / nqb, qb = blockIdx.x % nqb;
    const int tr = qb * FS_WARPS + warp;
    const long long t = (long long)p.t0 + tr;
    const bool valid = tr < p.Rt && t < p.T;
    const long long n_w = valid ? fs_candidates(t, p.window) : 0;
    // the block's last query has the most candidates
    int tr_last = min(qb * FS_WARPS + FS_WARPS, p.Rt) - 1;
    long long t_last = (long long)p.t0 + tr_last;
    if (t_last > p.T - 1) t_last = p.T - 1;
    const long long n_max = fs_candidates(t_last, p.window);
    const int n_chunks = (int)((n_max + FS_NK - 1) / FS_NK);
    const int n_hc = (p.G + 15) / 16;
    int32_t *drow = p.dense + ((long long)b * p.Rt + (valid ? tr : 0)) * p.stride;

    // Q A fragments of a 16-head chunk (rows past the group are zero)
    auto load_q = [&](int g, int hc, unsigned (&qa)[KS_D][4]) {
        const int h0 = g * p.G + hc * 16;
        const bool r0 = hc * 16 + gr < p.G, r1 = hc * 16 + gr + 8 < p.G;
        const __nv_bfloat16 *qrow = p.q + ((long long)(b * p.T + (valid ? t : 0)) * p.Hq + h0) * D;
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
            const int c0 = ks * 16 + 2 * qc;
            qa[ks][0] = r0 ? __ldg(reinterpret_cast<const unsigned *>(qrow + (long long)gr * D + c0)) : 0u;
            qa[ks][1] = r1 ? __ldg(reinterpret_cast<const unsigned *>(qrow + (long long)(gr + 8) * D + c0)) : 0u;
            qa[ks][2] = r0 ? __ldg(reinterpret_cast<const unsigned *>(qrow + (long long)gr * D + c0 + 8)) : 0u;
            qa[ks][3] = r1 ? __ldg(reinterpret_cast<const unsigned *>(qrow + (long long)(gr + 8) * D + c0 + 8)) : 0u;
        }
    };
    unsigned qa[KS_D][4];

    for (int g = 0; g < p.Hkv; ++g) {
        const __nv_bfloat16 *kb = p.k + ((long long)b * p.T * p.Hkv + g) * D;
        // one head chunk (G <= 16): its fragments stay in registers for the whole key loop
        if (n_hc == 1 && valid) load_q(g, 0, qa);
        const long long rstride = (long long)p.Hkv * D;
        auto issue = [&](int ci) {
            if (ci < n_chunks) {
                unsigned char *dst = smem + (ci & 1) * CH;
#pragma unroll
                for (int it = 0; it < CP_ITERS; ++it) {
                    const int lin = (it * FS_WARPS + warp) * 32 + lane;
                    const int r = lin / UNITS, u = lin % UNITS;
                    const long long j = (long long)ci * FS_NK + r;
                    const bool ok = j < n_max;
                    cp_async16(dst + r * ROWB + ((u ^ (r & 7)) * 16), ok ? kb + j * rstride + u * 8 : kb,
                               ok ? 16 : 0);
                }
            }
            cp_async_commit();
        };
        issue(0);
        for (int ci = 0; ci < n_chunks; ++ci) {
            issue(ci + 1);
            cp_async_wait<1>();
            __syncthreads();
            const long long j0 = (long long)ci * FS_NK;
            if (j0 < n_w) {
                const unsigned char *ks_ = smem + (ci & 1) * CH;
                float acc[8][2];
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
                for (int hc = 0; hc < n_hc; ++hc) {
                    const int h0 = g * p.G + hc * 16;
                    const bool r0 = hc * 16 + gr < p.G, r1 = hc * 16 + gr + 8 < p.G;
                    const float *lrow = p.lse + (long long)(b * p.T + t) * p.Hq + h0;
                    const float l0 = r0 ? lrow[gr] * kLog2e : 0.f, l1 = r1 ? lrow[gr + 8] * kLog2e : 0.f;
                    if (n_hc > 1) load_q(g, hc, qa);
                    float sc[8][4];
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
                    for (int ks = 0; ks < KS_D; ++ks) {
                        const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
                        for (int kg = 0; kg < 4; ++kg) {
                            const int key = kg * 16 + (mi >> 1) * 8 + ri;
                            const int unit = ks * 2 + (mi & 1);
                            unsigned b0, b1, b2, b3;
                            ldsm_x4(b0, b1, b2, b3, ks_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                            mma_bf16_16816(sc[2 * kg], qa[ks], b0, b1);
                            mma_bf16_16816(sc[2 * kg + 1], qa[ks], b2, b3);
                        }
                    }
                    // P of the two rows of each column, summed over the 16 heads
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const long long j = j0 + nt * 8 + 2 * qc + c;
                            const bool kj = j < n_w;
                            float s = 0.f;
                            if (kj && r0) s += ex2_fast(sc[nt][c] * p.scale_log2 - l0);
                            if (kj && r1) s += ex2_fast(sc[nt][2 + c] * p.scale_log2 - l1);
                            s += __shfl_xor_sync(0xffffffffu, s, 4);
                            s += __shfl_xor_sync(0xffffffffu, s, 8);
                            s += __shfl_xor_sync(0xffffffffu, s, 16);
                            acc[nt][c] += s;
                        }
                    }
                }
                // lane (gr, qc) stores columns gr*8 + 2qc, +1: one coalesced 256-byte row piece
                float v0 = 0.f, v1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
                    if (nt == gr) { v0 = acc[nt][0]; v1 = acc[nt][1]; }
                const long long j = j0 + gr * 8 + 2 * qc;
                if (g > 0) {
                    if (j < n_w) v0 += __int_as_float(drow[j]);
                    if (j + 1 < n_w) v1 += __int_as_float(drow[j + 1]);
                }
                if (j + 1 < n_w) {
                    *reinterpret_cast<int2 *>(drow + j) = make_int2(__float_as_int(v0), __float_as_int(v1));
                } else if (j < n_w) {
                    drow[j] = __float_as_int(v0);
                }
            }
            __syncthreads();
        }
        cp_async_wait<0>();
        __syncthreads();
    }
}

// ------------------------------------------------- tcgen05 form (d = 128)
constexpr int FX_QB = 16;                 // queries per block (x 16 heads = 256 columns)
constexpr int FX_KT = 128;                // keys per tile
constexpr int FX_KSTAGES = 4;
constexpr int FX_PIECE = 32;              // key tiles per work item
constexpr int FX_THREADS = 320;
constexpr uint32_t FX_TM_COLS = 512;      // two S buffers of 256 columns

struct FxSmem {
    static constexpr int Q_BYTES = FX_QB * 16 * 256;      // 2 halves x 256 rows x 128 B
    static constexpr int K_BYTES = FX_KT * 256;           // 2 halves x 128 rows x 128 B
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_LSE = OFF_K + FX_KSTAGES * K_BYTES;   // [16 queries][16 heads] natural lse
    static constexpr int OFF_NL = OFF_LSE + FX_QB * 16 * 4;       // per score warp: -lse * log2(e) of its 8 queries
    static constexpr int OFF_BAR = OFF_NL + 8 * 8 * 16 * 4;
    // q_full, q_empty, lse_free, k_full[S], k_empty[S], s_full[2], s_empty[2], drain
    static constexpr int N_BAR = 3 + 2 * FX_KSTAGES + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;           // tmem slot, abort flag
    static constexpr int TOTAL = OFF_MISC + 16;
    static constexpr int ALLOC = TOTAL + 1024;
};

struct FxParams {
    FullScoreParams f;
    int nqb;            // query blocks per batch element (ceil(Rt / 16))
    int n_items;        // n_piece * B * nqb
    unsigned *err;
};

// Item -> (b, query block, first key tile, tile count); 0 = empty item.
// Pieces are the slow index, so every block's first piece comes first.
__device__ __forceinline__ int fx_item(const FxParams &cp, int it, int &b, int &qb, int &kt0) {
    const FullScoreParams &p = cp.f;
    const int per = p.B * cp.nqb;
    const int s = it / per, r = it % per;
    b = r / cp.nqb;
    qb = r % cp.nqb;
    const int tr_last = min(qb * FX_QB + FX_QB, p.Rt) - 1;
    const long long n_max = fs_candidates((long long)p.t0 + tr_last, p.window);
    const int n_kt = (int)((n_max + FX_KT - 1) / FX_KT);
    kt0 = s * FX_PIECE;
    return kt0 < n_kt ? min(FX_PIECE, n_kt - kt0) : 0;
}

__global__ void __launch_bounds__(FX_THREADS, 1)
    full_score_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                         const FxParams cp) {
    grid_dependency_sync();
    using L = FxSmem;
    const FullScoreParams &p = cp.f;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *q_full = bars, *q_empty = bars + 1, *lse_free = bars + 2;
    uint64_t *k_full = bars + 3, *k_empty = k_full + FX_KSTAGES;
    uint64_t *s_full = k_empty + FX_KSTAGES, *s_empty = s_full + 2, *drain = s_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, FX_TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(q_full, 1); tc::mbar_init(q_empty, 1); tc::mbar_init(lse_free, 256);
        for (int i = 0; i < FX_KSTAGES; ++i) { tc::mbar_init(k_full + i, 1); tc::mbar_init(k_empty + i, 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(s_full + i, 1); tc::mbar_init(s_empty + i, 256); }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() {
        raise_error(cp.err, ERR_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int qn = 0, kn = 0;                           // Q blocks and K tiles issued
            const int n_items = debug_stall() ? 0 : cp.n_items;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                int b, qb, kt0;
                const int nt = fx_item(cp, it, b, qb, kt0);
                if (nt == 0) continue;
                const int tb = p.t0 + qb * FX_QB;         // first query of the block
                for (int g = 0; g < p.Hkv && ok; ++g) {
                    // the previous block's last MMA and last score reads are done
                    if (qn > 0 && (!atc::wait(q_empty, (qn - 1) & 1, abort_flag) ||
                                   !atc::wait(lse_free, (qn - 1) & 1, abort_flag))) { ok = false; break; }
                    atc::expect_tx(q_full, L::Q_BYTES + FX_QB * 64);
                    for (int w = 0; w < FX_QB; ++w) {
                        // queries past the sequence load the last one (masked by the score warps)
                        const int tw = min(tb + w, p.T - 1);
                        const int qrow = (b * p.T + tw) * p.Hq + g * 16;
                        for (int h = 0; h < 2; ++h)
                            atc::load_2d(smem + L::OFF_Q + h * (FX_QB * 16 * 128) + w * (16 * 128), &qmap, h * 64,
                                         qrow, q_full);
                        asm volatile(
                            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                                tc::smem_u32(smem + L::OFF_LSE + w * 64)),
                            "l"(p.lse + (long long)qrow), "r"(64), "r"(tc::smem_u32(q_full))
                            : "memory");
                    }
                    ++qn;
                    for (int i = 0; i < nt; ++i) {
                        const int ks = kn % FX_KSTAGES;
                        if (!atc::wait(k_empty + ks, ((kn / FX_KSTAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                        atc::expect_tx(k_full + ks, L::K_BYTES);
                        const int z = b * p.T + (kt0 + i) * FX_KT;
                        for (int h = 0; h < 2; ++h)
                            atc::load_3d(smem + L::OFF_K + ks * L::K_BYTES + h * (FX_KT * 128), &kmap, h * 64, g, z,
                                         k_full + ks);
                        ++kn;
                    }
                }
            }
            if (!ok) fail();
            // let the copies land before the CTA exits
            if (qn > 0) tc::mbar_wait_bounded(q_full, (qn - 1) & 1, ATC_WAIT);
            for (int i = 0; i < FX_KSTAGES && i < kn; ++i) {
                const int q = kn - 1 - i;
                tc::mbar_wait_bounded(k_full + q % FX_KSTAGES, (q / FX_KSTAGES) & 1, ATC_WAIT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t ID = tc::make_idesc(1, 1, 128, 256);
            const uint32_t qa = tc::smem_u32(smem + L::OFF_Q);
            bool ok = true;
            int qn = 0, kn = 0;
            for (int it = blockIdx.x; it < cp.n_items && ok; it += gridDim.x) {
                int b, qb, kt0;
                const int nt = fx_item(cp, it, b, qb, kt0);
                if (nt == 0) continue;
                for (int g = 0; g < p.Hkv && ok; ++g) {
                    if (!atc::wait(q_full, qn & 1, abort_flag)) { ok = false; break; }
                    ++qn;
                    for (int i = 0; i < nt; ++i) {
                        const int ks = kn % FX_KSTAGES, sb = kn & 1;
                        if (!atc::wait(k_full + ks, (kn / FX_KSTAGES) & 1, abort_flag)) { ok = false; break; }
                        // buffer sb was last read by the score warps for tile kn - 2
                        if (kn >= 2 && !atc::wait(s_empty + sb, ((kn >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                        tc::fence_after_sync();
                        const uint32_t ka = tc::smem_u32(smem + L::OFF_K + ks * L::K_BYTES);
#pragma unroll
                        for (int kq = 0; kq < 8; ++kq) {
                            const int h = kq / 4, kk = kq % 4;
                            const uint64_t ad = atc::desc_sw128(ka + h * (FX_KT * 128) + kk * 32, 16, 1024);
                            const uint64_t bd = atc::desc_sw128(qa + h * (FX_QB * 16 * 128) + kk * 32, 16, 1024);
                            tc::mma_bf16(tmem + sb * 256, ad, bd, ID, kq > 0 ? 1u : 0u);
                        }
                        tc::mma_commit(k_empty + ks);
                        tc::mma_commit(s_full + sb);
                        ++kn;
                    }
                    if (!ok) break;
                    tc::mma_commit(q_empty);
                }
            }
            if (!ok) fail();
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, ATC_WAIT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ score warps
        // Thread = one key of the tile (TMEM lane); the two warps of a lane
        // quadrant take the block's queries 0-7 / 8-15 (columns 0-127 / 128-255).
        const int quad = warp & 3, half = (warp - 2) >> 2;
        const int kr = quad * 32 + lane;
        const uint32_t lrow = (uint32_t)(quad * 32) << 16;
        const float4 *ls = reinterpret_cast<const float4 *>(smem + L::OFF_LSE) + half * 8 * 4;
        float4 *nl = reinterpret_cast<float4 *>(smem + L::OFF_NL) + (warp - 2) * 8 * 4;
        bool ok = true;
        int qn = 0, kn = 0;
        for (int it = blockIdx.x; it < cp.n_items && ok; it += gridDim.x) {
            int b, qb, kt0;
            const int nt = fx_item(cp, it, b, qb, kt0);
            if (nt == 0) continue;
            // this thread's eight queries: chunk rows trb .. trb + 7 and their candidate counts
            const int trb = qb * FX_QB + half * 8;
            int nw[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                nw[u] = trb + u < p.Rt ? (int)fs_candidates((long long)p.t0 + trb + u, p.window) : 0;
            int32_t *drow = p.dense + ((long long)b * p.Rt + min(trb, p.Rt - 1)) * p.stride;
            for (int g = 0; g < p.Hkv && ok; ++g) {
                // the block's Q and lse (the wait makes the lse copy visible)
                if (!__all_sync(0xffffffffu, atc::wait(q_full, qn & 1, abort_flag))) { ok = false; break; }
                ++qn;
                {   // this warp's copy of -lse * log2(e) for its 8 queries x 16 heads
                    const float4 l = ls[lane];
                    nl[lane] = make_float4(-l.x * kLog2e, -l.y * kLog2e, -l.z * kLog2e, -l.w * kLog2e);
                    __syncwarp();
                }
                for (int i = 0; i < nt; ++i) {
                    const int sb = kn & 1;
                    if (!__all_sync(0xffffffffu, atc::wait(s_full + sb, (kn >> 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const int j = (kt0 + i) * FX_KT + kr;
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        uint32_t sr[64];
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tc::tmem_ld16(tmem + lrow + sb * 256 + half * 128 + part * 64 + c * 16,
                                          *reinterpret_cast<uint32_t(*)[16]>(sr + c * 16));
                        tc::tmem_ld_wait();
                        if (part == 1) {
                            tc::fence_before_sync();
                            atc::arrive(s_empty + sb);
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int u = part * 4 + c;
                            float acc = 0.f;
#pragma unroll
                            for (int h4 = 0; h4 < 4; ++h4) {
                                const float4 l = nl[u * 4 + h4];
                                const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float x = fmaf(__uint_as_float(sr[c * 16 + h4 * 4 + e]), p.scale_log2, lv[e]);
                                    acc += ex2_fast(x);
                                }
                            }
                            if (j < nw[u]) {
                                int32_t *dp = drow + (long long)u * p.stride + j;
                                *dp = __float_as_int(g > 0 ? acc + __int_as_float(*dp) : acc);
                            }
                        }
                    }
                    ++kn;
                }
                if (!ok) break;
                atc::arrive(lse_free);
            }
        }
        if (!ok) fail();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, FX_TM_COLS);
}

// fp32 -> bf16 rows (the full layer's output)
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float *__restrict__ x, long long n2,
                                                          __nv_bfloat16 *__restrict__ y) {
    grid_dependency_sync();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n2) return;
    const float2 v = reinterpret_cast<const float2 *>(x)[i];
    reinterpret_cast<__nv_bfloat162 *>(y)[i] = __floats2bfloat162_rn(v.x, v.y);
}

}  // namespace sa
