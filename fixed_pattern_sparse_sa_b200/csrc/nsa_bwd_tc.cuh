// nsa_bwd_tc.cuh -- dq of the NSA compressed and window branches on the
// tcgen05 tensor cores (Native Sparse Attention page, "Puntos Clave":
// natively trainable, with a faster backward pass; "Diseno Consciente del
// Hardware": tensor-core-aligned, group-centric loading).
//
// The backward of a range branch for 8 consecutive queries of a KV group
// (8 x 16 heads = 128 rows, the TMEM lanes), as nsa_tc_kernel runs its
// forward: the keys visible to any of the 8 queries are one contiguous range
// (compressed rows 0 .. n_vis(t_last), or the union of the windows), walked
// in tiles of 64 keys.  Per tile one thread issues
//   S  = Q K_hi^T (+ Q K_lo^T)   and   dP = dO V^T      (N = 64 keys)
// into tensor memory; the score warps form
//   dS = gate * P * (dP - D),  P = exp2(S * scale_log2 - lse2)
// with the forward's lse (no running maximum: the LSE is known), masked to
// each row's visible keys, and store it as bf16 pairs in tensor memory; the
// MMA thread then adds dq += dS K_hi (+ dS K_lo), K read as an MN-major B
// operand.  dq (128 fp32 columns) is scaled and added to the global dq once
// per item.  D = dout . O_branch and the gates come from the caller.
//
// Q, dO and the K_hi / K_lo / V tiles arrive by TMA box loads in the
// 128B-swizzled canonical layouts (two 64-column halves).  Warps: 0 TMA
// producer, 1 MMA issuer and TMEM owner, 2-9 score warps (two per TMEM lane
// quadrant, 32 key columns and 64 dq columns each).  Every wait is bounded; a
// timeout sets ERR_TIMEOUT and the CTA drains and exits.
#pragma once

#include "attn_bwd.cuh"
#include "attn_cmp_tc.cuh"

namespace sa {

constexpr int DQ_KT = 64;               // keys per tile
constexpr int DQ_STAGES = 3;
constexpr int DQ_THREADS = 320;
constexpr uint32_t DQ_TM_S = 0;         // S: 2 buffers x 64 fp32 columns
constexpr uint32_t DQ_TM_DP = 128;      // dP: 2 buffers x 64
constexpr uint32_t DQ_TM_DS = 256;      // dS: 2 buffers x 32 columns (bf16 pairs)
constexpr uint32_t DQ_TM_Q = 384;       // dq: 128 fp32 columns
constexpr uint32_t DQ_TM_COLS = 512;

struct DqSmem {                         // head dim 128
    static constexpr int Q_BYTES = 128 * 256;             // 2 halves x 128 rows x 128 B
    static constexpr int KT_BYTES = DQ_KT * 256;          // one K (or V) tile: 2 halves x 64 rows x 128 B
    static constexpr int STAGE = 3 * KT_BYTES;            // K_hi | K_lo | V
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_DO = OFF_Q + Q_BYTES;
    static constexpr int OFF_KV = OFF_DO + Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + DQ_STAGES * STAGE;
    // q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], s_free[2], ds_full[2],
    // ds_done[2], dq_full, dq_free, drain
    static constexpr int N_BAR = 2 + 2 * DQ_STAGES + 8 + 3;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
    static constexpr int TOTAL = OFF_MISC + 16;
    static constexpr int ALLOC = TOTAL + 1024;
};

struct DqTcParams {
    TileParams t;            // q, k (K_hi), klo, v, shapes, window / cmp_len / cmp_stride, scale_log2
    const float *lse;        // the branch's lse: lse[row * lse_stride]
    const float *Dt;         // dout . O_branch per row
    const float *gate;       // gate[row * gate_stride]
    int lse_stride, gate_stride;
    float *dq;               // [B, T, Hq, 128] fp32
    int dq_accum;
    float scale;
    unsigned *err;
    int n_items;             // B * Hkv * ceil(T / 8)
};

template <int SRC>
__global__ void __launch_bounds__(DQ_THREADS, 1)
    nsa_dq_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap domap,
                     const __grid_constant__ CUtensorMap khimap, const __grid_constant__ CUtensorMap klomap,
                     const __grid_constant__ CUtensorMap vmap, const DqTcParams cp) {
    grid_dependency_sync();
    constexpr int D = 128;
    constexpr bool LO = SRC == TS_CMP;
    using L = DqSmem;
    const TileParams &p = cp.t;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *q_full = bars, *q_empty = bars + 1, *kv_full = bars + 2, *kv_empty = kv_full + DQ_STAGES;
    uint64_t *s_full = kv_empty + DQ_STAGES, *s_free = s_full + 2, *ds_full = s_free + 2, *ds_done = ds_full + 2;
    uint64_t *dq_full = ds_done + 2, *dq_free = dq_full + 1, *drain = dq_free + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, DQ_TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(q_full, 1); tc::mbar_init(q_empty, 1);
        for (int i = 0; i < DQ_STAGES; ++i) { tc::mbar_init(kv_full + i, 1); tc::mbar_init(kv_empty + i, 1); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(s_full + i, 1); tc::mbar_init(s_free + i, 256);
            tc::mbar_init(ds_full + i, 256); tc::mbar_init(ds_done + i, 1);
        }
        tc::mbar_init(dq_full, 1); tc::mbar_init(dq_free, 256);
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
    auto key_lo = [&](int t0) -> int { return SRC == TS_CMP ? 0 : max(0, t0 - p.window + 1); };
    auto tiles_of = [&](int t0) -> int {
        const int t_last = min(t0 + CT_Q - 1, p.T - 1);
        return ((int)tile_key_end<SRC>(p, t_last) - key_lo(t0) + DQ_KT - 1) / DQ_KT;
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int tile = 0, qn = 0;
            const int n_items = debug_stall() ? 0 : cp.n_items;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                int b, g, t0;
                ct_item(p, it, b, g, t0);
                const int nt = tiles_of(t0);
                if (nt == 0) continue;
                if (!atc::wait(q_empty, (qn & 1) ^ 1, abort_flag)) { ok = false; break; }
                atc::expect_tx(q_full, 2 * L::Q_BYTES);
                for (int w = 0; w < CT_Q; ++w) {
                    const int qrow = (b * p.T + min(t0 + w, p.T - 1)) * p.Hq + g * p.G;
                    for (int h = 0; h < 2; ++h) {
                        atc::load_2d(smem + L::OFF_Q + h * (128 * 128) + w * (16 * 128), &qmap, h * 64, qrow, q_full);
                        atc::load_2d(smem + L::OFF_DO + h * (128 * 128) + w * (16 * 128), &domap, h * 64, qrow, q_full);
                    }
                }
                ++qn;
                for (int kt = 0; kt < nt; ++kt, ++tile) {
                    const int st = tile % DQ_STAGES;
                    if (!atc::wait(kv_empty + st, ((tile / DQ_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    atc::expect_tx(kv_full + st, LO ? L::STAGE : 2 * L::KT_BYTES);
                    unsigned char *dst = smem + L::OFF_KV + st * L::STAGE;
                    const int z = b * p.Lk + key_lo(t0) + kt * DQ_KT;
                    for (int h = 0; h < 2; ++h) {
                        atc::load_3d(dst + h * (DQ_KT * 128), &khimap, h * 64, g, z, kv_full + st);
                        if (LO) atc::load_3d(dst + L::KT_BYTES + h * (DQ_KT * 128), &klomap, h * 64, g, z, kv_full + st);
                        atc::load_3d(dst + 2 * L::KT_BYTES + h * (DQ_KT * 128), &vmap, h * 64, g, z, kv_full + st);
                    }
                }
            }
            if (!ok) fail();
            // let the copies land before the CTA exits
            if (qn > 0) tc::mbar_wait_bounded(q_full, (qn - 1) & 1, ATC_WAIT);
            for (int i = 0; i < DQ_STAGES && i < tile; ++i) {
                const int kt = tile - 1 - i;
                tc::mbar_wait_bounded(kv_full + kt % DQ_STAGES, (kt / DQ_STAGES) & 1, ATC_WAIT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::make_idesc(1, 1, 128, DQ_KT);
            constexpr uint32_t ID_Q = tc::make_idesc(1, 1, 128, D) | (1u << 16);   // B (K) MN-major
            const uint32_t qa = tc::smem_u32(smem + L::OFF_Q);
            const uint32_t da = tc::smem_u32(smem + L::OFF_DO);
            bool ok = true;
            int tile = 0, qn = 0, on = 0;
            // S and dP of tile tl into buffer tl & 1
            auto issue_s = [&](int tl) -> bool {
                const int st = tl % DQ_STAGES, sb = tl & 1;
                if (!atc::wait(kv_full + st, (tl / DQ_STAGES) & 1, abort_flag)) return false;
                if (!atc::wait(s_free + sb, ((tl >> 1) & 1) ^ 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t ka = tc::smem_u32(smem + L::OFF_KV + st * L::STAGE);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int h = ks / 4, kk = ks % 4;
                    const uint64_t aq = atc::desc_sw128(qa + h * (128 * 128) + kk * 32, 16, 1024);
                    const uint64_t ad = atc::desc_sw128(da + h * (128 * 128) + kk * 32, 16, 1024);
                    const uint64_t bh = atc::desc_sw128(ka + h * (DQ_KT * 128) + kk * 32, 16, 1024);
                    const uint64_t bl = atc::desc_sw128(ka + L::KT_BYTES + h * (DQ_KT * 128) + kk * 32, 16, 1024);
                    const uint64_t bv = atc::desc_sw128(ka + 2 * L::KT_BYTES + h * (DQ_KT * 128) + kk * 32, 16, 1024);
                    tc::mma_bf16(tmem + DQ_TM_S + sb * DQ_KT, aq, bh, ID_S, ks > 0 ? 1u : 0u);
                    if (LO) tc::mma_bf16(tmem + DQ_TM_S + sb * DQ_KT, aq, bl, ID_S, 1u);
                    tc::mma_bf16(tmem + DQ_TM_DP + sb * DQ_KT, ad, bv, ID_S, ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(s_full + sb);
                return true;
            };
            for (int it = blockIdx.x; it < cp.n_items && ok; it += gridDim.x) {
                int b, g, t0;
                ct_item(p, it, b, g, t0);
                const int nt = tiles_of(t0);
                if (nt == 0) continue;
                if (!atc::wait(q_full, qn & 1, abort_flag)) { ok = false; break; }
                ++qn;
                if (!issue_s(tile)) { ok = false; break; }
                // the previous item's epilogue must have read dq before it is overwritten
                if (on > 0 && !atc::wait(dq_free, (on - 1) & 1, abort_flag)) { ok = false; break; }
                for (int kt = 0; kt < nt; ++kt, ++tile) {
                    const int st = tile % DQ_STAGES, db = tile & 1;
                    if (kt + 1 < nt && !issue_s(tile + 1)) { ok = false; break; }
                    if (kt + 1 == nt) tc::mma_commit(q_empty);   // Q and dO are free once the last S / dP is done
                    if (!atc::wait(ds_full + db, (tile >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    // dq += dS K: dS (A) from tensor memory, K (B) MN-major from shared memory
                    const uint32_t ka = tc::smem_u32(smem + L::OFF_KV + st * L::STAGE);
#pragma unroll
                    for (int kk = 0; kk < DQ_KT / 16; ++kk) {
                        const uint32_t adS = tmem + DQ_TM_DS + db * (DQ_KT / 2) + kk * 8;
                        const uint64_t bh = atc::desc_sw128(ka + kk * 2048, DQ_KT * 128, 1024);
                        tc::mma_bf16_ts(tmem + DQ_TM_Q, adS, bh, ID_Q, (kt > 0 || kk > 0) ? 1u : 0u);
                        if (LO) {
                            const uint64_t bl = atc::desc_sw128(ka + L::KT_BYTES + kk * 2048, DQ_KT * 128, 1024);
                            tc::mma_bf16_ts(tmem + DQ_TM_Q, adS, bl, ID_Q, 1u);
                        }
                    }
                    tc::mma_commit(kv_empty + st);
                    tc::mma_commit(ds_done + db);
                    if (kt + 1 == nt) tc::mma_commit(dq_full);
                }
                ++on;
            }
            if (!ok) fail();
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, ATC_WAIT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ score warps
        // Two warps per TMEM lane quadrant share its 32 rows: half 0 takes
        // key columns 0-31 of each tile and dq columns 0-63, half 1 the rest.
        // The pair agrees on each wait through a 64-thread named barrier.
        const int quad = warp & 3, half = (warp - 2) >> 2;
        const int pair = 1 + quad;
        constexpr int SC = DQ_KT / 2, OC = D / 2;
        const int r = quad * 32 + lane;                   // row = query w x 16 + head h
        const int w = r >> 4, h = r & 15;
        const uint32_t lrow = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        int tile = 0, on = 0;
        for (int it = blockIdx.x; it < cp.n_items && ok; it += gridDim.x) {
            int b, g, t0;
            ct_item(p, it, b, g, t0);
            const int nt = tiles_of(t0);
            const int t_last = min(t0 + CT_Q - 1, p.T - 1);
            const int t = t0 + w;
            const bool row_ok = t <= t_last && h < p.G;
            const long long orow = row_ok ? (long long)(b * p.T + t) * p.Hq + g * p.G + h : 0;
            // the row's lse (base 2), D and gate; a row with no key has lse = -inf
            const float lse = row_ok ? cp.lse[orow * cp.lse_stride] : -INFINITY;
            const bool live = row_ok && lse != -INFINITY;
            const float nb = live ? -lse * kLog2e : 0.f;
            const float Dr = row_ok ? cp.Dt[orow] : 0.f;
            const float gr_ = row_ok ? (cp.gate ? cp.gate[orow * cp.gate_stride] : 1.f) : 0.f;
            // visible keys of this row as item-relative indices [vlo, vhi)
            const int klo = key_lo(t0);
            const int vhi = live ? (int)tile_key_end<SRC>(p, t) - klo : 0;
            const int vlo = (live && SRC == TS_WINDOW) ? max(0, t - p.window + 1) - klo : 0;
            for (int kt = 0; kt < nt; ++kt, ++tile) {
                const int sb = tile & 1;
                bool got = atc::wait(s_full + sb, (tile >> 1) & 1, abort_flag);
                // dS buffer sb was last read by the dq MMA of tile - 2
                if (got && tile >= 2) got = atc::wait(ds_done + sb, ((tile >> 1) & 1) ^ 1, abort_flag);
                if (!atc::agree(pair, 64, got)) { ok = false; break; }
                tc::fence_after_sync();
                uint32_t sr[SC], dr[SC];
#pragma unroll
                for (int c = 0; c < SC; c += 16) {
                    tc::tmem_ld16(tmem + lrow + DQ_TM_S + sb * DQ_KT + half * SC + c,
                                  *reinterpret_cast<uint32_t(*)[16]>(sr + c));
                    tc::tmem_ld16(tmem + lrow + DQ_TM_DP + sb * DQ_KT + half * SC + c,
                                  *reinterpret_cast<uint32_t(*)[16]>(dr + c));
                }
                tc::tmem_ld_wait();
                tc::fence_before_sync();
                atc::arrive(s_free + sb);
                const int i0 = kt * DQ_KT + half * SC;
                uint32_t pk[SC / 2];
#pragma unroll
                for (int k = 0; k < SC; k += 2) {
                    float ds2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int i = i0 + k + e;
                        const bool vis = i >= vlo && i < vhi;
                        const float pv = vis ? ex2_fast(fmaf(__uint_as_float(sr[k + e]), p.scale_log2, nb)) : 0.f;
                        ds2[e] = pv * gr_ * (__uint_as_float(dr[k + e]) - Dr);
                    }
                    pk[k / 2] = pack_bf16(ds2[0], ds2[1]);
                }
                atc::tmem_st16(tmem + lrow + DQ_TM_DS + sb * (DQ_KT / 2) + half * (SC / 2),
                               *reinterpret_cast<const uint32_t(*)[16]>(pk));
                atc::tmem_st_wait();
                tc::fence_before_sync();
                atc::arrive(ds_full + sb);
            }
            if (!ok) break;
            // ------------------------------------------------------ epilogue
            bool have = false;
            if (nt > 0) {
                have = atc::agree(pair, 64, atc::wait(dq_full, on & 1, abort_flag));
                if (!have) { ok = false; break; }
                tc::fence_after_sync();
            }
#pragma unroll
            for (int c = 0; c < OC; c += 16) {
                uint32_t o16[16];
                if (have) {
                    tc::tmem_ld16(tmem + lrow + DQ_TM_Q + half * OC + c, o16);
                    tc::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) o16[e] = 0u;
                }
                if (row_ok) {
                    float4 *dst = reinterpret_cast<float4 *>(cp.dq + orow * D + half * OC + c);
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        float4 v = make_float4(__uint_as_float(o16[e]) * cp.scale, __uint_as_float(o16[e + 1]) * cp.scale,
                                               __uint_as_float(o16[e + 2]) * cp.scale,
                                               __uint_as_float(o16[e + 3]) * cp.scale);
                        if (cp.dq_accum) {
                            const float4 o = dst[e / 4];
                            v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
                        }
                        dst[e / 4] = v;
                    }
                }
            }
            if (have) {
                tc::fence_before_sync();
                atc::arrive(dq_free);
                ++on;
            }
        }
        if (!ok) fail();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, DQ_TM_COLS);
}


// ------------------------------------------------------------------------
// dk / dv of the NSA compressed and window branches on the tcgen05 tensor
// cores, key-major: an item is 128 keys of one KV group (the TMEM lanes) and
// a run of up to KV_QSPLIT tiles of the queries that see them, each tile 4
// consecutive queries x 16 heads = 64 columns.  The keys' K_hi (+ K_lo) and
// V stay in shared memory for the item; per query tile one thread issues
//   S^T = K Q_t^T (+ K_lo Q_t^T)   and   dP^T = V dO_t^T      (N = 64)
// into tensor memory; the score warps (one key row per thread) form
//   P^T = gate * exp2(S^T * scale_log2 - lse2),  dS^T = P^T (dP^T - D)
// masked to the (key, query) pairs the branch relates, and store both as
// bf16 pairs in tensor memory over the S^T / dP^T columns they have just
// read (two buffers, so the next tile's S^T / dP^T overlaps this tile's
// scores); the MMA thread then adds
//   dV += P^T dO_t   and   dK += dS^T Q_t        (A from TMEM, B MN-major)
// into two 128-column accumulators that live for the whole item.  At the end
// of an item the score warps add dK * scale and dV to the global fp32 rows
// (one reduction per key and column per item).  The per-row lse / D / gate
// of a query tile come as one 1 KB bulk copy of a packed array
// (nsa_kv_scalars_kernel); three such stages are in flight.
constexpr int KV_QT = 4;                 // queries per tile (x 16 heads = 64 columns)
constexpr int KV_QSPLIT = 64;            // query tiles per item
constexpr int KV_QSTAGES = 3;            // Q / dO / scalar stages
constexpr int KV_THREADS = 320;
// buffer b (b = 0, 1) at b * 128: S^T in columns 0-63, dP^T in 64-127; P^T
// and dS^T overwrite them as bf16 pairs (score-warp half h writes the pairs of
// its 32 columns into the first 16 of them)
constexpr uint32_t KV_TM_S = 0;
constexpr uint32_t KV_TM_DP = 64;
constexpr uint32_t KV_TM_V = 256;        // dV: 128 fp32 columns
constexpr uint32_t KV_TM_K = 384;        // dK: 128
constexpr uint32_t KV_TM_COLS = 512;

struct KvSmem {                          // head dim 128
    static constexpr int KT_BYTES = 128 * 256;           // one K (or V) tile: 2 halves x 128 rows x 128 B
    static constexpr int QT_BYTES = 64 * 256;            // one Q (or dO) tile: 2 halves x 64 rows x 128 B
    static constexpr int SC_BYTES = KV_QT * 16 * 16;     // lse, D, gate, pad of the tile's 64 rows
    static constexpr int QSTAGE = 2 * QT_BYTES + 1024;   // Q | dO | scalars (1 KB slot)
    static constexpr int OFF_K = 0;                      // K_hi | K_lo | V
    static constexpr int OFF_Q = OFF_K + 3 * KT_BYTES;
    static constexpr int OFF_BAR = OFF_Q + KV_QSTAGES * QSTAGE;
    // kv_full, kv_empty, q_full[S], q_empty[S], s_full[2], pd_full[2], pd_done[2], acc_full, acc_free, drain
    static constexpr int N_BAR = 2 + 2 * KV_QSTAGES + 6 + 3;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;
    static constexpr int TOTAL = OFF_MISC + 16;
    static constexpr int ALLOC = TOTAL + 1024;
};

// Key source of the key-major pass beside the two range branches: the
// selected blocks, each a 64-key block (half of the 128 TMEM lanes, the rest
// masked) walked over the queries of its inverse list.
constexpr int KV_LISTS = 2;

struct KvTcParams {
    TileParams t;            // k (K_hi), klo, v, shapes (T queries, Lk keys), window / cmp_len / cmp_stride, scale_log2
    const float4 *scal;      // [B, Hkv, T, 16] (lse natural, D, gate, 0) of this branch
    float *dk, *dv;          // [B, Lk, Hkv, 128] fp32, added to
    float scale;
    unsigned *err;
    int n_kt;                // key tiles per sequence
    int n_split;             // query splits per key tile
    int n_items;             // B * Hkv * n_kt * n_split (range branches)
    // KV_LISTS: the inverse block lists (see bwd_sel_* kernels)
    const int32_t *qlist, *qoff;
    const int2 *items;
    const int32_t *n_items_dev;
    int nb, sel_block, list_split;
};

// Queries [q_lo, q_hi) that see at least one key of [j0, j1] (range branches).
template <int SRC>
__device__ __forceinline__ void kv_tc_range(const TileParams &p, int j0, int j1, int &q_lo, int &q_hi) {
    if constexpr (SRC == TS_CMP) {
        q_lo = j0 * p.cmp_stride + p.cmp_len - 1;
        q_hi = p.T;
    } else {
        q_lo = j0;
        q_hi = min(p.T, j1 + p.window);
    }
}

// Item -> (b, g, keys [j0, jend), first query tile or list entry, list end);
// returns the number of query tiles (0 = empty item).
template <int SRC>
__device__ __forceinline__ int kv_tc_item(const KvTcParams &cp, int it, int &b, int &g, int &j0, int &jend, int &qt0,
                                          int &qlim) {
    const TileParams &p = cp.t;
    if constexpr (SRC == KV_LISTS) {
        const int2 wi = cp.items[it];
        const int blk = wi.x % cp.nb;
        g = (wi.x / cp.nb) % p.Hkv;
        b = wi.x / cp.nb / p.Hkv;
        j0 = blk * cp.sel_block;
        jend = min(j0 + cp.sel_block, p.Lk);
        if (j0 >= jend) return 0;
        const int o1 = cp.qoff[wi.x + 1];
        qt0 = cp.qoff[wi.x] + wi.y * cp.list_split;           // first list entry
        qlim = min(o1, qt0 + cp.list_split);
        return qlim > qt0 ? (qlim - qt0 + KV_QT - 1) / KV_QT : 0;
    } else {
        const int s = it % cp.n_split;
        int rem = it / cp.n_split;
        const int kt = rem % cp.n_kt; rem /= cp.n_kt;
        g = rem % p.Hkv;
        b = rem / p.Hkv;
        j0 = kt * 128;
        jend = min(j0 + 128, p.Lk);
        qlim = p.T;
        int q_lo, q_hi;
        kv_tc_range<SRC>(p, j0, jend - 1, q_lo, q_hi);
        if (q_lo >= q_hi) return 0;
        const int a0 = q_lo / KV_QT;                               // first query tile (aligned)
        const int n_all = (q_hi + KV_QT - 1) / KV_QT - a0;
        qt0 = a0 + s * KV_QSPLIT;
        const int n = n_all - s * KV_QSPLIT;
        return n <= 0 ? 0 : min(n, KV_QSPLIT);
    }
}

template <int SRC>
__global__ void __launch_bounds__(KV_THREADS, 1)
    nsa_kv_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap domap,
                     const __grid_constant__ CUtensorMap khimap, const __grid_constant__ CUtensorMap klomap,
                     const __grid_constant__ CUtensorMap vmap, const KvTcParams cp) {
    grid_dependency_sync();
    constexpr int D = 128;
    constexpr bool LO = SRC == TS_CMP;
    constexpr bool LS = SRC == KV_LISTS;
    using L = KvSmem;
    const TileParams &p = cp.t;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *kv_full = bars, *kv_empty = bars + 1, *q_full = bars + 2, *q_empty = q_full + KV_QSTAGES;
    uint64_t *s_full = q_empty + KV_QSTAGES, *pd_full = s_full + 2, *pd_done = pd_full + 2;
    uint64_t *acc_full = pd_done + 2, *acc_free = acc_full + 1, *drain = acc_free + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, KV_TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(kv_full, 1); tc::mbar_init(kv_empty, 1);
        for (int i = 0; i < KV_QSTAGES; ++i) { tc::mbar_init(q_full + i, 1); tc::mbar_init(q_empty + i, 1); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(pd_full + i, 256); tc::mbar_init(pd_done + i, 1);
            tc::mbar_init(s_full + i, 1);
        }
        tc::mbar_init(acc_full, 1); tc::mbar_init(acc_free, 256);
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
    const int n_items_all = LS ? *cp.n_items_dev : cp.n_items;
    // query of list entry e of an item (entries past its end read its last one, masked later)
    auto list_t = [&](int e, int qlim) -> int { return __ldg(cp.qlist + min(e, qlim - 1)); };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int qt = 0, kn = 0;                           // query tiles and key tiles loaded
            const int n_items = debug_stall() ? 0 : n_items_all;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                int b, g, j0, jend, qt0, qlim;
                const int nq = kv_tc_item<SRC>(cp, it, b, g, j0, jend, qt0, qlim);
                if (nq == 0) continue;
                // the keys of the item, once the previous item's last MMA is done
                if (!atc::wait(kv_empty, (kn & 1) ^ 1, abort_flag)) { ok = false; break; }
                atc::expect_tx(kv_full, LO ? 3 * L::KT_BYTES : 2 * L::KT_BYTES);
                const int z = b * p.Lk + j0;
                for (int h = 0; h < 2; ++h) {
                    atc::load_3d(smem + L::OFF_K + h * (128 * 128), &khimap, h * 64, g, z, kv_full);
                    if (LO) atc::load_3d(smem + L::OFF_K + L::KT_BYTES + h * (128 * 128), &klomap, h * 64, g, z, kv_full);
                    atc::load_3d(smem + L::OFF_K + 2 * L::KT_BYTES + h * (128 * 128), &vmap, h * 64, g, z, kv_full);
                }
                ++kn;
                for (int i = 0; i < nq; ++i, ++qt) {
                    const int qs = qt % KV_QSTAGES;
                    if (!atc::wait(q_empty + qs, ((qt / KV_QSTAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    unsigned char *dst = smem + L::OFF_Q + qs * L::QSTAGE;
                    const int t0 = (qt0 + i) * KV_QT;
                    atc::expect_tx(q_full + qs, 2 * L::QT_BYTES + L::SC_BYTES);
                    for (int w = 0; w < KV_QT; ++w) {
                        const int tw = LS ? list_t(qt0 + i * KV_QT + w, qlim) : min(t0 + w, p.T - 1);
                        const int qrow = (b * p.T + tw) * p.Hq + g * p.G;
                        for (int h = 0; h < 2; ++h) {
                            atc::load_2d(dst + h * (64 * 128) + w * (16 * 128), &qmap, h * 64, qrow, q_full + qs);
                            atc::load_2d(dst + L::QT_BYTES + h * (64 * 128) + w * (16 * 128), &domap, h * 64, qrow,
                                         q_full + qs);
                        }
                    }
                    // lse / D / gate of the tile's rows: 4 consecutive queries of (b, g), one 1 KB copy
                    // (rows past the sequence read the last query's, masked later); list queries one
                    // 256 B copy each
                    if constexpr (LS) {
                        for (int w = 0; w < KV_QT; ++w) {
                            const int tw = list_t(qt0 + i * KV_QT + w, qlim);
                            const float4 *src = cp.scal + ((long long)(b * p.Hkv + g) * p.T + tw) * 16;
                            asm volatile(
                                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                                    tc::smem_u32(dst + 2 * L::QT_BYTES + w * 256)),
                                "l"(src), "r"(256), "r"(tc::smem_u32(q_full + qs))
                                : "memory");
                        }
                    } else {
                        const int tc0 = min(t0, p.T - KV_QT);
                        const float4 *src = cp.scal + ((long long)(b * p.Hkv + g) * p.T + tc0) * 16;
                        asm volatile(
                            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                                tc::smem_u32(dst + 2 * L::QT_BYTES)),
                            "l"(src), "r"(L::SC_BYTES), "r"(tc::smem_u32(q_full + qs))
                            : "memory");
                    }
                }
            }
            if (!ok) fail();
            // let the copies land before the CTA exits
            if (kn > 0) tc::mbar_wait_bounded(kv_full, (kn - 1) & 1, ATC_WAIT);
            for (int i = 0; i < KV_QSTAGES && i < qt; ++i) {
                const int q = qt - 1 - i;
                tc::mbar_wait_bounded(q_full + q % KV_QSTAGES, (q / KV_QSTAGES) & 1, ATC_WAIT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::make_idesc(1, 1, 128, 64);
            constexpr uint32_t ID_A = tc::make_idesc(1, 1, 128, D) | (1u << 16);   // B (dO, Q) MN-major
            const uint32_t ka = tc::smem_u32(smem + L::OFF_K);
            bool ok = true;
            int qt = 0, kn = 0, an = 0;
            // S^T and dP^T of query tile q (stage q & 1) into buffer q & 1, once
            // the dV / dK products of tile q - 2 (which read that buffer) are done
            auto issue_s = [&](int q) -> bool {
                const int qs = q % KV_QSTAGES, b = q & 1;
                if (!atc::wait(q_full + qs, (q / KV_QSTAGES) & 1, abort_flag)) return false;
                if (q >= 2 && !atc::wait(pd_done + b, ((q >> 1) & 1) ^ 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t qa = tc::smem_u32(smem + L::OFF_Q + qs * L::QSTAGE);
                const uint32_t da = qa + L::QT_BYTES;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int h = ks / 4, kk = ks % 4;
                    const uint64_t akh = atc::desc_sw128(ka + h * (128 * 128) + kk * 32, 16, 1024);
                    const uint64_t akl = atc::desc_sw128(ka + L::KT_BYTES + h * (128 * 128) + kk * 32, 16, 1024);
                    const uint64_t av = atc::desc_sw128(ka + 2 * L::KT_BYTES + h * (128 * 128) + kk * 32, 16, 1024);
                    const uint64_t bq = atc::desc_sw128(qa + h * (64 * 128) + kk * 32, 16, 1024);
                    const uint64_t bd = atc::desc_sw128(da + h * (64 * 128) + kk * 32, 16, 1024);
                    tc::mma_bf16(tmem + b * 128 + KV_TM_S, akh, bq, ID_S, ks > 0 ? 1u : 0u);
                    if (LO) tc::mma_bf16(tmem + b * 128 + KV_TM_S, akl, bq, ID_S, 1u);
                    tc::mma_bf16(tmem + b * 128 + KV_TM_DP, av, bd, ID_S, ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(s_full + b);
                return true;
            };
            for (int it = blockIdx.x; it < n_items_all && ok; it += gridDim.x) {
                int b, g, j0, jend, qt0, qlim;
                const int nq = kv_tc_item<SRC>(cp, it, b, g, j0, jend, qt0, qlim);
                if (nq == 0) continue;
                if (!atc::wait(kv_full, kn & 1, abort_flag)) { ok = false; break; }
                ++kn;
                if (!issue_s(qt)) { ok = false; break; }
                // the previous item's epilogue must have read dV / dK
                if (an > 0 && !atc::wait(acc_free, (an - 1) & 1, abort_flag)) { ok = false; break; }
                for (int i = 0; i < nq; ++i, ++qt) {
                    const int qs = qt % KV_QSTAGES, pb = qt & 1;
                    if (i + 1 < nq && !issue_s(qt + 1)) { ok = false; break; }
                    if (!atc::wait(pd_full + pb, (qt >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t qa = tc::smem_u32(smem + L::OFF_Q + qs * L::QSTAGE);
                    const uint32_t da = qa + L::QT_BYTES;
                    // dV += P^T dO_t, dK += dS^T Q_t: A from tensor memory, B MN-major
#pragma unroll
                    for (int kk = 0; kk < 64 / 16; ++kk) {
                        const uint32_t pc = pb * 128 + (kk < 2 ? kk * 8 : 32 + (kk - 2) * 8);
                        const uint64_t bdo = atc::desc_sw128(da + kk * 2048, 64 * 128, 1024);
                        const uint64_t bqq = atc::desc_sw128(qa + kk * 2048, 64 * 128, 1024);
                        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                        tc::mma_bf16_ts(tmem + KV_TM_V, tmem + pc + KV_TM_S, bdo, ID_A, acc);
                        tc::mma_bf16_ts(tmem + KV_TM_K, tmem + pc + KV_TM_DP, bqq, ID_A, acc);
                    }
                    tc::mma_commit(q_empty + qs);
                    tc::mma_commit(pd_done + pb);
                }
                if (!ok) break;
                tc::mma_commit(kv_empty);
                tc::mma_commit(acc_full);
                ++an;
            }
            if (!ok) fail();
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, ATC_WAIT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ score warps
        // Thread = one key (TMEM lane); the two warps of a lane quadrant take
        // the query-tile columns 0-31 / 32-63 and the dV / dK columns 0-63 /
        // 64-127.  The pair agrees on each wait through a 64-thread named barrier.
        const int quad = warp & 3, half = (warp - 2) >> 2;
        const int pair = 1 + quad;
        constexpr int SC = 32, OC = D / 2;
        const int kr = quad * 32 + lane;                  // key row of the tile
        const uint32_t lrow = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        int qt = 0, an = 0;
        for (int it = blockIdx.x; it < n_items_all && ok; it += gridDim.x) {
            int b, g, j0, jend, qt0, qlim;
            const int nq = kv_tc_item<SRC>(cp, it, b, g, j0, jend, qt0, qlim);
            if (nq == 0) continue;
            const int j = j0 + kr;                        // this thread's key
            for (int i = 0; i < nq; ++i, ++qt) {
                const int qs = qt % KV_QSTAGES, pb = qt & 1;
                // S^T / dP^T of the tile (its MMA waited for the Q / dO stage, and
                // with it the scalars' copy; the wait below makes them visible)
                bool got = atc::wait(s_full + pb, (qt >> 1) & 1, abort_flag);
                if (got) got = atc::wait(q_full + qs, (qt / KV_QSTAGES) & 1, abort_flag);
                if (!atc::agree(pair, 64, got)) { ok = false; break; }
                tc::fence_after_sync();
                uint32_t sr[SC], dr[SC];
#pragma unroll
                for (int c = 0; c < SC; c += 16) {
                    tc::tmem_ld16(tmem + lrow + pb * 128 + KV_TM_S + half * SC + c,
                                  *reinterpret_cast<uint32_t(*)[16]>(sr + c));
                    tc::tmem_ld16(tmem + lrow + pb * 128 + KV_TM_DP + half * SC + c,
                                  *reinterpret_cast<uint32_t(*)[16]>(dr + c));
                }
                tc::tmem_ld_wait();
                const float4 *sc = reinterpret_cast<const float4 *>(smem + L::OFF_Q + qs * L::QSTAGE + 2 * L::QT_BYTES);
                const int t0 = (qt0 + i) * KV_QT;
                const int tc0 = min(t0, p.T - KV_QT);
                // list queries of this warp's two columns groups (w = 2 half, 2 half + 1)
                int tl[2] = {0, 0};
                bool vl[2] = {false, false};
                if constexpr (LS) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int e = qt0 + i * KV_QT + 2 * half + u;
                        vl[u] = e < qlim;
                        tl[u] = list_t(e, qlim);
                    }
                }
                uint32_t pp[SC / 2], dp2[SC / 2];
#pragma unroll
                for (int c = 0; c < SC; c += 2) {
                    float pv[2], dv2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int col = half * SC + c + e;         // q-row of the tile: query col/16, head col%16
                        bool vis;
                        float4 s4;
                        if constexpr (LS) {
                            // the list query of column group col / 16 chose this key's block
                            const int u = (col >> 4) & 1;
                            const int t = tl[u];
                            s4 = sc[col];
                            vis = vl[u] && j < jend && j <= t;
                        } else {
                            const int t = t0 + (col >> 4);
                            // rows past the sequence read the last query's slot (masked below)
                            s4 = sc[(min(t, p.T - 1) - tc0) * 16 + (col & 15)];
                            if constexpr (SRC == TS_CMP) vis = j < p.Lk && j * p.cmp_stride + p.cmp_len - 1 <= t;
                            else vis = j <= t && j > t - p.window;
                            vis = vis && t < p.T;
                        }
                        vis = vis && s4.x != -INFINITY;
                        const float pr = vis ? s4.z * ex2_fast(fmaf(__uint_as_float(sr[c + e]), p.scale_log2,
                                                                  -s4.x * kLog2e)) : 0.f;
                        pv[e] = pr;
                        dv2[e] = pr * (__uint_as_float(dr[c + e]) - s4.y);
                    }
                    pp[c / 2] = pack_bf16(pv[0], pv[1]);
                    dp2[c / 2] = pack_bf16(dv2[0], dv2[1]);
                }
                // the pairs over the first 16 of the 32 columns this warp has read
                atc::tmem_st16(tmem + lrow + pb * 128 + KV_TM_S + half * SC, *reinterpret_cast<const uint32_t(*)[16]>(pp));
                atc::tmem_st16(tmem + lrow + pb * 128 + KV_TM_DP + half * SC, *reinterpret_cast<const uint32_t(*)[16]>(dp2));
                atc::tmem_st_wait();
                tc::fence_before_sync();
                atc::arrive(pd_full + pb);
            }
            if (!ok) break;
            // ------------------------------------------------------ epilogue
            if (!atc::agree(pair, 64, atc::wait(acc_full, an & 1, abort_flag))) { ok = false; break; }
            tc::fence_after_sync();
            const bool kv_ok = j < jend;
            float *dvr = cp.dv + (((long long)b * p.Lk + (kv_ok ? j : 0)) * p.Hkv + g) * D + half * OC;
            float *dkr = cp.dk + (((long long)b * p.Lk + (kv_ok ? j : 0)) * p.Hkv + g) * D + half * OC;
#pragma unroll
            for (int c = 0; c < OC; c += 16) {
                uint32_t v16[16], k16[16];
                tc::tmem_ld16(tmem + lrow + KV_TM_V + half * OC + c, v16);
                tc::tmem_ld16(tmem + lrow + KV_TM_K + half * OC + c, k16);
                tc::tmem_ld_wait();
                if (kv_ok) {
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        red_add2(dvr + c + e, __uint_as_float(v16[e]), __uint_as_float(v16[e + 1]));
                        red_add2(dkr + c + e, __uint_as_float(k16[e]) * cp.scale, __uint_as_float(k16[e + 1]) * cp.scale);
                    }
                }
            }
            tc::fence_before_sync();
            atc::arrive(acc_free);
            ++an;
        }
        if (!ok) fail();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, KV_TM_COLS);
}

// Packed per-(b, g, query, head) scalars of one branch for nsa_kv_tc_kernel:
// (lse natural, D, gate, 0); heads past the group get lse = -inf, gate 0.
__global__ void __launch_bounds__(256) nsa_kv_scalars_kernel(const float *__restrict__ lse, int lse_stride,
                                                             const float *__restrict__ Dt,
                                                             const float *__restrict__ gate, int gate_stride,
                                                             int B, int T, int Hq, int Hkv, int G,
                                                             float4 *__restrict__ out) {
    grid_dependency_sync();
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)B * Hkv * T * 16;
    if (e >= total) return;
    const int h = (int)(e % 16);
    long long r = e / 16;
    const int t = (int)(r % T); r /= T;
    const int g = (int)(r % Hkv);
    const int b = (int)(r / Hkv);
    float4 v = make_float4(-INFINITY, 0.f, 0.f, 0.f);
    if (h < G) {
        const long long row = ((long long)b * T + t) * Hq + (long long)g * G + h;
        v = make_float4(lse[row * lse_stride], Dt[row], gate ? gate[row * gate_stride] : 1.f, 0.f);
    }
    out[e] = v;
}

}  // namespace sa
