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

#include "attn_cmp_tc.cuh"

namespace sa {

constexpr int DQ_KT = 64;               // keys per tile
constexpr int DQ_STAGES = 2;
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
                        const float pv = vis ? exp2f(fmaf(__uint_as_float(sr[k + e]), p.scale_log2, nb)) : 0.f;
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

}  // namespace sa
