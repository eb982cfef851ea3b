// attn_cmp_tc.cuh -- NSA compressed and sliding-window branches on the tcgen05
// tensor cores.
//
// NSA page ("Native Sparse Attention ...", "Puntos Clave": coarse-grained
// token compression): every query attends to the compressed keys/values of
// its KV group whose source blocks it can see (compressed token i is visible
// to query t iff i*stride + len - 1 <= t).  All queries of a block read the
// same compressed keys, so the product is dense:
//   S[128 x 128]  = Q[128 rows x d] . Kc^T   (rows = 8 queries x 16 heads)
//   O[128 x d]   += P[128 x 128] . Vc
// with fp32 accumulators in TMEM (tcgen05.mma kind::f16), 128 keys per tile.  The compressed
// keys are means and do not fit bf16 exactly, so they are held as a bf16
// hi/lo pair and S accumulates both halves (Q.K_hi + Q.K_lo).  The same
// kernel (SRC = TS_WINDOW) runs the sliding-window branch (NSA page, "Puntos
// Clave": local context) over the raw keys t - window < j <= t, whose union
// over 8 consecutive queries is again one contiguous key range.
//
// Q, K_hi, K_lo and V tiles arrive by TMA box loads in the 128B-swizzled
// canonical layouts (K-major for Q and K; MN-major for V as the B operand of
// the second product); P goes from the softmax warps to tensor memory and is
// read there as the A operand of P.V.  Softmax: row r (one query head) is
// split between two warps of the same TMEM lane quadrant, 64 scores each;
// they swap partial row maxima and the final row sums through shared memory.
// The running max is raised (and the O row rescaled in TMEM) only when a
// tile's max exceeds it by more than 2^8.  Larger tiles halve the hand-offs
// between the MMA thread and the softmax warps per key, which is what bounds
// this kernel.
//
// Warps: 0 TMA producer (one thread), 1 MMA issuer (one thread) and TMEM
// owner, 2-9 softmax + epilogue (TMEM lane quadrants 2, 3, 0, 1, twice).
// Every wait is bounded; a timeout sets ERR_TIMEOUT and the CTA drains and
// exits.
#pragma once

#include <cuda.h>

#include "attn_tc.cuh"
#include "attn_tile.cuh"

namespace sa {

constexpr int CT_Q = 8;            // queries per item (x 16 heads = 128 rows)

// nsa_tc_kernel: 128-key tiles (S = Q.K^T at N = 128), two stages, P in
// tensor memory as the A operand of P.V, 8 softmax warps.
constexpr int NT_KT = 128;
constexpr int NT_STAGES = 2;
constexpr int NT_THREADS = 320;      // TMA warp, MMA warp, 8 softmax warps (two per TMEM lane quadrant)
constexpr uint32_t NT_TM_S = 0;      // S: 2 buffers x NT_KT fp32 columns
constexpr uint32_t NT_TM_P = 256;    // P: 2 buffers x NT_KT / 2 columns (bf16 pairs)
constexpr uint32_t NT_TM_O = 384;    // O: 128 fp32 columns
constexpr uint32_t NT_TM_COLS = 512;

struct CtSmem {                    // head dim 128
    static constexpr int Q_BYTES = 128 * 256;              // 2 halves x 128 rows x 128 B
    static constexpr int KT_BYTES = NT_KT * 256;           // one K (or V) tile: 2 halves x 128 rows x 128 B
    static constexpr int STAGE = 3 * KT_BYTES;             // K_hi | K_lo | V
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + NT_STAGES * STAGE;
    // q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], s_free[2], p_full[2],
    // pv_done[2], o_full, o_free, drain
    static constexpr int N_BAR = 2 + 2 * NT_STAGES + 8 + 3;
    // [half][row]: partial row maxima of the current tile, then the row sums
    static constexpr int OFF_XCH = OFF_BAR + N_BAR * 8;
    static constexpr int OFF_MISC = OFF_XCH + 2 * 128 * 4;
    static constexpr int TOTAL = OFF_MISC + 16;
    static constexpr int ALLOC = TOTAL + 1024;
};



struct CmpTcParams {
    TileParams t;          // q, shapes, cmp_len/stride (Lk = compressed tokens per sequence), outputs
    unsigned *err;
    int n_items;           // B * Hkv * ceil(T / CT_Q)
};

// Item -> (b, g, query block); items with the latest (heaviest) query blocks
// come first so the persistent CTAs finish together.
__device__ __forceinline__ void ct_item(const TileParams &p, int it, int &b, int &g, int &t0) {
    const int nqb = (p.T + CT_Q - 1) / CT_Q;
    const int bg = it % (p.B * p.Hkv);
    const int qb = nqb - 1 - it / (p.B * p.Hkv);
    b = bg / p.Hkv;
    g = bg % p.Hkv;
    t0 = qb * CT_Q;
}

template <int SRC>
__global__ void __launch_bounds__(NT_THREADS, 1)
    nsa_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap khimap,
                  const __grid_constant__ CUtensorMap klomap, const __grid_constant__ CUtensorMap vmap,
                  const CmpTcParams cp) {
    grid_dependency_sync();
    constexpr int D = 128;
    constexpr bool LO = SRC == TS_CMP;             // compressed keys carry a lo half
    using L = CtSmem;
    const TileParams &p = cp.t;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *q_full = bars, *q_empty = bars + 1, *kv_full = bars + 2, *kv_empty = kv_full + NT_STAGES;
    uint64_t *s_full = kv_empty + NT_STAGES, *s_free = s_full + 2, *p_full = s_free + 2, *pv_done = p_full + 2;
    uint64_t *o_full = pv_done + 2, *o_free = o_full + 1, *drain = o_free + 1;
    float *xch = reinterpret_cast<float *>(smem + L::OFF_XCH);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, NT_TM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(q_full, 1); tc::mbar_init(q_empty, 1);
        for (int i = 0; i < NT_STAGES; ++i) { tc::mbar_init(kv_full + i, 1); tc::mbar_init(kv_empty + i, 1); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(s_full + i, 1); tc::mbar_init(s_free + i, 256);
            tc::mbar_init(p_full + i, 256); tc::mbar_init(pv_done + i, 1);
        }
        tc::mbar_init(o_full, 1); tc::mbar_init(o_free, 256);
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
    // first key of an item's range (window: the first query's window start)
    auto key_lo = [&](int t0) -> int { return SRC == TS_CMP ? 0 : max(0, t0 - p.window + 1); };
    auto tiles_of = [&](int t0) -> int {
        const int t_last = min(t0 + CT_Q - 1, p.T - 1);
        return ((int)tile_key_end<SRC>(p, t_last) - key_lo(t0) + NT_KT - 1) / NT_KT;
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int tile = 0, qn = 0;
            // test hook: issue nothing, so the MMA thread's first wait runs out
            const int n_items = debug_stall() ? 0 : cp.n_items;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                int b, g, t0;
                ct_item(p, it, b, g, t0);
                const int nt = tiles_of(t0);
                if (nt == 0) continue;                     // the epilogue writes zeros without Q or keys
                if (!atc::wait(q_empty, (qn & 1) ^ 1, abort_flag)) { ok = false; break; }
                atc::expect_tx(q_full, L::Q_BYTES);
                for (int w = 0; w < CT_Q; ++w) {
                    const int qrow = (b * p.T + min(t0 + w, p.T - 1)) * p.Hq + g * p.G;
                    for (int h = 0; h < 2; ++h)
                        atc::load_2d(smem + L::OFF_Q + h * (128 * 128) + w * (16 * 128), &qmap, h * 64, qrow, q_full);
                }
                ++qn;
                for (int kt = 0; kt < nt; ++kt, ++tile) {
                    const int st = tile % NT_STAGES;
                    if (!atc::wait(kv_empty + st, ((tile / NT_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    atc::expect_tx(kv_full + st, LO ? L::STAGE : 2 * L::KT_BYTES);
                    unsigned char *dst = smem + L::OFF_KV + st * L::STAGE;
                    const int z = b * p.Lk + key_lo(t0) + kt * NT_KT;
                    for (int h = 0; h < 2; ++h) {
                        atc::load_3d(dst + h * (NT_KT * 128), &khimap, h * 64, g, z, kv_full + st);
                        if (LO) atc::load_3d(dst + L::KT_BYTES + h * (NT_KT * 128), &klomap, h * 64, g, z, kv_full + st);
                        atc::load_3d(dst + 2 * L::KT_BYTES + h * (NT_KT * 128), &vmap, h * 64, g, z, kv_full + st);
                    }
                }
            }
            if (!ok) fail();
            // let the copies land before the CTA exits
            if (qn > 0) tc::mbar_wait_bounded(q_full, (qn - 1) & 1, ATC_WAIT);
            for (int i = 0; i < NT_STAGES && i < tile; ++i) {
                const int kt = tile - 1 - i;
                tc::mbar_wait_bounded(kv_full + kt % NT_STAGES, (kt / NT_STAGES) & 1, ATC_WAIT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::make_idesc(1, 1, 128, NT_KT);
            constexpr uint32_t ID_O = tc::make_idesc(1, 1, 128, D) | (1u << 16);   // B (V) MN-major
            const uint32_t qa = tc::smem_u32(smem + L::OFF_Q);
            bool ok = true;
            int tile = 0, qn = 0, on = 0;   // tiles, Q loads, items with an O result
            auto issue_s = [&](int tl) -> bool {
                const int st = tl % NT_STAGES, sb = tl & 1;
                if (!atc::wait(kv_full + st, (tl / NT_STAGES) & 1, abort_flag)) return false;
                if (!atc::wait(s_free + sb, ((tl >> 1) & 1) ^ 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t ka = tc::smem_u32(smem + L::OFF_KV + st * L::STAGE);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int h = ks / 4, kk = ks % 4;
                    const uint64_t ad = atc::desc_sw128(qa + h * (128 * 128) + kk * 32, 16, 1024);
                    const uint64_t bh = atc::desc_sw128(ka + h * (NT_KT * 128) + kk * 32, 16, 1024);
                    const uint64_t bl = atc::desc_sw128(ka + L::KT_BYTES + h * (NT_KT * 128) + kk * 32, 16, 1024);
                    tc::mma_bf16(tmem + NT_TM_S + sb * NT_KT, ad, bh, ID_S, ks > 0 ? 1u : 0u);
                    if (LO) tc::mma_bf16(tmem + NT_TM_S + sb * NT_KT, ad, bl, ID_S, 1u);
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
                // the previous item's epilogue must have read O before it is overwritten
                if (on > 0 && !atc::wait(o_free, (on - 1) & 1, abort_flag)) { ok = false; break; }
                for (int kt = 0; kt < nt; ++kt, ++tile) {
                    const int st = tile % NT_STAGES, pb = tile & 1;
                    if (kt + 1 < nt && !issue_s(tile + 1)) { ok = false; break; }
                    if (kt + 1 == nt) tc::mma_commit(q_empty);   // Q is free once the last S is done
                    if (!atc::wait(p_full + pb, (tile >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    // O += P.V: P (A) from tensor memory, V (B) from shared memory
                    const uint32_t va = tc::smem_u32(smem + L::OFF_KV + st * L::STAGE + 2 * L::KT_BYTES);
#pragma unroll
                    for (int kk = 0; kk < NT_KT / 16; ++kk) {
                        // V: MN-major, 64-column atoms NT_KT * 128 B apart, 8-key groups 1 KB apart
                        const uint64_t bd = atc::desc_sw128(va + kk * 2048, NT_KT * 128, 1024);
                        tc::mma_bf16_ts(tmem + NT_TM_O, tmem + NT_TM_P + pb * (NT_KT / 2) + kk * 8, bd, ID_O,
                                        (kt > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(kv_empty + st);
                    tc::mma_commit(pv_done + pb);
                    if (kt + 1 == nt) tc::mma_commit(o_full);
                }
                ++on;
            }
            if (!ok) fail();
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, ATC_WAIT);
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- softmax rows
        // Two warps per TMEM lane quadrant share its 32 rows: half 0 takes S
        // and P columns 0-63 and O columns 0-63 of the quadrant's rows, half 1
        // the rest.  The pair agrees on each wait through a 64-thread named
        // barrier (ids 1-4) and swaps partial row maxima (per tile) and row
        // sums (per item) through shared memory; the agreement at the start
        // of each tile keeps one exchange slot per row safe to reuse.
        const int quad = warp & 3, half = (warp - 2) >> 2;
        const int pair = 1 + quad;
        constexpr int SC = NT_KT / 2, OC = D / 2;          // S and O columns per warp
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
            // visible keys of this row as item-relative indices [vlo, vhi)
            const int klo = key_lo(t0);
            const int vhi = t <= t_last ? (int)tile_key_end<SRC>(p, t) - klo : 0;
            const int vlo = (t <= t_last && SRC == TS_WINDOW) ? max(0, t - p.window + 1) - klo : 0;
            float m = -INFINITY, l = 0.f;
            for (int kt = 0; kt < nt; ++kt, ++tile) {
                const int sb = tile & 1, pb = tile & 1;
                // S of this tile; the P.V of tile - 2 (the last reader of P buffer
                // pb) was issued before it, so that wait costs nothing
                bool got = atc::wait(s_full + sb, (tile >> 1) & 1, abort_flag);
                if (got && tile >= 2) got = atc::wait(pv_done + pb, ((tile >> 1) & 1) ^ 1, abort_flag);
                if (!atc::agree(pair, 64, got)) { ok = false; break; }
                tc::fence_after_sync();
                uint32_t sr[SC];
#pragma unroll
                for (int c = 0; c < SC; c += 16)
                    tc::tmem_ld16(tmem + lrow + NT_TM_S + sb * NT_KT + half * SC + c,
                                  *reinterpret_cast<uint32_t(*)[16]>(sr + c));
                tc::tmem_ld_wait();
                tc::fence_before_sync();
                atc::arrive(s_free + sb);
                const int i0 = kt * NT_KT + half * SC;
                // partial row max of the raw scores (masked past the row's visible keys)
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (i0 >= vlo && i0 + SC <= vhi) {
#pragma unroll
                    for (int k = 0; k < SC; ++k) mx[k & 3] = fmaxf(mx[k & 3], __uint_as_float(sr[k]));
                } else {
#pragma unroll
                    for (int k = 0; k < SC; ++k) {
                        if (i0 + k < vlo || i0 + k >= vhi) sr[k] = __float_as_uint(-INFINITY);
                        mx[k & 3] = fmaxf(mx[k & 3], __uint_as_float(sr[k]));
                    }
                }
                float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                xch[half * 128 + r] = mt;
                atc::named_sync(pair, 64);
                mt = fmaxf(mt, xch[(half ^ 1) * 128 + r]);
                // m is kept in raw-score units; raise it only when the tile
                // exceeds it by more than 2^8 after scaling (both warps of the
                // pair see the same m and mt, so they decide alike)
                const bool raise = mt != -INFINITY && (m == -INFINITY || (mt - m) * p.scale_log2 > 8.f);
                float alpha = 1.f;
                if (raise) {
                    alpha = m == -INFINITY ? 0.f : ex2_fast((m - mt) * p.scale_log2);
                    m = mt;
                    l *= alpha;
                }
                if (kt > 0 && __any_sync(0xffffffffu, raise)) {
                    // rescale this warp's O columns once the previous P.V is done
                    const int pt = tile - 1;
                    if (!atc::agree(pair, 64, atc::wait(pv_done + (pt & 1), (pt >> 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
#pragma unroll
                    for (int c = 0; c < OC; c += 16) {
                        uint32_t o16[16];
                        tc::tmem_ld16(tmem + lrow + NT_TM_O + half * OC + c, o16);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o16[e] = __float_as_uint(__uint_as_float(o16[e]) * alpha);
                        atc::tmem_st16(tmem + lrow + NT_TM_O + half * OC + c, o16);
                    }
                    atc::tmem_st_wait();
                }
                // p = 2^((s - m) * scale_log2): one FFMA and one ex2 per score
                const float nb = m == -INFINITY ? 0.f : -m * p.scale_log2;
                uint32_t pk[SC / 2];
                float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < SC; k += 2) {
                    const float p0 = ex2_fast(fmaf(__uint_as_float(sr[k]), p.scale_log2, nb));
                    const float p1 = ex2_fast(fmaf(__uint_as_float(sr[k + 1]), p.scale_log2, nb));
                    rs[(k >> 1) & 3] += p0 + p1;
                    pk[k / 2] = pack_bf16(p0, p1);
                }
                l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
                // this warp's keys of row r as packed bf16 pairs in P buffer pb
#pragma unroll
                for (int c = 0; c < SC / 2; c += 16)
                    atc::tmem_st16(tmem + lrow + NT_TM_P + pb * (NT_KT / 2) + half * (SC / 2) + c,
                                   *reinterpret_cast<const uint32_t(*)[16]>(pk + c));
                atc::tmem_st_wait();
                tc::fence_before_sync();
                atc::arrive(p_full + pb);
            }
            if (!ok) break;
            // ------------------------------------------------------ epilogue
            const long long orow = (long long)(b * p.T + t) * p.Hq + g * p.G + h;
            bool have_o = false;
            float lr = 0.f;                               // the row sum over both halves
            if (nt > 0) {
                have_o = atc::agree(pair, 64, atc::wait(o_full, on & 1, abort_flag));
                if (!have_o) { ok = false; break; }
                tc::fence_after_sync();
                xch[half * 128 + r] = l;
                atc::named_sync(pair, 64);
                lr = half == 0 ? l + xch[128 + r] : xch[r] + l;
            }
            const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll
            for (int c = 0; c < OC; c += 16) {
                uint32_t o16[16];
                if (have_o) {
                    tc::tmem_ld16(tmem + lrow + NT_TM_O + half * OC + c, o16);
                    tc::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) o16[e] = 0u;
                }
                if (row_ok) {
                    float4 *dst = reinterpret_cast<float4 *>(p.out_f32 + orow * D + half * OC + c);
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        dst[e / 4] = make_float4(__uint_as_float(o16[e]) * inv, __uint_as_float(o16[e + 1]) * inv,
                                                 __uint_as_float(o16[e + 2]) * inv, __uint_as_float(o16[e + 3]) * inv);
                }
            }
            if (have_o) {
                tc::fence_before_sync();
                atc::arrive(o_free);
                ++on;
            }
            if (row_ok && half == 0 && p.lse) p.lse[orow] = lr > 0.f ? (m * p.scale_log2 + log2f(lr)) * kLn2 : -INFINITY;
        }
        if (!ok) fail();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, NT_TM_COLS);
}

}  // namespace sa

namespace sa {

// ---------------------------------------------------------------------------
// NSA block importance and top-k selection on tcgen05 (NSA page, "Puntos
// Clave": the compressed-branch attention scores rank the selection blocks).
// Persistent CTAs walk the same 8-query items as nsa_tc_kernel over the
// compressed keys in 128-key tiles: S = Q.K_hi^T + Q.K_lo^T in TMEM; two
// warps per TMEM lane quadrant each take one 64-key half of row r (one query
// head), turn it into probabilities with the compressed branch's LSE and sum
// them per selection block (sel_block / cmp_stride consecutive compressed
// tokens, never straddling the halves); the 16 heads of a query are summed by
// a transposing butterfly over the 16 lanes that hold them, so lane h ends
// with block h of the half tile.  The importances of an item stay in shared
// memory; each of the 8 score warps then takes one query's top-k blocks by
// repeated arg-max (ties to the lower block), written in ascending order.  Blocks past the last tile have no visible compressed
// token and count as 0.
constexpr int IT_KT = 128;            // compressed keys per tile
constexpr int IT_STAGES = 2;
constexpr int IT_THREADS = 320;       // TMA warp, MMA warp, 8 score warps (two per TMEM lane quadrant)
constexpr int IT_MAX_BLOCKS = 2048;   // candidate blocks per query held in shared memory

struct ItSmem {                       // head dim 128
    static constexpr int Q_BYTES = 128 * 256;
    static constexpr int KT_BYTES = IT_KT * 256;
    static constexpr int STAGE = 2 * KT_BYTES;                 // K_hi | K_lo
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + Q_BYTES;
    static constexpr int OFF_IMP = OFF_KV + IT_STAGES * STAGE; // [CT_Q][n_blocks] float
    static constexpr int N_BAR = 2 + 2 * IT_STAGES + 4 + 1;    // q_full, q_empty, kv x2, s_full x2, s_free x2, drain
    __host__ __device__ static int off_bar(int n_blocks) { return OFF_IMP + CT_Q * n_blocks * 4; }
    __host__ __device__ static int alloc(int n_blocks) { return off_bar(n_blocks) + N_BAR * 8 + 16 + 1024; }
};

struct ImpTcParams {
    TileParams t;          // q, shapes (Lk = compressed tokens), cmp_len / cmp_stride, scale
    const float *lse_cmp;  // [B,T,Hq] natural log
    int sel_block, sel_topk, n_blocks;
    int32_t *sel_idx;      // [B,T,Hkv,sel_topk]
    unsigned *err;
    int n_items;
};

__global__ void __launch_bounds__(IT_THREADS, 1)
    nsa_imp_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap khimap,
                      const __grid_constant__ CUtensorMap klomap, const ImpTcParams ip) {
    grid_dependency_sync();
    constexpr int D = 128;
    using L = ItSmem;
    const TileParams &p = ip.t;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int nbk = ip.n_blocks;
    float *imp_s = reinterpret_cast<float *>(smem + L::OFF_IMP);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::off_bar(nbk));
    uint64_t *q_full = bars, *q_empty = bars + 1, *kv_full = bars + 2, *kv_empty = kv_full + IT_STAGES;
    uint64_t *s_full = kv_empty + IT_STAGES, *s_free = s_full + 2, *drain = s_free + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cpb = ip.sel_block / p.cmp_stride;              // compressed tokens per block (4..64, divides 64)
    const int nbh = (IT_KT / 2) / cpb;                        // blocks per half tile (<= 16)

    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 2 * IT_KT);   // S x2
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        tc::mbar_init(q_full, 1); tc::mbar_init(q_empty, 1);
        for (int i = 0; i < IT_STAGES; ++i) { tc::mbar_init(kv_full + i, 1); tc::mbar_init(kv_empty + i, 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(s_full + i, 1); tc::mbar_init(s_free + i, 256); }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() {
        raise_error(ip.err, ERR_TIMEOUT);
        *abort_flag = 1;
    };
    auto tiles_of = [&](int t0) -> int {
        const int t_last = min(t0 + CT_Q - 1, p.T - 1);
        return ((int)tile_key_end<TS_CMP>(p, t_last) + IT_KT - 1) / IT_KT;
    };

    if (warp == 0) {
        if (lane == 0) {
            bool ok = true;
            int tile = 0, qn = 0;
            for (int it = blockIdx.x; it < ip.n_items && ok; it += gridDim.x) {
                int b, g, t0;
                ct_item(p, it, b, g, t0);
                const int nt = tiles_of(t0);
                if (nt == 0) continue;
                if (!atc::wait(q_empty, (qn & 1) ^ 1, abort_flag)) { ok = false; break; }
                atc::expect_tx(q_full, L::Q_BYTES);
                for (int w = 0; w < CT_Q; ++w) {
                    const int qrow = (b * p.T + min(t0 + w, p.T - 1)) * p.Hq + g * p.G;
                    for (int h = 0; h < 2; ++h)
                        atc::load_2d(smem + L::OFF_Q + h * (128 * 128) + w * (16 * 128), &qmap, h * 64, qrow, q_full);
                }
                ++qn;
                for (int kt = 0; kt < nt; ++kt, ++tile) {
                    const int st = tile % IT_STAGES;
                    if (!atc::wait(kv_empty + st, ((tile / IT_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    atc::expect_tx(kv_full + st, L::STAGE);
                    unsigned char *dst = smem + L::OFF_KV + st * L::STAGE;
                    const int z = b * p.Lk + kt * IT_KT;
                    for (int h = 0; h < 2; ++h) {
                        atc::load_3d(dst + h * (IT_KT * 128), &khimap, h * 64, g, z, kv_full + st);
                        atc::load_3d(dst + L::KT_BYTES + h * (IT_KT * 128), &klomap, h * 64, g, z, kv_full + st);
                    }
                }
            }
            if (!ok) fail();
            if (qn > 0) tc::mbar_wait_bounded(q_full, (qn - 1) & 1, ATC_WAIT);
            for (int i = 0; i < IT_STAGES && i < tile; ++i) {
                const int kt = tile - 1 - i;
                tc::mbar_wait_bounded(kv_full + kt % IT_STAGES, (kt / IT_STAGES) & 1, ATC_WAIT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::make_idesc(1, 1, 128, IT_KT);
            const uint32_t qa = tc::smem_u32(smem + L::OFF_Q);
            bool ok = true;
            int tile = 0, qn = 0;
            for (int it = blockIdx.x; it < ip.n_items && ok; it += gridDim.x) {
                int b, g, t0;
                ct_item(p, it, b, g, t0);
                const int nt = tiles_of(t0);
                if (nt == 0) continue;
                if (!atc::wait(q_full, qn & 1, abort_flag)) { ok = false; break; }
                ++qn;
                for (int kt = 0; kt < nt; ++kt, ++tile) {
                    const int st = tile % IT_STAGES, sb = tile & 1;
                    if (!atc::wait(kv_full + st, (tile / IT_STAGES) & 1, abort_flag)) { ok = false; break; }
                    if (!atc::wait(s_free + sb, ((tile >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t ka = tc::smem_u32(smem + L::OFF_KV + st * L::STAGE);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const int h = ks / 4, kk = ks % 4;
                        const uint64_t ad = atc::desc_sw128(qa + h * (128 * 128) + kk * 32, 16, 1024);
                        const uint64_t bh = atc::desc_sw128(ka + h * (IT_KT * 128) + kk * 32, 16, 1024);
                        const uint64_t bl = atc::desc_sw128(ka + L::KT_BYTES + h * (IT_KT * 128) + kk * 32, 16, 1024);
                        tc::mma_bf16(tmem + sb * IT_KT, ad, bh, ID_S, ks > 0 ? 1u : 0u);
                        tc::mma_bf16(tmem + sb * IT_KT, ad, bl, ID_S, 1u);
                    }
                    tc::mma_commit(kv_empty + st);
                    tc::mma_commit(s_full + sb);
                    if (kt + 1 == nt) tc::mma_commit(q_empty);
                }
            }
            if (!ok) fail();
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, ATC_WAIT);
        }
        __syncwarp();
    } else {
        // two warps per TMEM lane quadrant: half 0 scores keys 0-63 of each
        // tile, half 1 keys 64-127; a block never straddles the halves
        const int quad = warp & 3, half = (warp - 2) >> 2;
        constexpr int SC = IT_KT / 2;
        const int r = quad * 32 + lane;                   // row = query w x 16 + head h
        const int w = r >> 4, h = r & 15;
        const uint32_t lrow = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        int tile = 0;
        for (int it = blockIdx.x; it < ip.n_items; it += gridDim.x) {
            int b, g, t0;
            ct_item(p, it, b, g, t0);
            const int nt = tiles_of(t0);
            const int t_last = min(t0 + CT_Q - 1, p.T - 1);
            const int t = t0 + w;
            const bool row_ok = t <= t_last && h < p.G;
            const int nv = t <= t_last ? (int)tile_key_end<TS_CMP>(p, t) : 0;
            const float ls = row_ok ? ip.lse_cmp[(long long)(b * p.T + t) * p.Hq + g * p.G + h] * kLog2e : 0.f;
            for (int kt = 0; kt < nt && ok; ++kt, ++tile) {
                const int sb = tile & 1;
                if (!__all_sync(0xffffffffu, atc::wait(s_full + sb, (tile >> 1) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                uint32_t sr[SC];
#pragma unroll
                for (int c = 0; c < SC; c += 16)
                    tc::tmem_ld16(tmem + lrow + sb * IT_KT + half * SC + c, *reinterpret_cast<uint32_t(*)[16]>(sr + c));
                tc::tmem_ld_wait();
                tc::fence_before_sync();
                atc::arrive(s_free + sb);
                // p = 2^(s * scale_log2 - lse_log2): one FFMA and one ex2 per score
                const int i0 = kt * IT_KT + half * SC;
                const bool full = row_ok && i0 + SC <= nv;
                float pv[SC];
#pragma unroll
                for (int k = 0; k < SC; ++k) {
                    const float e = ex2_fast(fmaf(__uint_as_float(sr[k]), p.scale_log2, -ls));
                    pv[k] = (full || (row_ok && i0 + k < nv)) ? e : 0.f;
                }
                float bs[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) bs[j] = 0.f;
                if (cpb == 4) {
#pragma unroll
                    for (int k = 0; k < SC; ++k) bs[k / 4] += pv[k];
                } else {
#pragma unroll
                    for (int k = 0; k < SC; ++k) {
                        const int j = k / cpb;                   // < 16 since cpb >= 4
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            if (jj == j) bs[jj] += pv[k];
                    }
                }
                // sum over the 16 heads of the query (lane bits 0-3): lane h
                // ends with the sum of block h of this half tile
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) {
                    const bool hi = (lane & o) != 0;
#pragma unroll
                    for (int j = 0; j < o; ++j) {
                        const float mine = hi ? bs[j + o] : bs[j];
                        const float other = hi ? bs[j] : bs[j + o];
                        bs[j] = mine + __shfl_xor_sync(0xffffffffu, other, o);
                    }
                }
                const int blk = (kt * 2 + half) * nbh + h;
                if (t <= t_last && h < nbh && blk < nbk) imp_s[w * nbk + blk] = bs[0];
            }
            // all importances of the item are in shared memory
            if (!atc::agree(1, 256, ok)) { ok = false; break; }
            const int covered = min(nt * 2 * nbh, nbk);
            {
                const int wq = warp - 2;                  // each score warp: one query
                const int tq = t0 + wq;
                if (tq <= t_last) {
                    float *imp = imp_s + wq * nbk;
                    const int nb_t = min(tq / ip.sel_block + 1, nbk);
                    const int k = min(ip.sel_topk, nb_t);
                    for (int i = covered + lane; i < nb_t; i += 32) imp[i] = 0.f;   // no visible token
                    __syncwarp();
                    int mine = -1;
                    for (int rr = 0; rr < k; ++rr) {
                        float bv = -1.f;
                        int bi = 0x7fffffff;
                        for (int i = lane; i < nb_t; i += 32) {
                            const float x = imp[i];
                            if (x > bv) { bv = x; bi = i; }  // lanes scan ascending i: ties keep the lower i
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
                        }
                        if (lane == rr) mine = bi < nb_t ? bi : -1;
                        if (lane == 0 && bi < nb_t) imp[bi] = -1.f;
                        __syncwarp();
                    }
                    int rank = 0;
                    for (int rr = 0; rr < k; ++rr) {
                        const int other = __shfl_sync(0xffffffffu, mine, rr);
                        rank += (lane < k && other < mine) ? 1 : 0;
                    }
                    int32_t *dst = ip.sel_idx + ((long long)(b * p.T + tq) * p.Hkv + g) * ip.sel_topk;
                    if (lane < k) dst[rank] = mine;
                    for (int i = k + lane; i < ip.sel_topk; i += 32) dst[i] = -1;
                }
            }
            // the next item's tiles overwrite imp_s
            if (!atc::agree(1, 256, ok)) { ok = false; break; }
        }
        if (!ok) fail();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 2 * IT_KT);
}

}  // namespace sa
