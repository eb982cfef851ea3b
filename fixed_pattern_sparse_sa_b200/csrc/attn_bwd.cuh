// attn_bwd.cuh -- backward of gathered-KV sparse attention over explicit
// index lists.
//
// The training results of the SpatialLM page ("SpatialLM-Mini acelero el
// entrenamiento ...") and the backward speed-up of the NSA page ("Native
// Sparse Attention ...", "Puntos Clave") need the gradient of the sparse
// forward.  For query t, head h and its set S (z_j = scale q.k_j,
// p_j = exp(z_j - lse), lse saved by the forward):
//   dP_j = dO . v_j,   D = dO . O = sum_j p_j dP_j,   dS_j = p_j (dP_j - D)
//   dq = scale sum_j dS_j k_j,  dk_j += scale dS_j q,  dv_j += p_j dO
//
// One warp per (query, KV group, 16-head chunk): the heads of the group are
// the 16 rows of m16 tiles, as in the forward.  Keys come in chunks of 16,
// gathered by cp.async (two stages) into XOR-swizzled shared memory.  Per
// chunk: S = Q K^T and dP = dO V^T (mma.sync m16n8k16, bf16 -> fp32), P and
// dS in registers, dq += dS K (kept in registers); dS^T and P^T go through a
// 16 x 16 shared-memory tile (ldmatrix.trans) to form dK = dS^T Q and
// dV = P^T dO for the chunk's 16 keys, which are added to the fp32 dk / dv
// with vector reductions (a key selected by several queries collects all of
// their contributions).  D comes from a first pass (attn_bwd_prep_kernel).
//
// The same kernel serves the NSA backward (Native Sparse Attention page,
// "Puntos Clave": natively trainable, with a faster backward pass).  The key
// source is a template parameter: explicit lists (BW_LIST), the keys of
// selected blocks masked to j <= t (BW_BLOCKS: the selected branch's dq), or
// a contiguous range per query (BW_RANGE: the sliding window, or the
// compressed rows visible to t, with the keys as a bf16 hi/lo pair (HILO) as
// in the forward; the range branches normally take attn_bwd_dq_tile_kernel
// or the tcgen05 kernels of nsa_bwd_tc.cuh instead).  A per-row factor (the
// branch gate) scales the upstream gradient, the LSE is read with a stride
// (the forward stores the three branches' LSEs side by side), and dq can
// accumulate over the branches' launches.  The key-major
// attn_bwd_kv_kernel below gives dk / dv without per-(query, key)
// reductions for the range branches and, over inverse block lists, for the
// selected blocks.
#pragma once

#include "attn_gather.cuh"

namespace sa {

enum { BW_LIST = 0, BW_BLOCKS = 1, BW_RANGE = 2 };

struct BwdParams {
    const __nv_bfloat16 *q, *k, *v, *o, *dout;   // q/o/dout [B,Tq,Hq,D], k/v [B,L,Hkv,D]
    const __nv_bfloat16 *klo;                    // HILO: low halves of the keys
    const float *lse;                            // [rows * lse_stride] natural log (forward)
    const int32_t *idx;                          // [B,Tq,idx_heads,K] keys (BW_LIST) or blocks (BW_BLOCKS)
    const float *gate;                           // nullable: factor on dO, gate[row * gate_stride]
    int B, Tq, L, Hq, Hkv, G, idx_heads, K;
    int lse_stride, gate_stride;
    int block, block_shift;                      // BW_BLOCKS: keys per block, log2 or -1
    int window, cmp_len, cmp_stride;             // BW_RANGE: window > 0, else compressed rows
    int dq_accum;                                // add to dq instead of writing it
    long long q_pos0;
    float scale, scale_log2;
    float *Dt;                                   // [B,Tq,Hq] dO . O
    float *dq;                                   // [B,Tq,Hq,D]
    float *dk, *dv;                              // [B,L,Hkv,D] (zeroed before)
    unsigned *err;
};

// D = sum_c dO[row, c] * O[row, c], one warp per row.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const BwdParams p, long long rows) {
    grid_dependency_sync();
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(p.dout + row * D);
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(p.o + row * D);
    float s = 0.f;
#pragma unroll
    for (int c = lane; c < D / 2; c += 32) {
        const float2 x = __bfloat1622float2(a[c]), y = __bfloat1622float2(b[c]);
        s += x.x * y.x + x.y * y.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) p.Dt[row] = s;
}

// Shared memory of one warp: K/V stages and their keys, the Q and dO tiles of
// the 16 heads and two 16 x 16 transpose tiles, rounded to 1 KB so that every
// warp's region (and each tile in it) stays 16-byte aligned.
template <int D, bool HILO = false>
__host__ __device__ constexpr int attn_bwd_warp_bytes() {
    return (2 * ((HILO ? 3 : 2) * 16 * D * 2 + 16 * 4) + 2 * 16 * D * 2 + 2 * 16 * 32 + 1023) / 1024 * 1024;
}

__device__ __forceinline__ void red_add2(float *addr, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};\n" ::"l"(addr), "f"(a), "f"(b) : "memory");
}

// ldmatrix of one 16 x 16 bf16 tile stored row-major with 32-byte rows
// (element (r, c) at r * 32 + c * 2): A fragment of the tile (trans = false)
// or of its transpose (trans = true).
template <bool TRANS>
__device__ __forceinline__ void ldsm_tile16(unsigned (&a)[4], const unsigned char *tile, int lane) {
    const int mi = lane >> 3, ri = lane & 7;
    if constexpr (!TRANS) {
        // matrices: rows 0-7 / 8-15 x cols 0-7 / 8-15 in A-fragment order
        const int row = (mi & 1) * 8 + ri, col = (mi >> 1) * 8;
        ldsm_x4(a[0], a[1], a[2], a[3], tile + row * 32 + col * 2);
    } else {
        // A of the transpose: (r, c) of A is tile (c, r)
        const int row = (mi >> 1) * 8 + ri, col = (mi & 1) * 8;
        ldsm_x4_t(a[0], a[1], a[2], a[3], tile + row * 32 + col * 2);
    }
}

// DKV = false: dq only (the key-major attn_bwd_kv_kernel gives dk / dv).
template <int D, int NW, int SRC = BW_LIST, bool HILO = false, bool DKV = true>
__global__ void __launch_bounds__(NW * 32) attn_bwd_kernel(const BwdParams p) {
    grid_dependency_sync();
    constexpr int NK = 16;                  // keys per chunk
    constexpr int STAGES = 2;
    constexpr int NARR = HILO ? 3 : 2;      // K (+ K low half) and V per stage
    constexpr int ROWB = D * 2;
    constexpr int UNITS = ROWB / 16;
    constexpr int CH = NK * ROWB;           // one K (or V) chunk
    constexpr int KS_D = D / 16;
    constexpr int NT_D = D / 8;
    constexpr int CP_ITERS = NK * UNITS / 32;
    constexpr int QT = 16 * ROWB;           // Q (or dO) tile of the 16 heads
    constexpr int WSM = attn_bwd_warp_bytes<D, HILO>();

    extern __shared__ __align__(1024) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *wsm = smem + warp * WSM;
    unsigned char *q_s = wsm;                       // [16 heads][D] swizzled
    unsigned char *do_s = q_s + QT;
    unsigned char *tp_s = do_s + QT;                // 16 x 16 bf16 tiles: dS, P
    unsigned char *kv_s = tp_s + 2 * 16 * 32;
    int *keys_s = reinterpret_cast<int *>(kv_s + STAGES * NARR * CH);

    const int n_hchunk = (p.G + 15) / 16;
    const long long n_items = (long long)p.B * p.Tq * p.Hkv * n_hchunk;
    const long long item = (long long)blockIdx.x * NW + warp;
    if (item >= n_items) return;
    long long rem = item;
    const int hc = (int)(rem % n_hchunk); rem /= n_hchunk;
    const int g = (int)(rem % p.Hkv); rem /= p.Hkv;
    const int t = (int)(rem % p.Tq); rem /= p.Tq;
    const int b = (int)rem;
    const long long pos = p.q_pos0 + t;

    const int gr = lane >> 2, qc = lane & 3;
    const int hr0 = hc * 16 + gr, hr1 = hr0 + 8;
    const bool v0 = hr0 < p.G, v1 = hr1 < p.G;
    const long long row0 = (long long)(b * p.Tq + t) * p.Hq + g * p.G + hr0;   // flat rows of the two heads
    const long long row1 = row0 + 8;

    // Q and dO of the 16 heads into shared memory (swizzled like K rows);
    // rows past the group are zero
    for (int i = lane; i < 16 * UNITS; i += 32) {
        const int r = i / UNITS, u = i % UNITS;
        const bool ok = hc * 16 + r < p.G;
        const long long base = ((long long)(b * p.Tq + t) * p.Hq + g * p.G + hc * 16 + r) * D + u * 8;
        const int sw = (u ^ (r & 7)) * 16;
        cp_async16(q_s + r * ROWB + sw, ok ? p.q + base : p.q, ok ? 16 : 0);
        cp_async16(do_s + r * ROWB + sw, ok ? p.dout + base : p.dout, ok ? 16 : 0);
    }
    cp_async_commit();
    const float lse0 = v0 ? p.lse[row0 * p.lse_stride] * kLog2e : 0.f;
    const float lse1 = v1 ? p.lse[row1 * p.lse_stride] * kLog2e : 0.f;
    const float D0 = v0 ? p.Dt[row0] : 0.f, D1 = v1 ? p.Dt[row1] : 0.f;
    const float gs0 = (p.gate && v0) ? p.gate[row0 * p.gate_stride] : 1.f;
    const float gs1 = (p.gate && v1) ? p.gate[row1 * p.gate_stride] : 1.f;
    // a row whose forward set was empty has lse = -inf: no gradient
    const bool live0 = v0 && lse0 != -INFINITY, live1 = v1 && lse1 != -INFINITY;

    // the query's key entries: list entries, block entries (K blocks x
    // block keys), or a range [lo, lo + n_e)
    const int32_t *list = SRC == BW_RANGE ? nullptr
        : p.idx + ((long long)(b * p.Tq + t) * p.idx_heads + (p.idx_heads == 1 ? 0 : g)) * p.K;
    int n_e = 0;
    long long lo = 0;
    if constexpr (SRC == BW_LIST) {
        n_e = p.K;
    } else if constexpr (SRC == BW_BLOCKS) {
        n_e = p.K * p.block;
    } else {
        if (p.window > 0) {
            lo = pos - p.window + 1 > 0 ? pos - p.window + 1 : 0;
            n_e = (int)(pos + 1 - lo);
        } else {
            const long long nv = pos >= p.cmp_len - 1 ? (pos - p.cmp_len + 1) / p.cmp_stride + 1 : 0;
            n_e = (int)(nv < p.L ? nv : p.L);
        }
    }
    const int n_chunks = (n_e + NK - 1) / NK;
    const __nv_bfloat16 *kb = p.k + ((long long)b * p.L * p.Hkv + g) * D;
    const __nv_bfloat16 *klb = HILO ? p.klo + ((long long)b * p.L * p.Hkv + g) * D : nullptr;
    const __nv_bfloat16 *vb = p.v + ((long long)b * p.L * p.Hkv + g) * D;
    const long long rstride = (long long)p.Hkv * D;

    auto issue = [&](int ci) {
        const int st = ci % STAGES;
        unsigned char *ks_ = kv_s + st * NARR * CH;
        unsigned char *vs_ = ks_ + CH;
        unsigned char *ls_ = vs_ + CH;          // HILO: K low halves
        int j = -1;
        if (ci < n_chunks && lane < NK) {
            const int e = ci * NK + lane;
            if (e < n_e) {
                if constexpr (SRC == BW_LIST) {
                    const int raw = __ldg(list + e);
                    if (raw >= 0) {
                        if (raw >= p.L || (long long)raw > pos) raise_error(p.err, ERR_BAD_INDEX);
                        else j = raw;
                    }
                } else if constexpr (SRC == BW_BLOCKS) {
                    const int bi = p.block_shift >= 0 ? e >> p.block_shift : e / p.block;
                    const int blk = __ldg(list + bi);
                    if (blk >= 0) {
                        const long long j0 = (long long)blk * p.block;
                        const long long jj = j0 + (e - bi * p.block);
                        if (j0 >= p.L) raise_error(p.err, ERR_BAD_INDEX);
                        else if (jj <= pos && jj < p.L) j = (int)jj;
                    }
                } else {
                    j = (int)(lo + e);
                }
            }
            keys_s[st * NK + lane] = j;
        }
        if (ci < n_chunks) {
#pragma unroll
            for (int it = 0; it < CP_ITERS; ++it) {
                const int lin = it * 32 + lane;
                const int rr = lin / UNITS, u = lin % UNITS;
                const int jr = __shfl_sync(0xffffffffu, j, rr);
                const long long off = jr >= 0 ? (long long)jr * rstride + u * 8 : 0;
                const int sw = (u ^ (rr & 7)) * 16;
                cp_async16(ks_ + rr * ROWB + sw, kb + off, jr >= 0 ? 16 : 0);
                cp_async16(vs_ + rr * ROWB + sw, vb + off, jr >= 0 ? 16 : 0);
                if constexpr (HILO) cp_async16(ls_ + rr * ROWB + sw, klb + off, jr >= 0 ? 16 : 0);
            }
        }
        cp_async_commit();
    };

    float dqa[NT_D][4];
#pragma unroll
    for (int i = 0; i < NT_D; ++i) dqa[i][0] = dqa[i][1] = dqa[i][2] = dqa[i][3] = 0.f;

    issue(0);
    for (int ci = 0; ci < n_chunks; ++ci) {
        issue(ci + 1);
        cp_async_wait<1>();
        __syncwarp();
        const int st = ci % STAGES;
        const unsigned char *ks_ = kv_s + st * NARR * CH;
        const unsigned char *vs_ = ks_ + CH;
        const unsigned char *ls_ = vs_ + CH;
        const int jl = lane < NK ? keys_s[st * NK + lane] : -1;
        const unsigned vmask = __ballot_sync(0xffffffffu, jl >= 0);
        if (vmask != 0u) {
            // S = Q K^T and dP = dO V^T over the head dimension
            float sc[2][4], dp[2][4];
#pragma unroll
            for (int i = 0; i < 2; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS_D; ++ks) {
                const int mi = lane >> 3, ri = lane & 7;
                unsigned qa[4], da[4];
                {
                    // A fragments of Q and dO (rows = heads) for k-step ks
                    const int row = (mi & 1) * 8 + ri, unit = ks * 2 + (mi >> 1);
                    ldsm_x4(qa[0], qa[1], qa[2], qa[3], q_s + row * ROWB + ((unit ^ (row & 7)) * 16));
                    ldsm_x4(da[0], da[1], da[2], da[3], do_s + row * ROWB + ((unit ^ (row & 7)) * 16));
                }
                const int key = (mi >> 1) * 8 + ri;
                const int unit = ks * 2 + (mi & 1);
                unsigned b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, ks_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                mma_bf16_16816(sc[0], qa, b0, b1);
                mma_bf16_16816(sc[1], qa, b2, b3);
                if constexpr (HILO) {
                    ldsm_x4(b0, b1, b2, b3, ls_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                    mma_bf16_16816(sc[0], qa, b0, b1);
                    mma_bf16_16816(sc[1], qa, b2, b3);
                }
                ldsm_x4(b0, b1, b2, b3, vs_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                mma_bf16_16816(dp[0], da, b0, b1);
                mma_bf16_16816(dp[1], da, b2, b3);
            }
            // P = exp(z - lse), dS = P (dP - D); masked keys and dead rows give 0
            float pr[2][4], ds[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int kk = nt * 8 + 2 * qc + (e & 1);
                    const bool hi = e >> 1;
                    const bool ok = ((vmask >> kk) & 1u) && (hi ? live1 : live0);
                    const float pv = ok ? ex2_fast(sc[nt][e] * p.scale_log2 - (hi ? lse1 : lse0)) : 0.f;
                    const float gv = pv * (hi ? gs1 : gs0);
                    pr[nt][e] = gv;
                    ds[nt][e] = gv * (dp[nt][e] - (hi ? D1 : D0));
                }
            }
            // dS and P as bf16 A fragments (rows = heads, k = keys)
            unsigned dsa[4], pa[4];
            dsa[0] = pack_bf16(ds[0][0], ds[0][1]); dsa[1] = pack_bf16(ds[0][2], ds[0][3]);
            dsa[2] = pack_bf16(ds[1][0], ds[1][1]); dsa[3] = pack_bf16(ds[1][2], ds[1][3]);
            pa[0] = pack_bf16(pr[0][0], pr[0][1]); pa[1] = pack_bf16(pr[0][2], pr[0][3]);
            pa[2] = pack_bf16(pr[1][0], pr[1][1]); pa[3] = pack_bf16(pr[1][2], pr[1][3]);
            // dq += dS K  (B = K rows [key][d], transposed loads as V in the forward)
#pragma unroll
            for (int dpi = 0; dpi < NT_D / 2; ++dpi) {
                const int mi = lane >> 3, ri = lane & 7;
                const int key = (mi & 1) * 8 + ri;
                const int unit = dpi * 2 + (mi >> 1);
                unsigned b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, ks_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                mma_bf16_16816(dqa[2 * dpi], dsa, b0, b1);
                mma_bf16_16816(dqa[2 * dpi + 1], dsa, b2, b3);
                if constexpr (HILO) {
                    ldsm_x4_t(b0, b1, b2, b3, ls_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                    mma_bf16_16816(dqa[2 * dpi], dsa, b0, b1);
                    mma_bf16_16816(dqa[2 * dpi + 1], dsa, b2, b3);
                }
            }
            if constexpr (DKV) {
            // dS and P tiles (row = head, col = key) for the transposed products
            {
                unsigned *t0 = reinterpret_cast<unsigned *>(tp_s);
                unsigned *t1 = reinterpret_cast<unsigned *>(tp_s + 16 * 32);
                // element (head gr / gr+8, key 2qc..2qc+1 / +8) of the C layout
                t0[gr * 8 + qc] = dsa[0];       t0[(gr + 8) * 8 + qc] = dsa[1];
                t0[gr * 8 + 4 + qc] = dsa[2];   t0[(gr + 8) * 8 + 4 + qc] = dsa[3];
                t1[gr * 8 + qc] = pa[0];        t1[(gr + 8) * 8 + qc] = pa[1];
                t1[gr * 8 + 4 + qc] = pa[2];    t1[(gr + 8) * 8 + 4 + qc] = pa[3];
            }
            __syncwarp();
            unsigned dsT[4], pT[4];
            ldsm_tile16<true>(dsT, tp_s, lane);
            ldsm_tile16<true>(pT, tp_s + 16 * 32, lane);
            // dK = scale dS^T Q and dV = P^T dO for the 16 keys (rows gr, gr+8),
            // 16 columns at a time, added to the global accumulators
            const int j0 = __shfl_sync(0xffffffffu, jl, gr), j1 = __shfl_sync(0xffffffffu, jl, gr + 8);
            float *dk0 = p.dk + ((long long)(b * p.L + (j0 >= 0 ? j0 : 0)) * p.Hkv + g) * D;
            float *dk1 = p.dk + ((long long)(b * p.L + (j1 >= 0 ? j1 : 0)) * p.Hkv + g) * D;
            float *dv0 = p.dv + ((long long)(b * p.L + (j0 >= 0 ? j0 : 0)) * p.Hkv + g) * D;
            float *dv1 = p.dv + ((long long)(b * p.L + (j1 >= 0 ? j1 : 0)) * p.Hkv + g) * D;
#pragma unroll
            for (int dpi = 0; dpi < NT_D / 2; ++dpi) {
                const int mi = lane >> 3, ri = lane & 7;
                const int hrow = (mi & 1) * 8 + ri;
                const int unit = dpi * 2 + (mi >> 1);
                unsigned b0, b1, b2, b3;
                float ck[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                float cv[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                ldsm_x4_t(b0, b1, b2, b3, q_s + hrow * ROWB + ((unit ^ (hrow & 7)) * 16));
                mma_bf16_16816(ck[0], dsT, b0, b1);
                mma_bf16_16816(ck[1], dsT, b2, b3);
                ldsm_x4_t(b0, b1, b2, b3, do_s + hrow * ROWB + ((unit ^ (hrow & 7)) * 16));
                mma_bf16_16816(cv[0], pT, b0, b1);
                mma_bf16_16816(cv[1], pT, b2, b3);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int col = (2 * dpi + h2) * 8 + 2 * qc;
                    if (j0 >= 0) {
                        red_add2(dk0 + col, ck[h2][0] * p.scale, ck[h2][1] * p.scale);
                        red_add2(dv0 + col, cv[h2][0], cv[h2][1]);
                    }
                    if (j1 >= 0) {
                        red_add2(dk1 + col, ck[h2][2] * p.scale, ck[h2][3] * p.scale);
                        red_add2(dv1 + col, cv[h2][2], cv[h2][3]);
                    }
                }
            }
            }   // DKV
        }
        __syncwarp();
    }
    cp_async_wait<0>();
#pragma unroll
    for (int nt = 0; nt < NT_D; ++nt) {
        const int col = nt * 8 + 2 * qc;
        float2 a0 = make_float2(dqa[nt][0] * p.scale, dqa[nt][1] * p.scale);
        float2 a1 = make_float2(dqa[nt][2] * p.scale, dqa[nt][3] * p.scale);
        float2 *q0 = reinterpret_cast<float2 *>(p.dq + row0 * D + col);
        float2 *q1 = reinterpret_cast<float2 *>(p.dq + row1 * D + col);
        if (p.dq_accum) {
            if (v0) { const float2 o = *q0; a0.x += o.x; a0.y += o.y; }
            if (v1) { const float2 o = *q1; a1.x += o.x; a1.y += o.y; }
        }
        if (v0) *q0 = a0;
        if (v1) *q1 = a1;
    }
}

// Key-major backward of a range branch (the sliding window, or the
// compressed rows): dK and dV of a block of KB = 16 * KV_NWK keys of one KV
// group, summed in registers over the queries that see them, so that a key
// gets one reduction per CTA instead of one per (query, key).  The queries
// seeing the block are cut into splits of q_split (one CTA each).  The CTA
// stages the block's K (and K low halves) and V once; per query and 16-head
// chunk it stages Q_t and dO_t (two stages, cp.async) with the heads' lse,
// D and gate.  Warp w owns keys 16w .. 16w+15: S^T = K Q_t^T and
// dP^T = V dO_t^T (rows = keys, columns = heads), P^T and dS^T in registers,
// dV += P^T dO_t and dK += dS^T Q_t with the C fragments reused as A
// fragments.  dq of the branch comes from attn_bwd_kernel with DKV = false.
constexpr int KV_NWK = 4;

// Selected branch: the queries that chose each block, as lists per
// (b, g, block) (built by the three kernels below), cut into work items of
// at most q_split queries.
struct KvLists {
    const int32_t *qlist;   // queries, grouped by list
    const int32_t *qoff;    // [n_lists + 1] list starts
    const int2 *items;      // (list, split) work items
    const int32_t *n_items; // device count of items
    int nb;                 // selection blocks per sequence
    int sel_block;
    int n_kbpb;             // key blocks of KB keys per selection block
};

template <int D, bool HILO>
constexpr int attn_bwd_kv_smem() {
    return (HILO ? 3 : 2) * 16 * KV_NWK * D * 2 + 2 * ((2 * 16 * D * 2 + 3 * 16 * 4 + 1023) / 1024 * 1024);
}

// Queries that see at least one key of [j_first, j_last] (range branches).
__device__ __forceinline__ void kv_query_range(const BwdParams &p, long long j_first, long long j_last,
                                               long long &q_lo, long long &q_hi) {
    if (p.window > 0) {
        q_lo = j_first;
        q_hi = j_last + p.window < (long long)p.Tq ? j_last + p.window : (long long)p.Tq;
    } else {
        q_lo = j_first * p.cmp_stride + p.cmp_len - 1;
        q_hi = p.Tq;
    }
}

template <int D, bool HILO, bool LISTS = false>
__global__ void __launch_bounds__(KV_NWK * 32) attn_bwd_kv_kernel(const BwdParams p, int n_kb, int n_split,
                                                                  int q_split, const KvLists kl) {
    grid_dependency_sync();
    constexpr int KB = 16 * KV_NWK;
    constexpr int NT = KV_NWK * 32;
    constexpr int ROWB = D * 2;
    constexpr int UNITS = ROWB / 16;
    constexpr int KS_D = D / 16;
    constexpr int NT_D = D / 8;
    constexpr int KCH = KB * ROWB;
    constexpr int QT = 16 * ROWB;
    constexpr int QSTAGE = (2 * QT + 3 * 16 * 4 + 1023) / 1024 * 1024;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *k_s = smem;
    unsigned char *v_s = smem + KCH;
    unsigned char *l_s = smem + 2 * KCH;                    // HILO: K low halves
    unsigned char *qst = smem + (HILO ? 3 : 2) * KCH;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, qc = lane & 3;
    int b, g;
    long long j_first, j_end, qa, qe;
    const int32_t *ql = nullptr;
    if constexpr (LISTS) {
        // work item (list, split) x key block of the selection block
        const int item = blockIdx.x / kl.n_kbpb, kbs = blockIdx.x % kl.n_kbpb;
        if (item >= *kl.n_items) return;
        const int2 wi = kl.items[item];
        const int blk = wi.x % kl.nb;
        g = (wi.x / kl.nb) % p.Hkv;
        b = wi.x / kl.nb / p.Hkv;
        j_first = (long long)blk * kl.sel_block + (long long)kbs * KB;
        j_end = (long long)blk * kl.sel_block + kl.sel_block;
        if (j_end > p.L) j_end = p.L;
        if (j_first >= j_end) return;
        const long long o0 = kl.qoff[wi.x], o1 = kl.qoff[wi.x + 1];
        qa = o0 + (long long)wi.y * q_split;
        qe = qa + q_split < o1 ? qa + q_split : o1;
        ql = kl.qlist;
    } else {
        long long rem = blockIdx.x;
        const int s = (int)(rem % n_split); rem /= n_split;
        const int kb = (int)(rem % n_kb); rem /= n_kb;
        g = (int)(rem % p.Hkv); rem /= p.Hkv;
        b = (int)rem;
        j_first = (long long)kb * KB;
        if (j_first >= p.L) return;
        j_end = j_first + KB < (long long)p.L ? j_first + KB : (long long)p.L;
        long long q_lo, q_hi;
        kv_query_range(p, j_first, j_end - 1, q_lo, q_hi);
        qa = q_lo + (long long)s * q_split;
        qe = qa + q_split < q_hi ? qa + q_split : q_hi;
    }
    if (qa >= qe) return;                                   // the whole CTA leaves together
    const int n_hc = (p.G + 15) / 16;
    const int n_it = (int)(qe - qa) * n_hc;

    // the key block (rows past L are zero)
    const long long rstride = (long long)p.Hkv * D;
    const __nv_bfloat16 *kbase = p.k + ((long long)b * p.L * p.Hkv + g) * D;
    const __nv_bfloat16 *vbase = p.v + ((long long)b * p.L * p.Hkv + g) * D;
    const __nv_bfloat16 *lbase = HILO ? p.klo + ((long long)b * p.L * p.Hkv + g) * D : nullptr;
    for (int i = threadIdx.x; i < KB * UNITS; i += NT) {
        const int r = i / UNITS, u = i % UNITS;
        const long long j = j_first + r;
        const bool ok = j < j_end;
        const long long off = ok ? j * rstride + u * 8 : 0;
        const int sw = (u ^ (r & 7)) * 16;
        cp_async16(k_s + r * ROWB + sw, kbase + off, ok ? 16 : 0);
        cp_async16(v_s + r * ROWB + sw, vbase + off, ok ? 16 : 0);
        if constexpr (HILO) cp_async16(l_s + r * ROWB + sw, lbase + off, ok ? 16 : 0);
    }

    // one query stage: Q_t and dO_t of 16 heads, then lse2 / D / gate of the heads
    auto issue = [&](int it) {
        if (it < n_it) {
            const long long t = LISTS ? (long long)__ldg(ql + qa + it / n_hc) : qa + it / n_hc;
            const int hc = it % n_hc;
            unsigned char *st = qst + (it & 1) * QSTAGE;
            float *fs = reinterpret_cast<float *>(st + 2 * QT);
            const long long row0 = ((long long)b * p.Tq + t) * p.Hq + (long long)g * p.G + hc * 16;
            for (int i = threadIdx.x; i < 16 * UNITS; i += NT) {
                const int r = i / UNITS, u = i % UNITS;
                const bool ok = hc * 16 + r < p.G;
                const long long src = (row0 + r) * D + u * 8;
                const int sw = (u ^ (r & 7)) * 16;
                cp_async16(st + r * ROWB + sw, ok ? p.q + src : p.q, ok ? 16 : 0);
                cp_async16(st + QT + r * ROWB + sw, ok ? p.dout + src : p.dout, ok ? 16 : 0);
            }
            if (threadIdx.x < 48) {
                // lse, D and gate of the 16 heads, copied asynchronously with the
                // tiles (zero past the group: a zero gate gives P = 0)
                const int r = threadIdx.x & 15, which = threadIdx.x >> 4;
                const bool ok = hc * 16 + r < p.G;
                const long long row = row0 + r;
                const float *src = which == 0 ? p.lse + row * p.lse_stride
                                 : which == 1 ? p.Dt + row
                                 : (p.gate ? p.gate + row * p.gate_stride : p.lse);
                if (which == 2 && !p.gate && ok) fs[32 + r] = 1.f;
                else cp_async4_zfill(fs + which * 16 + r, ok ? src : p.lse, ok ? 4 : 0);
            }
        }
        cp_async_commit();
    };

    float dka[NT_D][4], dva[NT_D][4];
#pragma unroll
    for (int i = 0; i < NT_D; ++i) {
        dka[i][0] = dka[i][1] = dka[i][2] = dka[i][3] = 0.f;
        dva[i][0] = dva[i][1] = dva[i][2] = dva[i][3] = 0.f;
    }
    const long long jk0 = j_first + warp * 16 + gr, jk1 = jk0 + 8;
    const unsigned char *kw = k_s + warp * 16 * ROWB;
    const unsigned char *vw = v_s + warp * 16 * ROWB;
    const unsigned char *lw = l_s + warp * 16 * ROWB;

    issue(0);
    for (int it = 0; it < n_it; ++it) {
        issue(it + 1);
        cp_async_wait<1>();
        __syncthreads();
        const long long t = LISTS ? (long long)__ldg(ql + qa + it / n_hc) : qa + it / n_hc;
        const unsigned char *q_t = qst + (it & 1) * QSTAGE;
        const unsigned char *do_t = q_t + QT;
        const float *fs = reinterpret_cast<const float *>(q_t + 2 * QT);
        auto visible = [&](long long j) -> bool {
            if (j >= j_end) return false;
            if (LISTS) return j <= t;
            if (p.window > 0) return j <= t && j > t - p.window;
            return j * p.cmp_stride + p.cmp_len - 1 <= t;
        };
        const bool vk0 = visible(jk0), vk1 = visible(jk1);
        if (__any_sync(0xffffffffu, vk0 || vk1)) {
            float sc[2][4], dp[2][4];
#pragma unroll
            for (int i = 0; i < 2; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
            const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
            for (int ks = 0; ks < KS_D; ++ks) {
                unsigned ka[4], va[4];
                {
                    // A fragments: the warp's 16 keys (rows) for k-step ks
                    const int row = (mi & 1) * 8 + ri, unit = ks * 2 + (mi >> 1);
                    ldsm_x4(ka[0], ka[1], ka[2], ka[3], kw + row * ROWB + ((unit ^ (row & 7)) * 16));
                    ldsm_x4(va[0], va[1], va[2], va[3], vw + row * ROWB + ((unit ^ (row & 7)) * 16));
                }
                // B fragments: the 16 heads of Q_t / dO_t (columns)
                const int hrow = (mi >> 1) * 8 + ri;
                const int unit = ks * 2 + (mi & 1);
                unsigned b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, q_t + hrow * ROWB + ((unit ^ (hrow & 7)) * 16));
                mma_bf16_16816(sc[0], ka, b0, b1);
                mma_bf16_16816(sc[1], ka, b2, b3);
                if constexpr (HILO) {
                    unsigned la[4];
                    const int row = (mi & 1) * 8 + ri, unit2 = ks * 2 + (mi >> 1);
                    ldsm_x4(la[0], la[1], la[2], la[3], lw + row * ROWB + ((unit2 ^ (row & 7)) * 16));
                    mma_bf16_16816(sc[0], la, b0, b1);
                    mma_bf16_16816(sc[1], la, b2, b3);
                }
                ldsm_x4(b0, b1, b2, b3, do_t + hrow * ROWB + ((unit ^ (hrow & 7)) * 16));
                mma_bf16_16816(dp[0], va, b0, b1);
                mma_bf16_16816(dp[1], va, b2, b3);
            }
            // P^T (gate folded in) and dS^T: rows = keys gr / gr+8, columns = heads;
            // a head with no key (lse = -inf) gets P = 0
            float pg[2][4], ds[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int h = nt * 8 + 2 * qc + (e & 1);
                    const bool vk = (e >> 1) ? vk1 : vk0;
                    const float lh = fs[h];
                    const float pv = (vk && lh != -INFINITY) ? ex2_fast(sc[nt][e] * p.scale_log2 - lh * kLog2e) : 0.f;
                    const float gv = pv * fs[32 + h];
                    pg[nt][e] = gv;
                    ds[nt][e] = gv * (dp[nt][e] - fs[16 + h]);
                }
            }
            unsigned pa[4], dsa[4];
            pa[0] = pack_bf16(pg[0][0], pg[0][1]); pa[1] = pack_bf16(pg[0][2], pg[0][3]);
            pa[2] = pack_bf16(pg[1][0], pg[1][1]); pa[3] = pack_bf16(pg[1][2], pg[1][3]);
            dsa[0] = pack_bf16(ds[0][0], ds[0][1]); dsa[1] = pack_bf16(ds[0][2], ds[0][3]);
            dsa[2] = pack_bf16(ds[1][0], ds[1][1]); dsa[3] = pack_bf16(ds[1][2], ds[1][3]);
            // dV += P^T dO_t, dK += dS^T Q_t (B = the [head][d] tiles, transposed loads)
#pragma unroll
            for (int dpi = 0; dpi < NT_D / 2; ++dpi) {
                const int hrow = (mi & 1) * 8 + ri;
                const int unit = dpi * 2 + (mi >> 1);
                unsigned b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, do_t + hrow * ROWB + ((unit ^ (hrow & 7)) * 16));
                mma_bf16_16816(dva[2 * dpi], pa, b0, b1);
                mma_bf16_16816(dva[2 * dpi + 1], pa, b2, b3);
                ldsm_x4_t(b0, b1, b2, b3, q_t + hrow * ROWB + ((unit ^ (hrow & 7)) * 16));
                mma_bf16_16816(dka[2 * dpi], dsa, b0, b1);
                mma_bf16_16816(dka[2 * dpi + 1], dsa, b2, b3);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
    // one reduction per key and column for this CTA's queries
    float *dk0 = p.dk + ((long long)(b * (long long)p.L + (jk0 < j_end ? jk0 : 0)) * p.Hkv + g) * D;
    float *dk1 = p.dk + ((long long)(b * (long long)p.L + (jk1 < j_end ? jk1 : 0)) * p.Hkv + g) * D;
    float *dv0 = p.dv + ((long long)(b * (long long)p.L + (jk0 < j_end ? jk0 : 0)) * p.Hkv + g) * D;
    float *dv1 = p.dv + ((long long)(b * (long long)p.L + (jk1 < j_end ? jk1 : 0)) * p.Hkv + g) * D;
#pragma unroll
    for (int nt = 0; nt < NT_D; ++nt) {
        const int col = nt * 8 + 2 * qc;
        if (jk0 < j_end) {
            red_add2(dk0 + col, dka[nt][0] * p.scale, dka[nt][1] * p.scale);
            red_add2(dv0 + col, dva[nt][0], dva[nt][1]);
        }
        if (jk1 < j_end) {
            red_add2(dk1 + col, dka[nt][2] * p.scale, dka[nt][3] * p.scale);
            red_add2(dv1 + col, dva[nt][2], dva[nt][3]);
        }
    }
}

// dq of a range branch (the window, or the compressed rows) with the keys
// shared: a CTA = 8 consecutive queries of one KV group (one warp each, the
// group's 16-head chunk hc); chunks of 32 keys of the union of their ranges
// are staged once per CTA (K, K low halves, V; two stages, cp.async) and
// every warp runs S = Q K^T, dP = dO V^T, dS = gate P (dP - D) and
// dq += dS K on its own query (Q and dO A fragments held in registers).
constexpr int DQ_WARPS = 8;
constexpr int DQ_NK = 32;

template <int D, bool HILO>
constexpr int attn_bwd_dq_tile_smem() {
    return 2 * (HILO ? 3 : 2) * DQ_NK * D * 2;
}

template <int D, bool HILO>
__global__ void __launch_bounds__(DQ_WARPS * 32) attn_bwd_dq_tile_kernel(const BwdParams p) {
    grid_dependency_sync();
    constexpr int ROWB = D * 2;
    constexpr int UNITS = ROWB / 16;
    constexpr int KS_D = D / 16;
    constexpr int NT_D = D / 8;
    constexpr int NARR = HILO ? 3 : 2;
    constexpr int CH = DQ_NK * ROWB;
    constexpr int CP_ITERS = NARR * DQ_NK * UNITS / (DQ_WARPS * 32);
    static_assert(CP_ITERS * DQ_WARPS * 32 == NARR * DQ_NK * UNITS, "copy split");
    extern __shared__ __align__(1024) unsigned char smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, qc = lane & 3;
    const int n_hc = (p.G + 15) / 16;
    const int nqb = (p.Tq + DQ_WARPS - 1) / DQ_WARPS;
    long long rem = blockIdx.x;
    const int qb = (int)(rem % nqb); rem /= nqb;
    const int hc = (int)(rem % n_hc); rem /= n_hc;
    const int g = (int)(rem % p.Hkv); rem /= p.Hkv;
    const int b = (int)rem;
    const int t = qb * DQ_WARPS + warp;
    const bool tv = t < p.Tq;
    const int t_first = qb * DQ_WARPS;
    const int t_last = min(t_first + DQ_WARPS, p.Tq) - 1;
    // key range of a query, and the union over the CTA's queries
    auto range_of = [&](long long tt, long long &lo, long long &hi) {
        if (p.window > 0) {
            lo = tt - p.window + 1 > 0 ? tt - p.window + 1 : 0;
            hi = tt + 1;
        } else {
            const long long nv = tt >= p.cmp_len - 1 ? (tt - p.cmp_len + 1) / p.cmp_stride + 1 : 0;
            lo = 0;
            hi = nv < p.L ? nv : p.L;
        }
    };
    long long u_lo, u_hi, dummy, w_lo = 0, w_hi = 0;
    range_of(t_first, u_lo, dummy);
    range_of(t_last, dummy, u_hi);
    if (tv) range_of(t, w_lo, w_hi);
    const int n_chunks = u_hi > u_lo ? (int)((u_hi - u_lo + DQ_NK - 1) / DQ_NK) : 0;

    const int hr0 = hc * 16 + gr, hr1 = hr0 + 8;
    const bool v0 = tv && hr0 < p.G, v1 = tv && hr1 < p.G;
    const long long rowb = ((long long)b * p.Tq + (tv ? t : 0)) * p.Hq + (long long)g * p.G + hc * 16;
    const long long row0 = rowb + gr, row1 = row0 + 8;
    float lse0 = v0 ? p.lse[row0 * p.lse_stride] : -INFINITY, lse1 = v1 ? p.lse[row1 * p.lse_stride] : -INFINITY;
    const bool live0 = v0 && lse0 != -INFINITY, live1 = v1 && lse1 != -INFINITY;
    lse0 *= kLog2e; lse1 *= kLog2e;
    const float D0 = v0 ? p.Dt[row0] : 0.f, D1 = v1 ? p.Dt[row1] : 0.f;
    const float gs0 = (p.gate && v0) ? p.gate[row0 * p.gate_stride] : 1.f;
    const float gs1 = (p.gate && v1) ? p.gate[row1 * p.gate_stride] : 1.f;
    // Q and dO A fragments of the 16 heads (zero past the group)
    unsigned qa[KS_D][4], da[KS_D][4];
#pragma unroll
    for (int ks = 0; ks < KS_D; ++ks) {
        const int c0 = ks * 16 + 2 * qc;
        const unsigned *q0 = reinterpret_cast<const unsigned *>(p.q + row0 * D + c0);
        const unsigned *q1 = reinterpret_cast<const unsigned *>(p.q + row1 * D + c0);
        const unsigned *d0 = reinterpret_cast<const unsigned *>(p.dout + row0 * D + c0);
        const unsigned *d1 = reinterpret_cast<const unsigned *>(p.dout + row1 * D + c0);
        qa[ks][0] = v0 ? __ldg(q0) : 0u; qa[ks][1] = v1 ? __ldg(q1) : 0u;
        qa[ks][2] = v0 ? __ldg(q0 + 4) : 0u; qa[ks][3] = v1 ? __ldg(q1 + 4) : 0u;
        da[ks][0] = v0 ? __ldg(d0) : 0u; da[ks][1] = v1 ? __ldg(d1) : 0u;
        da[ks][2] = v0 ? __ldg(d0 + 4) : 0u; da[ks][3] = v1 ? __ldg(d1 + 4) : 0u;
    }

    const long long rstride = (long long)p.Hkv * D;
    const __nv_bfloat16 *kbase = p.k + ((long long)b * p.L * p.Hkv + g) * D;
    const __nv_bfloat16 *vbase = p.v + ((long long)b * p.L * p.Hkv + g) * D;
    const __nv_bfloat16 *lbase = HILO ? p.klo + ((long long)b * p.L * p.Hkv + g) * D : nullptr;
    auto issue = [&](int ci) {
        if (ci < n_chunks) {
            unsigned char *st = smem + (ci & 1) * NARR * CH;
#pragma unroll
            for (int it = 0; it < CP_ITERS; ++it) {
                const int lin = (it * DQ_WARPS + warp) * 32 + lane;
                const int arr = lin / (DQ_NK * UNITS);
                const int rr = (lin / UNITS) % DQ_NK, u = lin % UNITS;
                const long long j = u_lo + (long long)ci * DQ_NK + rr;
                const bool ok = j < u_hi;
                const __nv_bfloat16 *src = arr == 0 ? kbase : (arr == 1 ? vbase : lbase);
                cp_async16(st + arr * CH + rr * ROWB + ((u ^ (rr & 7)) * 16),
                           ok ? src + j * rstride + u * 8 : kbase, ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };

    float dqa[NT_D][4];
#pragma unroll
    for (int i = 0; i < NT_D; ++i) dqa[i][0] = dqa[i][1] = dqa[i][2] = dqa[i][3] = 0.f;
    issue(0);
    for (int ci = 0; ci < n_chunks; ++ci) {
        issue(ci + 1);
        cp_async_wait<1>();
        __syncthreads();
        const long long j0 = u_lo + (long long)ci * DQ_NK;
        if (tv && j0 < w_hi && j0 + DQ_NK > w_lo) {
            const unsigned char *ks_ = smem + (ci & 1) * NARR * CH;
            const unsigned char *vs_ = ks_ + CH;
            const unsigned char *ls_ = vs_ + CH;
            const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
            for (int kh = 0; kh < DQ_NK / 16; ++kh) {
                float sc[2][4], dp[2][4];
#pragma unroll
                for (int i = 0; i < 2; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
                const int key = kh * 16 + (mi >> 1) * 8 + ri;
#pragma unroll
                for (int ks = 0; ks < KS_D; ++ks) {
                    const int unit = ks * 2 + (mi & 1);
                    unsigned b0, b1, b2, b3;
                    ldsm_x4(b0, b1, b2, b3, ks_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                    mma_bf16_16816(sc[0], qa[ks], b0, b1);
                    mma_bf16_16816(sc[1], qa[ks], b2, b3);
                    if constexpr (HILO) {
                        ldsm_x4(b0, b1, b2, b3, ls_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                        mma_bf16_16816(sc[0], qa[ks], b0, b1);
                        mma_bf16_16816(sc[1], qa[ks], b2, b3);
                    }
                    ldsm_x4(b0, b1, b2, b3, vs_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                    mma_bf16_16816(dp[0], da[ks], b0, b1);
                    mma_bf16_16816(dp[1], da[ks], b2, b3);
                }
                // dS = gate P (dP - D) over this query's own range
                float ds[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const long long j = j0 + kh * 16 + nt * 8 + 2 * qc + (e & 1);
                        const bool hi = e >> 1;
                        const bool ok = j >= w_lo && j < w_hi && (hi ? live1 : live0);
                        const float pv = ok ? ex2_fast(sc[nt][e] * p.scale_log2 - (hi ? lse1 : lse0)) : 0.f;
                        ds[nt][e] = pv * (hi ? gs1 : gs0) * (dp[nt][e] - (hi ? D1 : D0));
                    }
                }
                unsigned dsa[4];
                dsa[0] = pack_bf16(ds[0][0], ds[0][1]); dsa[1] = pack_bf16(ds[0][2], ds[0][3]);
                dsa[2] = pack_bf16(ds[1][0], ds[1][1]); dsa[3] = pack_bf16(ds[1][2], ds[1][3]);
                // dq += dS K (B = K rows [key][d], transposed loads)
#pragma unroll
                for (int dpi = 0; dpi < NT_D / 2; ++dpi) {
                    const int krow = kh * 16 + (mi & 1) * 8 + ri;
                    const int unit = dpi * 2 + (mi >> 1);
                    unsigned b0, b1, b2, b3;
                    ldsm_x4_t(b0, b1, b2, b3, ks_ + krow * ROWB + ((unit ^ (krow & 7)) * 16));
                    mma_bf16_16816(dqa[2 * dpi], dsa, b0, b1);
                    mma_bf16_16816(dqa[2 * dpi + 1], dsa, b2, b3);
                    if constexpr (HILO) {
                        ldsm_x4_t(b0, b1, b2, b3, ls_ + krow * ROWB + ((unit ^ (krow & 7)) * 16));
                        mma_bf16_16816(dqa[2 * dpi], dsa, b0, b1);
                        mma_bf16_16816(dqa[2 * dpi + 1], dsa, b2, b3);
                    }
                }
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
#pragma unroll
    for (int nt = 0; nt < NT_D; ++nt) {
        const int col = nt * 8 + 2 * qc;
        float2 a0 = make_float2(dqa[nt][0] * p.scale, dqa[nt][1] * p.scale);
        float2 a1 = make_float2(dqa[nt][2] * p.scale, dqa[nt][3] * p.scale);
        float2 *q0 = reinterpret_cast<float2 *>(p.dq + row0 * D + col);
        float2 *q1 = reinterpret_cast<float2 *>(p.dq + row1 * D + col);
        if (p.dq_accum) {
            if (v0) { const float2 o = *q0; a0.x += o.x; a0.y += o.y; }
            if (v1) { const float2 o = *q1; a1.x += o.x; a1.y += o.y; }
        }
        if (v0) *q0 = a0;
        if (v1) *q1 = a1;
    }
}

// dq of the NSA selected branch: one warp per (query, KV group) with at most
// 16 heads.  The chunks are 16 consecutive keys of one selected block, only
// those holding keys <= t (a block's chunk count is ceil(valid keys / 16));
// the chunk -> block mapping is a ballot over the lanes' prefix counts.  K
// and V chunks are gathered per warp by cp.async into a 3-stage ring; Q and
// dO A fragments stay in registers; S = Q K^T, dP = dO V^T, dS = gate P
// (dP - D), dq += dS K.
constexpr int DQB_WARPS = 8;
constexpr int DQB_STAGES = 3;

template <int D>
constexpr int attn_bwd_dq_blocks_smem() {
    return DQB_WARPS * DQB_STAGES * 2 * 16 * D * 2;
}

template <int D>
__global__ void __launch_bounds__(DQB_WARPS * 32) attn_bwd_dq_blocks_kernel(const BwdParams p) {
    grid_dependency_sync();
    constexpr int NK = 16;
    constexpr int ROWB = D * 2;
    constexpr int UNITS = ROWB / 16;
    constexpr int KS_D = D / 16;
    constexpr int NT_D = D / 8;
    constexpr int CH = NK * ROWB;
    constexpr int CP_ITERS = NK * UNITS / 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gr = lane >> 2, qc = lane & 3;
    const long long item = (long long)blockIdx.x * DQB_WARPS + warp;
    if (item >= (long long)p.B * p.Tq * p.Hkv) return;       // no block-wide barrier in this kernel
    const int g = (int)(item % p.Hkv);
    const long long bt = item / p.Hkv;
    const int t = (int)(bt % p.Tq), b = (int)(bt / p.Tq);
    const long long pos = p.q_pos0 + t;
    unsigned char *wsm = smem + warp * (DQB_STAGES * 2 * CH);

    const bool v0 = gr < p.G, v1 = gr + 8 < p.G;
    const long long row0 = (bt * p.Hq + (long long)g * p.G + gr), row1 = row0 + 8;
    float lse0 = v0 ? p.lse[row0 * p.lse_stride] : -INFINITY, lse1 = v1 ? p.lse[row1 * p.lse_stride] : -INFINITY;
    const bool live0 = v0 && lse0 != -INFINITY, live1 = v1 && lse1 != -INFINITY;
    lse0 *= kLog2e; lse1 *= kLog2e;
    const float D0 = v0 ? p.Dt[row0] : 0.f, D1 = v1 ? p.Dt[row1] : 0.f;
    const float gs0 = (p.gate && v0) ? p.gate[row0 * p.gate_stride] : 1.f;
    const float gs1 = (p.gate && v1) ? p.gate[row1 * p.gate_stride] : 1.f;
    unsigned qa[KS_D][4], da[KS_D][4];
#pragma unroll
    for (int ks = 0; ks < KS_D; ++ks) {
        const int c0 = ks * 16 + 2 * qc;
        const unsigned *q0 = reinterpret_cast<const unsigned *>(p.q + (v0 ? row0 : 0) * D + c0);
        const unsigned *q1 = reinterpret_cast<const unsigned *>(p.q + (v1 ? row1 : 0) * D + c0);
        const unsigned *d0 = reinterpret_cast<const unsigned *>(p.dout + (v0 ? row0 : 0) * D + c0);
        const unsigned *d1 = reinterpret_cast<const unsigned *>(p.dout + (v1 ? row1 : 0) * D + c0);
        qa[ks][0] = v0 ? __ldg(q0) : 0u; qa[ks][1] = v1 ? __ldg(q1) : 0u;
        qa[ks][2] = v0 ? __ldg(q0 + 4) : 0u; qa[ks][3] = v1 ? __ldg(q1 + 4) : 0u;
        da[ks][0] = v0 ? __ldg(d0) : 0u; da[ks][1] = v1 ? __ldg(d1) : 0u;
        da[ks][2] = v0 ? __ldg(d0 + 4) : 0u; da[ks][3] = v1 ? __ldg(d1 + 4) : 0u;
    }

    // lane m < K: block m of the list, its first key, last visible key and chunk count
    const int32_t *list = p.idx + (bt * p.idx_heads + (p.idx_heads == 1 ? 0 : g)) * p.K;
    long long jb = 0, je = -1;
    int nch = 0;
    if (lane < p.K) {
        const int blk = __ldg(list + lane);
        if (blk >= 0) {
            jb = (long long)blk * p.block;
            if (jb >= p.L) {
                raise_error(p.err, ERR_BAD_INDEX);
            } else {
                je = jb + p.block - 1;
                if (je > pos) je = pos;
                if (je > p.L - 1) je = p.L - 1;
                if (je >= jb) nch = (int)((je - jb + NK) / NK);
            }
        }
    }
    int pre = nch;                                    // inclusive prefix of the chunk counts
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += x;
    }
    const int n_chunks = __shfl_sync(0xffffffffu, pre, 31);
    const int pex = pre - nch;                        // exclusive prefix
    // chunk ci -> (first key, last key of its block)
    auto chunk_of = [&](int ci, long long &j0, long long &jl) {
        const unsigned m_mask = __ballot_sync(0xffffffffu, nch > 0 && pex <= ci);
        const int m = 31 - __clz(m_mask);           // last block starting at or before ci
        const int off = ci - __shfl_sync(0xffffffffu, pex, m);
        j0 = __shfl_sync(0xffffffffu, jb, m) + (long long)off * NK;
        jl = __shfl_sync(0xffffffffu, je, m);
    };
    const long long rstride = (long long)p.Hkv * D;
    const __nv_bfloat16 *kbase = p.k + ((long long)b * p.L * p.Hkv + g) * D;
    const __nv_bfloat16 *vbase = p.v + ((long long)b * p.L * p.Hkv + g) * D;
    auto issue = [&](int ci) {
        if (ci < n_chunks) {
            long long j0, jl;
            chunk_of(ci, j0, jl);
            unsigned char *st = wsm + (ci % DQB_STAGES) * 2 * CH;
#pragma unroll
            for (int it = 0; it < CP_ITERS; ++it) {
                const int lin = it * 32 + lane;
                const int r = lin / UNITS, u = lin % UNITS;
                const long long j = j0 + r;
                const bool ok = j <= jl;
                const long long off = ok ? j * rstride + u * 8 : 0;
                const int sw = (u ^ (r & 7)) * 16;
                cp_async16(st + r * ROWB + sw, kbase + off, ok ? 16 : 0);
                cp_async16(st + CH + r * ROWB + sw, vbase + off, ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };

    float dqa[NT_D][4];
#pragma unroll
    for (int i = 0; i < NT_D; ++i) dqa[i][0] = dqa[i][1] = dqa[i][2] = dqa[i][3] = 0.f;
    issue(0);
    issue(1);
    const int mi = lane >> 3, ri = lane & 7;
    for (int ci = 0; ci < n_chunks; ++ci) {
        issue(ci + 2);
        cp_async_wait<2>();
        __syncwarp();
        long long j0, jl;
        chunk_of(ci, j0, jl);
        const int nvalid = (int)min((long long)NK, jl - j0 + 1);
        const unsigned char *ks_ = wsm + (ci % DQB_STAGES) * 2 * CH;
        const unsigned char *vs_ = ks_ + CH;
        float sc[2][4], dp[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
        const int key = (mi >> 1) * 8 + ri;
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
            const int unit = ks * 2 + (mi & 1);
            unsigned b0, b1, b2, b3;
            ldsm_x4(b0, b1, b2, b3, ks_ + key * ROWB + ((unit ^ (key & 7)) * 16));
            mma_bf16_16816(sc[0], qa[ks], b0, b1);
            mma_bf16_16816(sc[1], qa[ks], b2, b3);
            ldsm_x4(b0, b1, b2, b3, vs_ + key * ROWB + ((unit ^ (key & 7)) * 16));
            mma_bf16_16816(dp[0], da[ks], b0, b1);
            mma_bf16_16816(dp[1], da[ks], b2, b3);
        }
        float ds[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int kk = nt * 8 + 2 * qc + (e & 1);
                const bool hi = e >> 1;
                const bool ok = kk < nvalid && (hi ? live1 : live0);
                const float pv = ok ? ex2_fast(sc[nt][e] * p.scale_log2 - (hi ? lse1 : lse0)) : 0.f;
                ds[nt][e] = pv * (hi ? gs1 : gs0) * (dp[nt][e] - (hi ? D1 : D0));
            }
        }
        unsigned dsa[4];
        dsa[0] = pack_bf16(ds[0][0], ds[0][1]); dsa[1] = pack_bf16(ds[0][2], ds[0][3]);
        dsa[2] = pack_bf16(ds[1][0], ds[1][1]); dsa[3] = pack_bf16(ds[1][2], ds[1][3]);
#pragma unroll
        for (int dpi = 0; dpi < NT_D / 2; ++dpi) {
            const int krow = (mi & 1) * 8 + ri;
            const int unit = dpi * 2 + (mi >> 1);
            unsigned b0, b1, b2, b3;
            ldsm_x4_t(b0, b1, b2, b3, ks_ + krow * ROWB + ((unit ^ (krow & 7)) * 16));
            mma_bf16_16816(dqa[2 * dpi], dsa, b0, b1);
            mma_bf16_16816(dqa[2 * dpi + 1], dsa, b2, b3);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
#pragma unroll
    for (int nt = 0; nt < NT_D; ++nt) {
        const int col = nt * 8 + 2 * qc;
        float2 a0 = make_float2(dqa[nt][0] * p.scale, dqa[nt][1] * p.scale);
        float2 a1 = make_float2(dqa[nt][2] * p.scale, dqa[nt][3] * p.scale);
        float2 *q0 = reinterpret_cast<float2 *>(p.dq + row0 * D + col);
        float2 *q1 = reinterpret_cast<float2 *>(p.dq + row1 * D + col);
        if (p.dq_accum) {
            if (v0) { const float2 o = *q0; a0.x += o.x; a0.y += o.y; }
            if (v1) { const float2 o = *q1; a1.x += o.x; a1.y += o.y; }
        }
        if (v0) *q0 = a0;
        if (v1) *q1 = a1;
    }
}

// Inverse of the block choice: per (b, g, block) the queries that chose it.
// 1. counts per list
__global__ void __launch_bounds__(256) bwd_sel_count_kernel(const int32_t *__restrict__ sel, long long n_entries,
                                                            int T, int Hkv, int K, int nb, int32_t *__restrict__ cnt) {
    grid_dependency_sync();
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n_entries) return;
    const int blk = sel[e];
    if (blk < 0 || blk >= nb) return;
    const long long bt_g = e / K;                  // (b, t, g)
    const int g = (int)(bt_g % Hkv);
    const long long b = bt_g / Hkv / T;
    atomicAdd(cnt + (b * Hkv + g) * nb + blk, 1);
}

// 2. one CTA: list starts (exclusive scan of the counts), fill cursors, and
//    the (list, split) work items of at most q_split queries each
__global__ void __launch_bounds__(1024) bwd_sel_scan_kernel(const int32_t *__restrict__ cnt, int n_lists,
                                                            int q_split, int32_t *__restrict__ qoff,
                                                            int32_t *__restrict__ cursor, int2 *__restrict__ items,
                                                            int32_t *__restrict__ n_items) {
    grid_dependency_sync();
    __shared__ int s_off[1024], s_it[1024];
    __shared__ int carry_off, carry_it;
    if (threadIdx.x == 0) { carry_off = 0; carry_it = 0; }
    __syncthreads();
    for (int base = 0; base < n_lists; base += 1024) {
        const int l = base + threadIdx.x;
        const int c = l < n_lists ? cnt[l] : 0;
        const int ni = (c + q_split - 1) / q_split;
        s_off[threadIdx.x] = c;
        s_it[threadIdx.x] = ni;
        __syncthreads();
        for (int o = 1; o < 1024; o <<= 1) {          // inclusive scans (Hillis-Steele)
            const int a = threadIdx.x >= o ? s_off[threadIdx.x - o] : 0;
            const int bb = threadIdx.x >= o ? s_it[threadIdx.x - o] : 0;
            __syncthreads();
            s_off[threadIdx.x] += a;
            s_it[threadIdx.x] += bb;
            __syncthreads();
        }
        const int off = carry_off + s_off[threadIdx.x] - c;
        const int it0 = carry_it + s_it[threadIdx.x] - ni;
        if (l < n_lists) {
            qoff[l] = off;
            cursor[l] = off;
            for (int s = 0; s < ni; ++s) items[it0 + s] = make_int2(l, s);
        }
        __syncthreads();
        if (threadIdx.x == 1023) { carry_off += s_off[1023]; carry_it += s_it[1023]; }
        __syncthreads();
    }
    if (threadIdx.x == 0) { qoff[n_lists] = carry_off; *n_items = carry_it; }
}

// 3. the queries into their lists (order inside a list is not fixed)
__global__ void __launch_bounds__(256) bwd_sel_fill_kernel(const int32_t *__restrict__ sel, long long n_entries,
                                                           int T, int Hkv, int K, int nb,
                                                           int32_t *__restrict__ cursor, int32_t *__restrict__ qlist) {
    grid_dependency_sync();
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n_entries) return;
    const int blk = sel[e];
    if (blk < 0 || blk >= nb) return;
    const long long bt_g = e / K;
    const int g = (int)(bt_g % Hkv);
    const long long bt = bt_g / Hkv;
    const int t = (int)(bt % T);
    const long long b = bt / T;
    const int pos = atomicAdd(cursor + (b * Hkv + g) * nb + blk, 1);
    qlist[pos] = t;
}

template <int D, int NW, bool HILO = false>
constexpr int attn_bwd_smem_bytes() {
    return NW * attn_bwd_warp_bytes<D, HILO>();
}

// NSA: per row, r_b = dO . O_b for the three branch outputs (fp32, [3, rows,
// D]).  r_b is the branch's D term before the gate factor and the gradient
// of the output with respect to gate b.  One warp per row.
template <int D>
__global__ void __launch_bounds__(256) nsa_bwd_prep_kernel(const __nv_bfloat16 *__restrict__ dout,
                                                           const float *__restrict__ o3, long long rows,
                                                           float *__restrict__ Dt, float *__restrict__ dgates) {
    grid_dependency_sync();
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(dout + row * D);
    float s[3] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int c = lane; c < D / 2; c += 32) {
        const float2 x = __bfloat1622float2(a[c]);
#pragma unroll
        for (int br = 0; br < 3; ++br) {
            const float2 y = reinterpret_cast<const float2 *>(o3 + (br * rows + row) * D)[c];
            s[br] += x.x * y.x + x.y * y.y;
        }
    }
#pragma unroll
    for (int br = 0; br < 3; ++br) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s[br] += __shfl_xor_sync(0xffffffffu, s[br], o);
    }
    if (lane < 3) {
        const float r = lane == 0 ? s[0] : (lane == 1 ? s[1] : s[2]);
        Dt[lane * rows + row] = r;
        dgates[row * 3 + lane] = r;
    }
}

// NSA: the compressed row i is the mean of rows i*stride .. i*stride+len-1,
// so raw row j receives dKc_i / len from every i that covers it (likewise
// V).  One thread per 4 columns of a (b, j, g) row; added to dk / dv.
__global__ void __launch_bounds__(256) nsa_pool_bwd_kernel(const float *__restrict__ dkc, const float *__restrict__ dvc,
                                                           float *__restrict__ dk, float *__restrict__ dv, int B, int T,
                                                           int Hkv, int d, int nc, int len, int stride) {
    grid_dependency_sync();
    const int d4 = d / 4;
    const long long total = (long long)B * T * Hkv * d4;
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= total) return;
    const int c4 = (int)(e % d4);
    long long r = e / d4;
    const int g = (int)(r % Hkv); r /= Hkv;
    const int j = (int)(r % T);
    const int b = (int)(r / T);
    int i_hi = j / stride;
    if (i_hi > nc - 1) i_hi = nc - 1;
    const int i_lo = j - len + 1 <= 0 ? 0 : (j - len + stride) / stride;
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
    for (int i = i_lo; i <= i_hi; ++i) {
        const long long o = (((long long)b * nc + i) * Hkv + g) * d4 + c4;
        const float4 x = reinterpret_cast<const float4 *>(dkc)[o];
        const float4 y = reinterpret_cast<const float4 *>(dvc)[o];
        sk.x += x.x; sk.y += x.y; sk.z += x.z; sk.w += x.w;
        sv.x += y.x; sv.y += y.y; sv.z += y.z; sv.w += y.w;
    }
    const float inv = 1.f / (float)len;
    float4 *pk = reinterpret_cast<float4 *>(dk) + e;
    float4 *pv = reinterpret_cast<float4 *>(dv) + e;
    float4 a = *pk, c = *pv;
    a.x += sk.x * inv; a.y += sk.y * inv; a.z += sk.z * inv; a.w += sk.w * inv;
    c.x += sv.x * inv; c.y += sv.y * inv; c.z += sv.z * inv; c.w += sv.w * inv;
    *pk = a;
    *pv = c;
}

}  // namespace sa
