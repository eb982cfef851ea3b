// attn_tile.cuh -- attention over a key range shared by consecutive queries
// (NSA compressed and sliding-window branches).
//
// NSA page ("Native Sparse Attention ...", "Puntos Clave": coarse compression
// and sliding window; "Analisis Profundo": group-centric data loading, shared
// KV fetch).  A CTA of TW warps handles TW consecutive queries of one KV group;
// warp w owns query t0 + w and its rows are the group's query heads (the m16
// tile).  Keys of the union range the CTA needs are staged once per CTA in a
// multi-stage cp.async ring of 32-key chunks and read by every warp, each
// applying its own causal/visibility mask.  Scores and P.V use mma.sync
// m16n8k16 (bf16 -> fp32) with an online softmax, as in attn_gather.cuh.
#pragma once

#include "sa_common.cuh"

namespace sa {

enum TileSource : int {
    TS_CMP = 0,      // compressed tokens: key i visible iff i*stride + len - 1 <= t
    TS_WINDOW = 1,   // raw keys t - window < j <= t
};

struct TileParams {
    const __nv_bfloat16 *q;    // [B, T, Hq, D]
    const __nv_bfloat16 *k;    // [B, Lk, Hkv, D]
    const __nv_bfloat16 *klo;  // [B, Lk, Hkv, D] (TS_CMP: low half of the keys)
    const __nv_bfloat16 *v;    // [B, Lk, Hkv, D]
    int B, T, Lk, Hq, Hkv, G;
    int window;                // TS_WINDOW
    int cmp_len, cmp_stride;   // TS_CMP
    float scale_log2;
    float *out_f32;            // [B, T, Hq, D]
    float *lse;                // [B, T, Hq]
};

template <int SRC>
__device__ __forceinline__ long long tile_key_end(const TileParams &p, long long t) {
    // one past the last key visible to query t
    if constexpr (SRC == TS_CMP) {
        const long long nv = t >= p.cmp_len - 1 ? (t - p.cmp_len + 1) / p.cmp_stride + 1 : 0;
        return nv < p.Lk ? nv : p.Lk;
    } else {
        return t + 1;
    }
}
template <int SRC>
__device__ __forceinline__ long long tile_key_begin(const TileParams &p, long long t) {
    if constexpr (SRC == TS_CMP) {
        return 0;
    } else {
        const long long lo = t - p.window + 1;
        return lo > 0 ? lo : 0;
    }
}

template <int D, int STAGES, int SRC, int TW>
__global__ void __launch_bounds__(TW * 32) tile_attn_kernel(const TileParams p) {
    grid_dependency_sync();
    constexpr bool KLO = SRC == TS_CMP;
    constexpr int NK = 32;
    constexpr int ROWB = D * 2;
    constexpr int UNITS = ROWB / 16;
    constexpr int CH = NK * ROWB;
    constexpr int SB = (KLO ? 3 : 2) * CH;          // one stage: K | V | (K lo)
    constexpr int KS_D = D / 16;
    constexpr int NT_D = D / 8;
    constexpr int NTHR = TW * 32;

    extern __shared__ __align__(1024) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;

    // CTA -> (b, g, query block)
    const int nqb = (p.T + TW - 1) / TW;
    long long rem = blockIdx.x;
    const int qb = (int)(rem % nqb); rem /= nqb;
    const int g = (int)(rem % p.Hkv);
    const int b = (int)(rem / p.Hkv);
    const int t_first = qb * TW;
    const int t_last = min(t_first + TW - 1, p.T - 1);
    const int t = t_first + warp;                    // this warp's query
    const bool q_ok = t <= t_last;

    const long long k_lo = tile_key_begin<SRC>(p, t_first);
    const long long k_hi = tile_key_end<SRC>(p, t_last);
    const int n_chunks = k_hi > k_lo ? (int)((k_hi - k_lo + NK - 1) / NK) : 0;
    const long long my_lo = q_ok ? tile_key_begin<SRC>(p, t) : 0;
    const long long my_hi = q_ok ? tile_key_end<SRC>(p, t) : 0;

    const int gr = lane >> 2, qc = lane & 3;
    const bool v0 = q_ok && gr < p.G, v1 = q_ok && gr + 8 < p.G;
    const int h0 = g * p.G + gr, h1 = h0 + 8;
    unsigned qf[KS_D][4];
    {
        const unsigned *q0 = reinterpret_cast<const unsigned *>(p.q + ((long long)(b * p.T + (q_ok ? t : 0)) * p.Hq + h0) * D);
        const unsigned *q1 = reinterpret_cast<const unsigned *>(p.q + ((long long)(b * p.T + (q_ok ? t : 0)) * p.Hq + h1) * D);
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
            qf[ks][0] = v0 ? __ldg(q0 + ks * 8 + qc) : 0u;
            qf[ks][1] = v1 ? __ldg(q1 + ks * 8 + qc) : 0u;
            qf[ks][2] = v0 ? __ldg(q0 + ks * 8 + qc + 4) : 0u;
            qf[ks][3] = v1 ? __ldg(q1 + ks * 8 + qc + 4) : 0u;
        }
    }
    const long long rstride = (long long)p.Hkv * D;
    const __nv_bfloat16 *kb = p.k + ((long long)b * p.Lk * p.Hkv + g) * D;
    const __nv_bfloat16 *vb = p.v + ((long long)b * p.Lk * p.Hkv + g) * D;
    const __nv_bfloat16 *lb = KLO ? p.klo + ((long long)b * p.Lk * p.Hkv + g) * D : nullptr;

    auto issue = [&](int ci) {
        if (ci < n_chunks) {
            unsigned char *ks_ = smem + (ci % STAGES) * SB;
            unsigned char *vs_ = ks_ + CH;
            const long long c0 = k_lo + (long long)ci * NK;
            for (int lin = tid; lin < NK * UNITS; lin += NTHR) {
                const int rr = lin / UNITS, u = lin % UNITS;
                const long long j = c0 + rr;
                const bool ok = j < k_hi;
                const long long off = ok ? j * rstride + u * 8 : 0;
                const int sw = (u ^ (rr & 7)) * 16;
                cp_async16(ks_ + rr * ROWB + sw, kb + off, ok ? 16 : 0);
                cp_async16(vs_ + rr * ROWB + sw, vb + off, ok ? 16 : 0);
                if constexpr (KLO) cp_async16(vs_ + CH + rr * ROWB + sw, lb + off, ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };

    float o[NT_D][4];
#pragma unroll
    for (int i = 0; i < NT_D; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

#pragma unroll
    for (int ci = 0; ci < STAGES - 1; ++ci) issue(ci);
    for (int ci = 0; ci < n_chunks; ++ci) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();                          // chunk ci landed; chunk ci-1 fully consumed
        issue(ci + STAGES - 1);
        const long long c0 = k_lo + (long long)ci * NK;
        // keys of this chunk visible to this warp's query: [max(c0,my_lo), min(c0+NK,my_hi))
        if (c0 + NK <= my_lo || c0 >= my_hi) continue;        // warp-uniform skip
        const unsigned char *ks_ = smem + (ci % STAGES) * SB;
        const unsigned char *vs_ = ks_ + CH;
        float sc[NK / 8][4], sc2[NK / 8][4];
#pragma unroll
        for (int i = 0; i < NK / 8; ++i)
            sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = sc2[i][0] = sc2[i][1] = sc2[i][2] = sc2[i][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
            float (&acc)[NK / 8][4] = (ks & 1) ? sc2 : sc;
#pragma unroll
            for (int np = 0; np < NK / 16; ++np) {
                const int mi = lane >> 3, ri = lane & 7;
                const int key = np * 16 + (mi >> 1) * 8 + ri;
                const int unit = ks * 2 + (mi & 1);
                unsigned b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, ks_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                mma_bf16_16816(acc[2 * np], qf[ks], b0, b1);
                mma_bf16_16816(acc[2 * np + 1], qf[ks], b2, b3);
                if constexpr (KLO) {
                    ldsm_x4(b0, b1, b2, b3, vs_ + CH + key * ROWB + ((unit ^ (key & 7)) * 16));
                    mma_bf16_16816(acc[2 * np], qf[ks], b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], qf[ks], b2, b3);
                }
            }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NK / 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const long long j = c0 + nt * 8 + 2 * qc + (e & 1);
                const bool vis = j >= my_lo && j < my_hi;
                const float x = vis ? (sc[nt][e] + sc2[nt][e]) * p.scale_log2 : -INFINITY;
                sc[nt][e] = x;
            }
            mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
            mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
        const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = exp2f(m0 - mu0), al1 = exp2f(m1 - mu1);
        const bool grew = __any_sync(0xffffffffu, mn0 > m0 || mn1 > m1);
        m0 = mn0; m1 = mn1;
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NK / 8; ++nt) {
            sc[nt][0] = exp2f(sc[nt][0] - mu0);
            sc[nt][1] = exp2f(sc[nt][1] - mu0);
            sc[nt][2] = exp2f(sc[nt][2] - mu1);
            sc[nt][3] = exp2f(sc[nt][3] - mu1);
            rs0 += sc[nt][0] + sc[nt][1];
            rs1 += sc[nt][2] + sc[nt][3];
        }
        l0 = l0 * al0 + rs0;
        l1 = l1 * al1 + rs1;
        if (grew) {
#pragma unroll
            for (int i = 0; i < NT_D; ++i) {
                o[i][0] *= al0; o[i][1] *= al0;
                o[i][2] *= al1; o[i][3] *= al1;
            }
        }
#pragma unroll
        for (int kp = 0; kp < NK / 16; ++kp) {
            unsigned pa[4];
            pa[0] = pack_bf16(sc[2 * kp][0], sc[2 * kp][1]);
            pa[1] = pack_bf16(sc[2 * kp][2], sc[2 * kp][3]);
            pa[2] = pack_bf16(sc[2 * kp + 1][0], sc[2 * kp + 1][1]);
            pa[3] = pack_bf16(sc[2 * kp + 1][2], sc[2 * kp + 1][3]);
#pragma unroll
            for (int dp = 0; dp < NT_D / 2; ++dp) {
                const int mi = lane >> 3, ri = lane & 7;
                const int key = kp * 16 + (mi & 1) * 8 + ri;
                const int unit = dp * 2 + (mi >> 1);
                unsigned b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, vs_ + key * ROWB + ((unit ^ (key & 7)) * 16));
                mma_bf16_16816(o[2 * dp], pa, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
            }
        }
    }
    cp_async_wait<0>();

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (!q_ok) return;
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
    const long long orow0 = (long long)(b * p.T + t) * p.Hq + h0;
    const long long orow1 = (long long)(b * p.T + t) * p.Hq + h1;
#pragma unroll
    for (int nt = 0; nt < NT_D; ++nt) {
        const int dcol = nt * 8 + 2 * qc;
        if (v0) *reinterpret_cast<float2 *>(p.out_f32 + orow0 * D + dcol) = make_float2(o[nt][0] * inv0, o[nt][1] * inv0);
        if (v1) *reinterpret_cast<float2 *>(p.out_f32 + orow1 * D + dcol) = make_float2(o[nt][2] * inv1, o[nt][3] * inv1);
    }
    if (p.lse && qc == 0) {
        if (v0) p.lse[orow0] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
        if (v1) p.lse[orow1] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
    }
}

template <int D, int STAGES, int SRC>
constexpr int tile_smem_bytes() {
    return STAGES * ((SRC == TS_CMP ? 3 : 2) * 32 * D * 2);
}

}  // namespace sa
