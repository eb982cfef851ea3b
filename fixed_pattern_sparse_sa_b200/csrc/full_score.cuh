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
#pragma once

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
