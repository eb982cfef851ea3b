// nsa_misc.cuh -- log-sum-exp combine and the NSA helper kernels.
#pragma once

#include "sa_common.cuh"

namespace sa {

// --------------------------------------------------------------- combine --
// Star Attention page ("NVIDIA AI Research presenta Star Attention ...",
// body): per-piece softmax results merge by a distributed softmax,
//   lse = log sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) o_s.
// One warp per row (two rows per CTA, so that small calls spread over the
// SMs); each lane owns d/32 consecutive columns.
constexpr int COMBINE_ROWS = 2;
template <int D>
__global__ void __launch_bounds__(COMBINE_ROWS * 32) lse_combine_kernel(const float *__restrict__ part_o,
                                                         const float *__restrict__ part_lse,
                                                         int n_split, long long rows,
                                                         __nv_bfloat16 *__restrict__ out,
                                                         float *__restrict__ lse) {
    grid_dependency_sync();
    constexpr int PER = D / 32;
    const long long row = (long long)blockIdx.x * COMBINE_ROWS + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float den = 0.f, m = -INFINITY;
    constexpr int PRE = 8;                                    // pieces whose rows load with the LSEs
    if (n_split <= PRE) {
        // few pieces (decode): every piece's slice of the row is loaded
        // together with the LSEs, so the merge costs one memory latency
        float2 x[PRE][PER / 2];
        const float lsl = lane < n_split ? __ldcg(part_lse + lane * rows + row) : -INFINITY;
#pragma unroll
        for (int q = 0; q < PRE; ++q)
#pragma unroll
            for (int i = 0; i < PER / 2; ++i)
                x[q][i] = q < n_split ? __ldcg(reinterpret_cast<const float2 *>(part_o + ((long long)q * rows + row) * D +
                                                                                 lane * PER) + i)
                                      : make_float2(0.f, 0.f);
        m = warp_max(lsl);
        if (m != -INFINITY) {
            const float fl = lsl == -INFINITY ? 0.f : exp2f((lsl - m) * kLog2e);
            den = warp_sum(fl);
#pragma unroll
            for (int q = 0; q < PRE; ++q) {
                const float f = __shfl_sync(0xffffffffu, fl, q);   // 0 for q >= n_split
#pragma unroll
                for (int i = 0; i < PER / 2; ++i) {
                    acc[2 * i] += f != 0.f ? f * x[q][i].x : 0.f;
                    acc[2 * i + 1] += f != 0.f ? f * x[q][i].y : 0.f;
                }
            }
        }
    } else if (n_split <= 32) {
        // lane s holds piece s's LSE; the pieces' partial rows are then read
        // with independent (unrolled) loads
        const float lsl = lane < n_split ? part_lse[lane * rows + row] : -INFINITY;
        m = warp_max(lsl);
        if (m != -INFINITY) {
            const float fl = lsl == -INFINITY ? 0.f : exp2f((lsl - m) * kLog2e);
            den = warp_sum(fl);
            // every piece's partial row is read (the loads carry no branch and
            // go out together); an empty piece's row counts with weight 0
            // whatever it holds
#pragma unroll 16
            for (int s = 0; s < n_split; ++s) {
                const float f = __shfl_sync(0xffffffffu, fl, s);
                const float *src = part_o + ((long long)s * rows + row) * D + lane * PER;
#pragma unroll
                for (int i = 0; i < PER; i += 2) {
                    const float2 x = __ldcg(reinterpret_cast<const float2 *>(src + i));
                    acc[i] += f != 0.f ? f * x.x : 0.f;
                    acc[i + 1] += f != 0.f ? f * x.y : 0.f;
                }
            }
        }
    } else {
        for (int s = lane; s < n_split; s += 32) m = fmaxf(m, part_lse[s * rows + row]);
        m = warp_max(m);
        if (m != -INFINITY) {
            for (int s = 0; s < n_split; ++s) {
                const float ls = part_lse[s * rows + row];
                if (ls == -INFINITY) continue;
                const float f = exp2f((ls - m) * kLog2e);
                den += f;
                const float *src = part_o + ((long long)s * rows + row) * D + lane * PER;
#pragma unroll
                for (int i = 0; i < PER; i += 2) {
                    const float2 x = *reinterpret_cast<const float2 *>(src + i);
                    acc[i] += f * x.x;
                    acc[i + 1] += f * x.y;
                }
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    __nv_bfloat16 *dst = out + row * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2)
        *reinterpret_cast<unsigned *>(dst + i) = pack_bf16(acc[i] * inv, acc[i + 1] * inv);
    if (lse && lane == 0) lse[row] = den > 0.f ? m + log2f(den) * kLn2 : -INFINITY;
}

// ------------------------------------------------------------ compression --
// NSA page ("Native Sparse Attention ...", "Puntos Clave": coarse
// compression): Kc[i] = mean(k[i*stride .. i*stride+len-1]) per KV head.
// One thread per (b, i, g, column pair); fp32 sums.  The key means are
// stored as a bf16 pair kc + kc_lo (kc_lo = the rounding residual), so the
// compressed logits keep ~16 mantissa bits; value means are rounded once.
__global__ void nsa_compress_kernel(const __nv_bfloat16 *__restrict__ k,
                                    const __nv_bfloat16 *__restrict__ v, int B, int T, int Hkv,
                                    int d, int nc, int len, int stride,
                                    __nv_bfloat16 *__restrict__ kc, __nv_bfloat16 *__restrict__ kc_lo,
                                    __nv_bfloat16 *__restrict__ vc) {
    grid_dependency_sync();
    const long long total = (long long)B * nc * Hkv * (d / 2);
    const long long i2 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i2 >= total) return;
    const int c2 = (int)(i2 % (d / 2));
    long long r = i2 / (d / 2);
    const int g = (int)(r % Hkv); r /= Hkv;
    const int i = (int)(r % nc);
    const int b = (int)(r / nc);
    float sk0 = 0.f, sk1 = 0.f, sv0 = 0.f, sv1 = 0.f;
    for (int u = 0; u < len; ++u) {
        const long long off = (((long long)b * T + (long long)i * stride + u) * Hkv + g) * d + 2 * c2;
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(k + off);
        const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162 *>(v + off);
        sk0 += __low2float(a); sk1 += __high2float(a);
        sv0 += __low2float(c); sv1 += __high2float(c);
    }
    const float inv = 1.f / (float)len;
    const long long o = (((long long)b * nc + i) * Hkv + g) * d + 2 * c2;
    const float m0 = sk0 * inv, m1 = sk1 * inv;
    const __nv_bfloat162 hi = __floats2bfloat162_rn(m0, m1);
    *reinterpret_cast<__nv_bfloat162 *>(kc + o) = hi;
    *reinterpret_cast<unsigned *>(kc_lo + o) = pack_bf16(m0 - __low2float(hi), m1 - __high2float(hi));
    *reinterpret_cast<unsigned *>(vc + o) = pack_bf16(sv0 * inv, sv1 * inv);
}

// ----------------------------------------------- importance + block top-k --
// NSA page ("Puntos Clave": fine-grained blockwise selection; "Analisis
// Profundo": group-centric loading, shared KV fetch).  One warp per (b, t, g):
// the 16 heads of the KV group are the 16 rows of an m16 tile over the
// compressed keys.  p_cmp = exp(z - lse_cmp) is summed over the group's heads
// and over the compressed tokens that start inside each selection block; the
// sel_topk most important candidate blocks (b*sel_block <= t; ties -> lower b)
// are written in ascending order.
struct NsaSelectParams {
    const __nv_bfloat16 *q;    // [B,T,Hq,D]
    const __nv_bfloat16 *kc;   // [B,nc,Hkv,D]
    const __nv_bfloat16 *klo;  // [B,nc,Hkv,D] low half of the compressed keys
    const float *lse_cmp;      // [B,T,Hq] natural log
    int B, T, Hq, Hkv, G, nc;
    int cmp_len, cmp_stride, sel_block, sel_topk, n_blocks;
    float scale_log2;
    int32_t *sel_idx;          // [B,T,Hkv,sel_topk]
    float *imp_out;            // optional [B,T,Hkv,n_blocks] (tests)
};

// CTA = SEL_TW consecutive queries of one KV group (warp w: query t0 + w,
// rows = the group's heads); compressed-key chunks (hi and lo halves) are
// staged once per CTA and read by every warp.
constexpr int NSA_TW = 8;

template <int D>
constexpr int nsa_select_smem(int n_blocks) {
    return 3 * 2 * 32 * D * 2 + NSA_TW * (32 * 4 + ((n_blocks * 4 + 15) / 16) * 16);
}

template <int D>
__global__ void __launch_bounds__(NSA_TW * 32) nsa_select_kernel(const NsaSelectParams p) {
    grid_dependency_sync();
    constexpr int NK = 32, ROWB = D * 2, UNITS = ROWB / 16, CH = NK * ROWB;
    constexpr int KS_D = D / 16, STAGES = 3;
    constexpr int SB = 2 * CH;                 // one stage: K hi | K lo
    constexpr int NTHR = NSA_TW * 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int imp_stride = ((p.n_blocks * 4 + 15) / 16) * 16;        // bytes per warp
    float *colsum = reinterpret_cast<float *>(smem + STAGES * SB) + warp * 32;
    float *imp = reinterpret_cast<float *>(smem + STAGES * SB + NSA_TW * 32 * 4 + warp * imp_stride);

    const int nqb = (p.T + NSA_TW - 1) / NSA_TW;
    long long rem = blockIdx.x;
    const int qb = (int)(rem % nqb); rem /= nqb;
    const int g = (int)(rem % p.Hkv);
    const int b = (int)(rem / p.Hkv);
    const int t_first = qb * NSA_TW;
    const int t_last = min(t_first + NSA_TW - 1, p.T - 1);
    const int t = t_first + warp;
    const bool q_ok = t <= t_last;
    auto n_vis_of = [&](int tt) {
        return tt >= p.cmp_len - 1 ? min(p.nc, (tt - p.cmp_len + 1) / p.cmp_stride + 1) : 0;
    };
    const int n_vis_cta = n_vis_of(t_last);
    const int n_vis = q_ok ? n_vis_of(t) : 0;
    const int n_chunks = (n_vis_cta + NK - 1) / NK;

    const int gr = lane >> 2, qc = lane & 3;
    const bool v0 = q_ok && gr < p.G, v1 = q_ok && gr + 8 < p.G;
    const int h0 = g * p.G + gr, h1 = h0 + 8;
    const int tq = q_ok ? t : 0;
    unsigned qf[KS_D][4];
    {
        const unsigned *q0 = reinterpret_cast<const unsigned *>(p.q + ((long long)(b * p.T + tq) * p.Hq + h0) * D);
        const unsigned *q1 = reinterpret_cast<const unsigned *>(p.q + ((long long)(b * p.T + tq) * p.Hq + h1) * D);
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
            qf[ks][0] = v0 ? __ldg(q0 + ks * 8 + qc) : 0u;
            qf[ks][1] = v1 ? __ldg(q1 + ks * 8 + qc) : 0u;
            qf[ks][2] = v0 ? __ldg(q0 + ks * 8 + qc + 4) : 0u;
            qf[ks][3] = v1 ? __ldg(q1 + ks * 8 + qc + 4) : 0u;
        }
    }
    const float ls0 = v0 ? p.lse_cmp[(long long)(b * p.T + tq) * p.Hq + h0] * kLog2e : INFINITY;
    const float ls1 = v1 ? p.lse_cmp[(long long)(b * p.T + tq) * p.Hq + h1] * kLog2e : INFINITY;

    const int nb_t = q_ok ? t / p.sel_block + 1 : 0;      // candidate blocks of this query
    for (int i = lane; i < nb_t; i += 32) imp[i] = 0.f;
    const __nv_bfloat16 *kb = p.kc + ((long long)b * p.nc * p.Hkv + g) * D;
    const __nv_bfloat16 *kl = p.klo + ((long long)b * p.nc * p.Hkv + g) * D;
    const long long rstride = (long long)p.Hkv * D;

    auto issue = [&](int ci) {
        if (ci < n_chunks) {
            unsigned char *ks_ = smem + (ci % STAGES) * SB;
            for (int lin = tid; lin < NK * UNITS; lin += NTHR) {
                const int rr = lin / UNITS, u = lin % UNITS;
                const int i = ci * NK + rr;
                const bool ok = i < n_vis_cta;
                const long long off = ok ? (long long)i * rstride + u * 8 : 0;
                const int sw = (u ^ (rr & 7)) * 16;
                cp_async16(ks_ + rr * ROWB + sw, kb + off, ok ? 16 : 0);
                cp_async16(ks_ + CH + rr * ROWB + sw, kl + off, ok ? 16 : 0);
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int ci = 0; ci < STAGES - 1; ++ci) issue(ci);

    for (int ci = 0; ci < n_chunks; ++ci) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        issue(ci + STAGES - 1);
        if (ci * NK >= n_vis) continue;                     // warp-uniform: nothing visible
        const unsigned char *ks_ = smem + (ci % STAGES) * SB;
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
                ldsm_x4(b0, b1, b2, b3, ks_ + CH + key * ROWB + ((unit ^ (key & 7)) * 16));
                mma_bf16_16816(acc[2 * np], qf[ks], b0, b1);
                mma_bf16_16816(acc[2 * np + 1], qf[ks], b2, b3);
            }
        }
        // probabilities, summed over the group's heads (rows) per column
#pragma unroll
        for (int nt = 0; nt < NK / 8; ++nt) {
            float cs[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = ci * NK + nt * 8 + 2 * qc + e;
                const bool ok = i < n_vis;
                const float p0 = (ok && v0) ? exp2f((sc[nt][e] + sc2[nt][e]) * p.scale_log2 - ls0) : 0.f;
                const float p1 = (ok && v1) ? exp2f((sc[nt][2 + e] + sc2[nt][2 + e]) * p.scale_log2 - ls1) : 0.f;
                float x = p0 + p1;
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                x += __shfl_xor_sync(0xffffffffu, x, 8);
                x += __shfl_xor_sync(0xffffffffu, x, 16);
                cs[e] = x;
            }
            if (gr == 0) {
                colsum[nt * 8 + 2 * qc] = cs[0];
                colsum[nt * 8 + 2 * qc + 1] = cs[1];
            }
        }
        __syncwarp();
        // one writer per selection block touched by this chunk, fixed order:
        // block blk holds the compressed tokens [blk*cpb, (blk+1)*cpb)
        {
            const int cpb = p.sel_block / p.cmp_stride;
            const int i_first = ci * NK;
            const int i_last = min(ci * NK + NK, n_vis) - 1;
            const int blk_first = i_first / cpb, blk_last = i_last / cpb;
            for (int blk = blk_first + lane; blk <= blk_last; blk += 32) {
                const int c_lo = max(blk * cpb, i_first) - i_first;
                const int c_hi = min((blk + 1) * cpb - 1, i_last) - i_first;
                float acc = 0.f;
                for (int c = c_lo; c <= c_hi; ++c) acc += colsum[c];
                imp[blk] += acc;
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    __syncwarp();
    if (!q_ok) return;

    const long long orow = ((long long)(b * p.T + t) * p.Hkv + g);
    if (p.imp_out) {
        for (int i = lane; i < p.n_blocks; i += 32)
            p.imp_out[orow * p.n_blocks + i] = i < nb_t ? imp[i] : 0.f;
    }
    // top-sel_topk by repeated warp arg-max; taken entries are set to -1
    const int k = min(p.sel_topk, nb_t);
    int mine = -1;
    for (int r = 0; r < k; ++r) {
        float bv = -1.f;
        int bi = 0x7fffffff;
        for (int i = lane; i < nb_t; i += 32) {
            const float x = imp[i];
            if (x > bv) { bv = x; bi = i; }   // lanes scan ascending i: ties keep the lower i
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (lane == r) mine = bi < nb_t ? bi : -1;
        if (lane == 0 && bi < nb_t) imp[bi] = -1.f;
        __syncwarp();
    }
    // ascending order: rank of each chosen block among the chosen ones
    int rank = 0;
    for (int r = 0; r < k; ++r) {
        const int other = __shfl_sync(0xffffffffu, mine, r);
        rank += (lane < k && other < mine) ? 1 : 0;
    }
    int32_t *dst = p.sel_idx + orow * p.sel_topk;
    if (lane < k) dst[rank] = mine;
    for (int i = k + lane; i < p.sel_topk; i += 32) dst[i] = -1;
}

// --------------------------------------------------------------- gated sum --
// out = g_c * o_cmp + g_s * o_slc + g_w * o_win (gates already sigmoid).
__global__ void nsa_gate_kernel(const float *__restrict__ o3, long long branch_stride,
                                const float *__restrict__ gates, long long rows, int d,
                                __nv_bfloat16 *__restrict__ out) {
    grid_dependency_sync();
    const long long i2 = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // column pair
    if (i2 >= rows * (d / 2)) return;
    const long long row = i2 / (d / 2);
    const float gc = gates[row * 3], gs = gates[row * 3 + 1], gw = gates[row * 3 + 2];
    const float2 a = reinterpret_cast<const float2 *>(o3)[i2];
    const float2 bb = reinterpret_cast<const float2 *>(o3 + branch_stride)[i2];
    const float2 c = reinterpret_cast<const float2 *>(o3 + 2 * branch_stride)[i2];
    reinterpret_cast<unsigned *>(out)[i2] =
        pack_bf16(gc * a.x + gs * bb.x + gw * c.x, gc * a.y + gs * bb.y + gw * c.y);
}

__global__ void nsa_lse_pack_kernel(const float *__restrict__ l3, long long rows,
                                    float *__restrict__ lse_branches) {
    grid_dependency_sync();
    const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    lse_branches[r * 3 + 0] = l3[r];
    lse_branches[r * 3 + 1] = l3[rows + r];
    lse_branches[r * 3 + 2] = l3[2 * rows + r];
}

}  // namespace sa
