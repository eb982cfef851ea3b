// attn_gather.cuh -- gathered-KV sparse attention, one warp per
// (query, KV head, 16-head chunk, split) work item, or (CTA-merged form, for
// launches too small to fill the GPU) one CTA of 8 warps per item whose warps
// split the item's keys and merge in shared memory.
//
// Operation (every page reduces to it once a query's index set is known):
//   z_j = scale * q.k_j + bias_j over j in S,  o = softmax(z) V,  lse = log sum exp z.
// The 16 query heads that share one KV head form the 16 rows of an m16
// tensor-core tile, so every gathered K/V row feeds 16 heads ("shared KV
// fetch" of the NSA page, section "Analisis Profundo").  Keys are streamed in
// chunks of 16 rows through a per-warp multi-stage cp.async pipeline into
// XOR-swizzled shared memory, scored with mma.sync m16n8k16 (bf16 -> fp32),
// folded into an online softmax and multiplied into V with a second mma.
#pragma once

#include <climits>

#include <cuda.h>

#include "sa_common.cuh"
#include "tc_common.cuh"

namespace sa {

enum KeySource : int {
    KS_IDX = 0,      // explicit index list idx[b, t, ih, e]
    KS_PATTERN = 1,  // fixed window + dilated powers of two
    KS_BLOCKS = 2,   // NSA selected blocks: idx holds block ids
    KS_RANGE = 3,    // recent window: j = p - window + 1 + e
    KS_PROWS = 4,    // fixed graph, rows = 16/G consecutive queries x G heads: the
                     // union of their sets (window band + one 16/G-key segment per
                     // dilated distance), masked per (row, key)
};

struct GatherParams {
    const __nv_bfloat16 *q;   // [B, Tq, Hq, D]
    const __nv_bfloat16 *k;   // [B, Lk, Hkv, D]
    const __nv_bfloat16 *v;   // [B, Lk, Hkv, D]
    const __nv_bfloat16 *klo; // optional low half of k (k ~ k + klo), same layout
    int B, Tq, Lk, Hq, Hkv, G;
    long long q_pos0;
    const int32_t *idx;       // KS_IDX: [B,Tq,idx_heads,K]; KS_BLOCKS: [B,Tq,Hkv,K] block ids
    int idx_heads, K;
    int window, dilated;      // KS_PATTERN / KS_RANGE
    int block;                // KS_BLOCKS block length
    int block_shift;          // log2(block) when block is a power of two, else -1
    int cmp_len;              // unused by the gather kernel
    int entries;              // virtual list length per item
    int per_split;            // entries handled by one split piece
    int n_split, n_hchunk;
    int q_units;              // query units of the item grid (Tq, or ceil(Tq/(16/G)) for KS_PROWS)
    const float *cq, *ck, *beta;   // optional coordinate bias
    float scale_log2;         // scale * log2(e)
    __nv_bfloat16 *out;       // [B,Tq,Hq,D] (n_split == 1)
    float *lse;               // [B,Tq,Hq]   (nullable)
    float *part_o;            // [n_split,B,Tq,Hq,D] (n_split > 1)
    float *part_lse;          // [n_split,B,Tq,Hq]
    int *merge_cnt;           // split-KV with out: per (b, t, g, head chunk) arrival tickets (zeroed);
                              // the last piece of a group merges the pieces into out / lse
    float *out_f32;           // optional fp32 output [B,Tq,Hq,D] instead of bf16
    unsigned *err;
};

// Keys are produced in two stages so that the list loads can be issued well
// before they are needed.  key_raw: the raw list value of virtual entry e (a
// global load for explicit lists; computed sources give the final key, -1 when
// masked).  key_finish: validation and translation to a key position, or -1
// for an empty/masked entry; an explicit index that is out of range or in the
// future raises the error word and is skipped.
constexpr int KEY_NONE = INT_MIN;

template <int SRC>
__device__ __forceinline__ int key_raw(const GatherParams &p, int b, int t, int g, long long pos,
                                       int e, int e_end) {
    if (e >= e_end) return KEY_NONE;
    if constexpr (SRC == KS_IDX) {
        const int32_t *list =
            p.idx + ((long long)(b * p.Tq + t) * p.idx_heads + (p.idx_heads == 1 ? 0 : g)) * p.K;
        return __ldg(list + e);
    } else if constexpr (SRC == KS_BLOCKS) {
        const int32_t *list = p.idx + ((long long)(b * p.Tq + t) * p.Hkv + g) * p.K;
        return __ldg(list + (p.block_shift >= 0 ? e >> p.block_shift : e / p.block));
    } else if constexpr (SRC == KS_PATTERN) {
        long long nw = pos + 1 < p.window ? pos + 1 : p.window;
        if (e < nw) return (int)(pos - e);
        if (!p.dilated) return -1;
        // dilated distances 2^i with 2^i >= window (the rest are in the window)
        int i0 = 0;
        while ((1LL << i0) < p.window) ++i0;
        int m = e - (int)nw;
        if (i0 + m >= 62) return -1;
        long long o = 1LL << (i0 + m);
        if (o >= pos) return -1;
        return (int)(pos - o);
    } else if constexpr (SRC == KS_RANGE) {
        long long j = pos - p.window + 1 + e;
        return j < 0 ? -1 : (int)j;
    } else {  // KS_PROWS: `pos` is the first query's position, see key_prows
        return -1;
    }
}

// KS_PROWS: entry e of the union for queries at positions [pa, pb]; returns
// the key (or -1) and, in seg, 0 for the window band or the dilated distance.
// i0 = the first dilated exponent (2^i0 >= window), lq = log2(nqw): both
// per-kernel constants (nqw = 16 / G is a power of two).
__device__ __forceinline__ int key_prows(const GatherParams &p, long long pa, long long pb, int lq, int i0, int e,
                                         int e_end, int &seg) {
    seg = 0;
    if (e >= e_end) return -1;
    const long long lo = pa - p.window + 1 > 0 ? pa - p.window + 1 : 0;
    const int nb = (int)(pb - lo + 1);
    if (e < nb) return (int)(lo + e);
    if (!p.dilated) return -1;
    const int e2 = e - nb;
    const int m = e2 >> lq, r = e2 & ((1 << lq) - 1);
    if (i0 + m >= 62) return -1;
    const long long o = 1LL << (i0 + m);
    if (o >= pb) return -1;
    const long long j = pa - o + r;
    if (j < 0 || pa + r > pb) return -1;
    seg = (int)o;
    return (int)j;
}

// KS_PROWS: the rows (bit r = row r; row r is query r / G of the item, G
// heads per query, nq_valid queries in the item) that see key j of segment
// seg, for queries at positions pa + qi: the window band reaches
// pa + qi - window < j <= pa + qi, a dilated distance o reaches only the
// query at j + o, and only when o < its position.
__device__ __forceinline__ unsigned prows_rowmask(int j, int seg, long long pa, int nq_valid, int window, int G) {
    if (j < 0) return 0u;
    const long long rel = (long long)j - pa;                 // key position relative to the first query
    long long qlo, qhi;
    if (seg == 0) {
        qlo = rel > 0 ? rel : 0;
        qhi = rel + window - 1;
    } else {
        qlo = qhi = rel + seg;
        if ((long long)seg >= pa + qlo) return 0u;
    }
    if (qhi > nq_valid - 1) qhi = nq_valid - 1;
    if (qhi < qlo) return 0u;
    const int rlo = (int)qlo * G, rhi = ((int)qhi + 1) * G;   // rows [rlo, rhi), rhi <= 16
    return ((rhi >= 32 ? 0xffffffffu : (1u << rhi)) - 1u) & ~((1u << rlo) - 1u);
}

template <int SRC>
__device__ __forceinline__ int key_finish(const GatherParams &p, long long pos, int raw, int e) {
    if (raw == KEY_NONE) return -1;
    if constexpr (SRC == KS_IDX) {
        if (raw == -1) return -1;
        if (raw < 0 || raw >= p.Lk || (long long)raw > pos) {
            raise_error(p.err, ERR_BAD_INDEX);
            return -1;
        }
        return raw;
    } else if constexpr (SRC == KS_BLOCKS) {
        const int blk = raw;
        if (blk == -1) return -1;
        if (blk < 0 || (long long)blk * p.block >= p.Lk) {
            raise_error(p.err, ERR_BAD_BLOCK);
            return -1;
        }
        const long long j = (long long)blk * p.block + (p.block_shift >= 0 ? e & (p.block - 1) : e % p.block);
        if (j > pos || j >= p.Lk) return -1;   // causal mask inside the block
        return (int)j;
    } else {
        return raw;
    }
}

// Log-sum-exp merge of the output rows of one item group (Star Attention
// page, body: distributed softmax) by the warp whose piece arrived last: lane
// l takes head row l / 2 of the group, columns (l % 2) * D/2 .. + D/2.  The
// pieces were written by other CTAs of the same launch, so they are read
// through L2; the LSEs of every piece first (up to 32, independent loads),
// then the partial rows with several pieces' loads in flight.
template <int D>
__device__ __forceinline__ void merge_pieces_half(const float *part_o, const float *part_lse, int n_split,
                                                  long long rows, long long row, int c0, __nv_bfloat16 *out,
                                                  float *lse) {
    constexpr int MAXS = 32;
    float ls[MAXS];
    float m = -INFINITY;
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
        ls[s] = s < n_split ? __ldcg(part_lse + s * rows + row) : -INFINITY;
        m = fmaxf(m, ls[s]);
    }
    float acc[D / 2];
#pragma unroll
    for (int i = 0; i < D / 2; ++i) acc[i] = 0.f;
    float den = 0.f;
    if (m != -INFINITY) {
#pragma unroll
        for (int s = 0; s < MAXS; ++s) {
            if (s >= n_split || ls[s] == -INFINITY) continue;
            const float f = exp2f((ls[s] - m) * kLog2e);
            den += f;
            const float4 *src = reinterpret_cast<const float4 *>(part_o + ((long long)s * rows + row) * D + c0);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                const float4 x = __ldcg(src + i);
                acc[4 * i] += f * x.x; acc[4 * i + 1] += f * x.y;
                acc[4 * i + 2] += f * x.z; acc[4 * i + 3] += f * x.w;
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    unsigned *dst = reinterpret_cast<unsigned *>(out + row * D + c0);
#pragma unroll
    for (int i = 0; i < D / 4; ++i) dst[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    if (lse) lse[row] = den > 0.f ? m + log2f(den) * kLn2 : -INFINITY;
}

// KLO: keys are held as a bf16 pair (hi, lo) whose sum carries ~16 mantissa
// bits; q.k is taken on both halves (used for the NSA compressed keys, which
// are means and do not fit bf16 exactly).
// TMAB (NSA selected blocks, head dim 128; opt-in, the row gather measured
// faster): the chunk's 16 consecutive rows of a block arrive by TMA box loads
// (kmap / vmap: [B*Lk rows, Hkv, D], box = 64 columns x 1 head x 16 rows,
// 128-byte swizzle) issued by lane 0, completion on a per-warp mbarrier; a K
// (or V) chunk is then two 64-column halves of 16 rows x 128 B instead of 16
// rows x 256 B.
// CTAM: the CTA-merged form above (explicit lists only).
template <int D, int STAGES, int SRC, bool BIAS, bool KLO = false, int NK = 32, int NW = 4, bool TMAB = false,
          bool CTAM = false>
__global__ void __launch_bounds__(NW * 32) gather_attn_kernel(const GatherParams p, const __grid_constant__ CUtensorMap kmap,
                                                              const __grid_constant__ CUtensorMap vmap) {
    grid_dependency_sync();
    // NK keys per chunk, NW independent warps per CTA
    constexpr int ROWB = D * 2;            // bytes of one K/V row
    constexpr int UNITS = ROWB / 16;       // 16-byte units per row
    constexpr int CH = NK * ROWB;          // bytes of one K (or V) chunk
    constexpr int KS_D = D / 16;           // k-steps of q.k
    constexpr int NT_D = D / 8;            // n-tiles of P.V
    constexpr int CP_ITERS = NK * UNITS / 32;
    constexpr int SB = (KLO ? 3 : 2) * CH;   // one stage: K | V | (K lo)
    static_assert(!TMAB || (SRC == KS_BLOCKS && D == 128 && NK == 16 && !KLO && !BIAS), "TMA block chunks");
    static_assert(!CTAM || (SRC == KS_IDX && !TMAB && !KLO && !BIAS), "CTA-merged pieces: explicit lists only");

    extern __shared__ __align__(1024) unsigned char smem_dyn[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool PR = SRC == KS_PROWS;
    constexpr int KEYB = NK * ((PR ? 8 : 4) + (BIAS ? 12 : 0));   // per stage: keys (+ segments, + coordinates)
    // TMA layout: every warp's stages first (1024-byte aligned for the 128-byte
    // swizzle), then the keys, then one mbarrier per stage and warp
    // cp.async layout: per warp its stages then its keys, the warp's region
    // padded to 256 bytes from a 256-byte aligned base, so that a K/V row
    // starts on a 256-byte boundary (the copy loop below relies on it)
    constexpr int WSTRIDE = STAGES * SB + ((STAGES * KEYB + 255) & ~255);
    unsigned char *smem = TMAB ? smem_dyn + ((1024u - (tc::smem_u32(smem_dyn) & 1023u)) & 1023u)
                               : smem_dyn + ((256u - (tc::smem_u32(smem_dyn) & 255u)) & 255u);
    unsigned char *wsm = TMAB ? smem + warp * (STAGES * SB) : smem + warp * WSTRIDE;
    int *keys_s = TMAB ? reinterpret_cast<int *>(smem + NW * STAGES * SB) + warp * STAGES * NK
                       : reinterpret_cast<int *>(wsm + STAGES * SB);
    uint64_t *full_s = reinterpret_cast<uint64_t *>(smem + NW * STAGES * (SB + NK * 4)) + warp * STAGES;
    int *segs_s = keys_s + STAGES * NK;                      // KS_PROWS only
    float *ck_s = reinterpret_cast<float *>(keys_s + STAGES * NK * (PR ? 2 : 1));   // [STAGES][NK][3] (bias only)
    if constexpr (TMAB) {
        if (lane == 0) {
            for (int i = 0; i < STAGES; ++i) tc::mbar_init(full_s + i, 1);
            tc::mbar_fence_init();
        }
        __syncwarp();
    }

    const long long n_items = (long long)p.B * p.q_units * p.Hkv * p.n_hchunk * p.n_split;
    // CTAM: one item per CTA, its warps take consecutive parts of the item's
    // entries and merge in shared memory at the end (the only block barrier);
    // otherwise one item per warp and the warps never wait for each other
    const long long item = CTAM ? (long long)blockIdx.x : (long long)blockIdx.x * NW + warp;
    if (item >= n_items) return;   // CTA-uniform under CTAM

    long long rem = item;
    const int s = (int)(rem % p.n_split); rem /= p.n_split;
    const int hc = (int)(rem % p.n_hchunk); rem /= p.n_hchunk;
    const int g = (int)(rem % p.Hkv); rem /= p.Hkv;
    const int tu = (int)(rem % p.q_units); rem /= p.q_units;
    const int b = (int)rem;
    // rows: 16/G queries x G heads (KS_PROWS) or 16 heads of one query
    const int nqw = PR ? 16 / p.G : 1;
    const int lq = 31 - __clz(nqw);                          // log2(nqw)
    int i0 = 0;                                              // first dilated exponent: 2^i0 >= window
    if constexpr (PR) {
        while ((1LL << i0) < p.window) ++i0;
    }
    const int t = tu * nqw;                                 // first query of the item
    const int t_end = min(t + nqw, p.Tq) - 1;              // last query of the item
    const long long pos = p.q_pos0 + t;

    const int gr = lane >> 2, qc = lane & 3;
    const int tr0 = PR ? t + gr / p.G : t, tr1 = PR ? t + (gr + 8) / p.G : t;   // query of each row
    const int hr0 = PR ? gr % p.G : hc * 16 + gr, hr1 = PR ? (gr + 8) % p.G : hc * 16 + gr + 8;
    const bool v0 = hr0 < p.G && tr0 <= t_end, v1 = hr1 < p.G && tr1 <= t_end;
    const int h0 = g * p.G + hr0, h1 = g * p.G + hr1;
    const long long qrow0 = ((long long)(b * p.Tq + (v0 ? tr0 : t)) * p.Hq + h0) * D;
    const long long qrow1 = ((long long)(b * p.Tq + (v1 ? tr1 : t)) * p.Hq + h1) * D;

    // Q fragments (A operand, 16 rows x D), straight from global memory.
    unsigned qf[KS_D][4];
    {
        const unsigned *q0 = reinterpret_cast<const unsigned *>(p.q + qrow0);
        const unsigned *q1 = reinterpret_cast<const unsigned *>(p.q + qrow1);
#pragma unroll
        for (int ks = 0; ks < KS_D; ++ks) {
            qf[ks][0] = v0 ? __ldg(q0 + ks * 8 + qc) : 0u;
            qf[ks][1] = v1 ? __ldg(q1 + ks * 8 + qc) : 0u;
            qf[ks][2] = v0 ? __ldg(q0 + ks * 8 + qc + 4) : 0u;
            qf[ks][3] = v1 ? __ldg(q1 + ks * 8 + qc + 4) : 0u;
        }
        // a negative scale is folded into Q (sign bits of both bf16 halves),
        // so every score below is scaled by |scale| and keeps the order of q.k
        if (p.scale_log2 < 0.f) {
#pragma unroll
            for (int ks = 0; ks < KS_D; ++ks)
#pragma unroll
                for (int r = 0; r < 4; ++r) qf[ks][r] ^= 0x80008000u;
        }
    }
    const float sl2 = fabsf(p.scale_log2);
    float cq0[3] = {0.f, 0.f, 0.f}, cq1[3] = {0.f, 0.f, 0.f}, be0 = 0.f, be1 = 0.f;
    if constexpr (BIAS) {
        if (v0) {
            const float *c = p.cq + ((long long)(b * p.Tq + tr0) * p.Hq + h0) * 3;
            cq0[0] = c[0]; cq0[1] = c[1]; cq0[2] = c[2];
            be0 = p.beta[h0] * kLog2e;
        }
        if (v1) {
            const float *c = p.cq + ((long long)(b * p.Tq + tr1) * p.Hq + h1) * 3;
            cq1[0] = c[0]; cq1[1] = c[1]; cq1[2] = c[2];
            be1 = p.beta[h1] * kLog2e;
        }
    }

    int e_beg = s * p.per_split;
    int e_end = min(p.entries, e_beg + p.per_split);
    if constexpr (CTAM) {
        // the warp's part of the piece: whole chunks, consecutive
        const int len = max(e_end - e_beg, 0);
        const int part = (len + NW * NK - 1) / (NW * NK) * NK;
        e_beg = min(e_beg + warp * part, e_end);
        e_end = min(e_end, e_beg + part);
    }
    const int n_chunks = e_end > e_beg ? (e_end - e_beg + NK - 1) / NK : 0;

    const __nv_bfloat16 *kb = p.k + ((long long)b * p.Lk * p.Hkv + g) * D;
    const __nv_bfloat16 *vb = p.v + ((long long)b * p.Lk * p.Hkv + g) * D;
    const __nv_bfloat16 *lb = KLO ? p.klo + ((long long)b * p.Lk * p.Hkv + g) * D : nullptr;
    const long long rstride = (long long)p.Hkv * D;
    [[maybe_unused]] const uint32_t rs_bytes = (uint32_t)(rstride * 2);    // Hkv * D * 2 < 2^32
    // copy lanes: lane = lrow * UNITS + u (u: 16-byte unit of a row, lrow: row within an instruction)
    [[maybe_unused]] constexpr int RPI = 32 / UNITS;
    [[maybe_unused]] const int lrow_c = lane / UNITS, u_c = lane % UNITS;
    [[maybe_unused]] const __nv_bfloat16 *kb_u = kb + u_c * 8, *vb_u = vb + u_c * 8;
    [[maybe_unused]] const __nv_bfloat16 *lb_u = KLO ? lb + u_c * 8 : nullptr;

    // raw list value of chunk ci for this lane (lane i < NK owns key i)
    auto raw_of = [&](int ci) -> int {
        return (ci < n_chunks && lane < NK) ? key_raw<SRC>(p, b, t, g, pos, e_beg + ci * NK + lane, e_end)
                                            : KEY_NONE;
    };
    auto issue = [&](int ci, int raw) {
        const int st = ci % STAGES;
        unsigned char *ks_ = wsm + st * SB;
        unsigned char *vs_ = ks_ + CH;
        int j, seg = 0;
        if constexpr (PR) {
            j = (ci < n_chunks && lane < NK)
                    ? key_prows(p, pos, p.q_pos0 + t_end, lq, i0, e_beg + ci * NK + lane, e_end, seg) : -1;
        } else {
            j = key_finish<SRC>(p, pos, raw, e_beg + ci * NK + lane);
        }
        if (lane < NK) {
            keys_s[st * NK + lane] = j;
            if constexpr (PR) segs_s[st * NK + lane] = (int)prows_rowmask(j, seg, pos, t_end - t + 1, p.window, p.G);
            if constexpr (BIAS) {
                // the key's coordinates ride with its K/V rows (same commit group)
                if (j >= 0) {
                    const float *c = p.ck + ((long long)(b * p.Lk + j) * p.Hkv + g) * 3;
                    float *dst = ck_s + (st * NK + lane) * 3;
                    cp_async4(dst, c);
                    cp_async4(dst + 1, c + 1);
                    cp_async4(dst + 2, c + 2);
                }
            }
        }
        if constexpr (TMAB) {
            // the chunk's 16 rows are consecutive rows of one block: four box
            // loads (K and V, two 64-column halves each); a chunk without a
            // valid block loads block 0 so masked rows stay finite
            if (ci < n_chunks && lane == 0) {
                const int e0 = e_beg + ci * NK;
                int blk = raw;                                   // lane 0's raw list value: the block id
                if (blk == KEY_NONE || blk < 0 || (long long)blk * p.block >= p.Lk) blk = 0;
                const int z = b * p.Lk + blk * p.block + (e0 % p.block);
                tc::fence_proxy_async_smem();                    // the stage's last readers are done (syncwarp)
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(tc::smem_u32(full_s + st)),
                             "r"(2 * CH)
                             : "memory");
                for (int h = 0; h < 2; ++h) {
                    asm volatile(
                        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(tc::smem_u32(ks_ + h * (NK * 128))),
                        "l"(reinterpret_cast<uint64_t>(&kmap)), "r"(h * 64), "r"(g), "r"(z), "r"(tc::smem_u32(full_s + st))
                        : "memory");
                    asm volatile(
                        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(tc::smem_u32(vs_ + h * (NK * 128))),
                        "l"(reinterpret_cast<uint64_t>(&vmap)), "r"(h * 64), "r"(g), "r"(z), "r"(tc::smem_u32(full_s + st))
                        : "memory");
                }
            }
            return;
        }
        if (ci < n_chunks) {
            if constexpr (D == 128) {
                // UNITS lanes per key row, RPI = 32 / UNITS rows per instruction,
                // so every copy instruction covers whole 128-byte lines.  Lane
                // (lrow, u) copies unit u of rows it * RPI + lrow to the swizzled
                // unit u ^ (row & 7); with the stage on a 256-byte boundary that
                // address is (base ^ (((it * RPI) & 7) << 4)) + it * RPI * ROWB,
                // one XOR per row; the row offsets are immediates.
                const uint32_t base = tc::smem_u32(ks_) + lrow_c * ROWB + ((u_c ^ lrow_c) << 4);
                static_for<CP_ITERS>([&](auto ic) {
                    constexpr int it = decltype(ic)::value;
                    const int jr = __shfl_sync(0xffffffffu, j, it * RPI + lrow_c);
                    // row offset in bytes: a 32 x 32 -> 64-bit multiply-add per
                    // pointer (the row stride Hkv * D * 2 fits 32 bits)
                    const uint32_t jc = (uint32_t)max(jr, 0);
                    const int nb = jr >= 0 ? 16 : 0;
                    const uint32_t dst = base ^ (uint32_t)(((it * RPI) & 7) << 4);
                    cp_async16_at<it * RPI * ROWB, 0>(dst, reinterpret_cast<const char *>(kb_u) + (size_t)jc * rs_bytes, nb);
                    cp_async16_at<it * RPI * ROWB + CH, 0>(dst, reinterpret_cast<const char *>(vb_u) + (size_t)jc * rs_bytes,
                                                         nb);
                    if constexpr (KLO)
                        cp_async16_at<it * RPI * ROWB + 2 * CH, 0>(
                            dst, reinterpret_cast<const char *>(lb_u) + (size_t)jc * rs_bytes, nb);
                });
            } else {
                // head dim 64 (measured faster for the fixed-graph rows): the
                // same lane mapping with addresses formed per copy
#pragma unroll
                for (int it = 0; it < CP_ITERS; ++it) {
                    const int lin = it * 32 + lane;
                    const int rr = lin / UNITS, u = lin % UNITS;
                    const int jr = __shfl_sync(0xffffffffu, j, rr);
                    const size_t off = (size_t)(uint32_t)max(jr, 0) * rs_bytes + u * 16;   // bytes
                    const int nb = jr >= 0 ? 16 : 0;
                    const int sw = (u ^ (rr & 7)) * 16;
                    cp_async16(ks_ + rr * ROWB + sw, reinterpret_cast<const char *>(kb) + off, nb);
                    cp_async16(vs_ + rr * ROWB + sw, reinterpret_cast<const char *>(vb) + off, nb);
                    if constexpr (KLO) cp_async16(vs_ + CH + rr * ROWB + sw, reinterpret_cast<const char *>(lb) + off, nb);
                }
            }
        }
        cp_async_commit();
    };

    float o[NT_D][4];
#pragma unroll
    for (int i = 0; i < NT_D; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool timed_out = false;

    // the list values of the first STAGES + 1 chunks are loaded together (one
    // memory latency, not one per prologue chunk), then the prologue copies
    // go out; in the loop, list values run two chunks ahead of their copies
    int raw0[STAGES + 1];
#pragma unroll
    for (int ci = 0; ci <= STAGES; ++ci) raw0[ci] = raw_of(ci);
#pragma unroll
    for (int ci = 0; ci < STAGES - 1; ++ci) issue(ci, raw0[ci]);
    int raw_a = raw0[STAGES - 1], raw_b = raw0[STAGES];

    for (int ci = 0; ci < n_chunks; ++ci) {
        const int raw = raw_a;
        raw_a = raw_b;
        raw_b = raw_of(ci + STAGES + 1);
        issue(ci + STAGES - 1, raw);
        const int st = ci % STAGES;
        if constexpr (TMAB) {
            // every lane waits for the chunk's bytes (bounded); a timeout is
            // recorded and the data is ignored, the CTA drains before exit
            const bool got = __all_sync(0xffffffffu, tc::mbar_wait_bounded(full_s + st, (ci / STAGES) & 1, spin_limit()));
            if (!got && !timed_out) {
                timed_out = true;
                if (lane == 0) raise_error(p.err, ERR_TIMEOUT);
            }
        } else {
            cp_async_wait<STAGES - 1>();
        }
        __syncwarp();
        const unsigned char *ks_ = wsm + st * SB;
        const unsigned char *vs_ = ks_ + CH;
        // ldmatrix addresses.  Row-gather layout: key row r at r * ROWB, its
        // 16-byte unit u at ((u ^ (r & 7)) << 4), stages 256-byte aligned.  TMA
        // block layout: 64-column halves NK * 128 bytes apart, rows of 128
        // bytes, unit u of a half at (((u & 7) ^ (r & 7)) << 4).  For the
        // row-gather layout at head dim 128 the lane's row and the XOR of its
        // swizzle are folded into one base, each 16-column step is then one XOR.  Q.K^T reads key rows (mi >> 1) * 8 + ri
        // at unit 2s + (mi & 1), P.V rows (mi & 1) * 8 + ri at unit 2s + (mi >> 1)
        // (mi = lane / 8, ri = lane % 8); the swizzle XORs the unit with ri
        [[maybe_unused]] const uint32_t ka_s =
            tc::smem_u32(ks_) + (uint32_t)((((lane >> 4) * 8) + (lane & 7)) * ROWB + ((((lane >> 3) & 1) ^ (lane & 7)) << 4));
        [[maybe_unused]] const uint32_t va_s =
            tc::smem_u32(vs_) + (uint32_t)(((((lane >> 3) & 1) * 8) + (lane & 7)) * ROWB + (((lane >> 4) ^ (lane & 7)) << 4));
        const int jl = lane < NK ? keys_s[st * NK + lane] : -1;
        const int sl = PR && lane < NK ? segs_s[st * NK + lane] : 0;
        const unsigned vmask = __ballot_sync(0xffffffffu, jl >= 0);
        if (vmask != 0u) {
            // q.k over the head dimension; even and odd k-steps accumulate
            // into separate registers so more MMA chains are independent
            float sc[NK / 8][4], sc2[NK / 8][4];
#pragma unroll
            for (int i = 0; i < NK / 8; ++i)
                sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = sc2[i][0] = sc2[i][1] = sc2[i][2] = sc2[i][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS_D; ++ks) {
                float (&acc)[NK / 8][4] = (ks & 1) ? sc2 : sc;
#pragma unroll
                for (int np = 0; np < NK / 16; ++np) {
                    unsigned b0, b1, b2, b3;
                    if constexpr (TMAB || D == 64) {
                        // per-step swizzle arithmetic: the folded form below
                        // measured no faster for the TMA block layout and
                        // slower at head dim 64
                        const int mi = lane >> 3, ri = lane & 7;
                        const int key = np * 16 + (mi >> 1) * 8 + ri;
                        const int unit = ks * 2 + (mi & 1);
                        const int off = TMAB ? (unit >> 3) * (NK * 128) + key * 128 + (((unit & 7) ^ (key & 7)) << 4)
                                             : key * ROWB + ((unit ^ (key & 7)) << 4);
                        ldsm_x4(b0, b1, b2, b3, ks_ + off);
                    } else {
                        ldsm_x4_a(b0, b1, b2, b3, (ka_s + np * 16 * ROWB) ^ (uint32_t)(ks << 5));
                    }
                    mma_bf16_16816(acc[2 * np], qf[ks], b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], qf[ks], b2, b3);
                    if constexpr (KLO) {
                        // the lo half of the keys, 2 * CH bytes after the hi half
                        ldsm_x4_a(b0, b1, b2, b3, (ka_s + 2 * CH + np * 16 * ROWB) ^ (uint32_t)(ks << 5));
                        mma_bf16_16816(acc[2 * np], qf[ks], b0, b1);
                        mma_bf16_16816(acc[2 * np + 1], qf[ks], b2, b3);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < NK / 8; ++i) {
                sc[i][0] += sc2[i][0]; sc[i][1] += sc2[i][1];
                sc[i][2] += sc2[i][2]; sc[i][3] += sc2[i][3];
            }
            // running max.  Plain lists keep the raw q.k (the scale, > 0 after
            // the sign fold, goes into the exponent's FFMA) and mask only a
            // chunk with empty entries; bias and row masks scale first.
            constexpr bool RAW = !BIAS && !PR;
            float mx0 = -INFINITY, mx1 = -INFINITY;
            constexpr unsigned kFull = NK == 32 ? 0xffffffffu : ((1u << NK) - 1u);
            const bool partial = RAW && vmask != kFull;        // warp-uniform
            if constexpr (RAW) {
                if (partial) {
#pragma unroll
                    for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (!((vmask >> (nt * 8 + 2 * qc + (e & 1))) & 1u)) sc[nt][e] = -INFINITY;
                }
#pragma unroll
                for (int nt = 0; nt < NK / 8; ++nt) {
                    mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
                    mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
                }
            } else {
                // per key of this thread (two per n-tile): its row mask (fixed
                // graph) and coordinates once, then its two rows
#pragma unroll
                for (int nt = 0; nt < NK / 8; ++nt) {
#pragma unroll
                    for (int par = 0; par < 2; ++par) {
                        const int kk = nt * 8 + 2 * qc + par;
                        const bool kv = (vmask >> kk) & 1u;
                        bool ok0 = kv, ok1 = kv;
                        if constexpr (PR) {
                            const unsigned km = (unsigned)__shfl_sync(0xffffffffu, sl, kk);   // rows seeing key kk
                            ok0 = ok0 && ((km >> gr) & 1u);
                            ok1 = ok1 && ((km >> (gr + 8)) & 1u);
                        }
                        float x0 = sc[nt][par] * sl2, x1 = sc[nt][2 + par] * sl2;
                        if constexpr (BIAS) {
                            // an empty entry's coordinates are stale: its
                            // score is replaced by -inf below
                            const float *c = ck_s + (st * NK + kk) * 3;
                            const float c0 = c[0], c1 = c[1], c2 = c[2];
                            float dx = cq0[0] - c0, dy = cq0[1] - c1, dz = cq0[2] - c2;
                            x0 -= be0 * (dx * dx + dy * dy + dz * dz);
                            dx = cq1[0] - c0; dy = cq1[1] - c1; dz = cq1[2] - c2;
                            x1 -= be1 * (dx * dx + dy * dy + dz * dz);
                        }
                        sc[nt][par] = ok0 ? x0 : -INFINITY;
                        sc[nt][2 + par] = ok1 ? x1 : -INFINITY;
                    }
                    mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
                    mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
                }
            }
            // m0 / m1 and everything below are in the scaled log2 domain.
            // m0 / m1 are reference maxima, not running maxima: they move
            // (and the accumulators are rescaled) only when some row's chunk
            // maximum exceeds its reference by more than kLazy, so weights
            // 2^(x - m) stay below 2^kLazy (exact in bf16 up to its usual
            // rounding, no overflow in fp32 sums) and most chunks skip the
            // rescale.  softmax is the same for any reference value.  The
            // test needs no row maximum: a row's maximum exceeds m + kLazy iff
            // one of its four lanes' partial maxima does, so the quad
            // shuffles run only when the reference moves.
            constexpr float kOne = 1.f, kLazy = 8.f;
            const float xs = RAW ? sl2 : kOne;                 // factor still to apply to sc
            if (__any_sync(0xffffffffu, (RAW ? mx0 * sl2 : mx0) > m0 + kLazy ||
                                            (RAW ? mx1 * sl2 : mx1) > m1 + kLazy)) {   // warp-uniform
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                const float cm0 = RAW ? mx0 * sl2 : mx0, cm1 = RAW ? mx1 * sl2 : mx1;
                const float mn0 = fmaxf(m0, cm0), mn1 = fmaxf(m1, cm1);
                const float al0 = m0 == -INFINITY ? 0.f : ex2_fast(m0 - mn0);
                const float al1 = m1 == -INFINITY ? 0.f : ex2_fast(m1 - mn1);
                m0 = mn0; m1 = mn1;
                l0 *= al0; l1 *= al1;
#pragma unroll
                for (int i = 0; i < NT_D; ++i) {
                    o[i][0] *= al0; o[i][1] *= al0;
                    o[i][2] *= al1; o[i][3] *= al1;
                }
            }
            const float mu0 = m0 == -INFINITY ? 0.f : m0;
            const float mu1 = m1 == -INFINITY ? 0.f : m1;
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < NK / 8; ++nt) {
                sc[nt][0] = ex2_fast(fmaf(sc[nt][0], xs, -mu0));
                sc[nt][1] = ex2_fast(fmaf(sc[nt][1], xs, -mu0));
                sc[nt][2] = ex2_fast(fmaf(sc[nt][2], xs, -mu1));
                sc[nt][3] = ex2_fast(fmaf(sc[nt][3], xs, -mu1));
                if (partial) {                                 // exact zeros for empty entries (any scale)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (!((vmask >> (nt * 8 + 2 * qc + (e & 1))) & 1u)) sc[nt][e] = 0.f;
                }
                rs0 += sc[nt][0] + sc[nt][1];
                rs1 += sc[nt][2] + sc[nt][3];
            }
            l0 += rs0;
            l1 += rs1;
            // P (bf16) * V
#pragma unroll
            for (int kp = 0; kp < NK / 16; ++kp) {
                unsigned pa[4];
                pa[0] = pack_bf16(sc[2 * kp][0], sc[2 * kp][1]);
                pa[1] = pack_bf16(sc[2 * kp][2], sc[2 * kp][3]);
                pa[2] = pack_bf16(sc[2 * kp + 1][0], sc[2 * kp + 1][1]);
                pa[3] = pack_bf16(sc[2 * kp + 1][2], sc[2 * kp + 1][3]);
#pragma unroll
                for (int dp = 0; dp < NT_D / 2; ++dp) {
                    unsigned b0, b1, b2, b3;
                    if constexpr (TMAB || D == 64) {
                        const int mi = lane >> 3, ri = lane & 7;
                        const int key = kp * 16 + (mi & 1) * 8 + ri;
                        const int unit = dp * 2 + (mi >> 1);
                        const int off = TMAB ? (unit >> 3) * (NK * 128) + key * 128 + (((unit & 7) ^ (key & 7)) << 4)
                                             : key * ROWB + ((unit ^ (key & 7)) << 4);
                        ldsm_x4_t(b0, b1, b2, b3, vs_ + off);
                    } else {
                        ldsm_x4_ta(b0, b1, b2, b3, (va_s + kp * 16 * ROWB) ^ (uint32_t)(dp << 5));
                    }
                    mma_bf16_16816(o[2 * dp], pa, b0, b1);
                    mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if constexpr (TMAB) {
        // after a timeout some loads may still be in flight: let every
        // stage's latest phase complete (fixed long limit) before exiting
        if (timed_out && lane == 0) {
            for (int ci = (n_chunks > STAGES ? n_chunks - STAGES : 0); ci < n_chunks; ++ci)
                tc::mbar_wait_bounded(full_s + ci % STAGES, (ci / STAGES) & 1, kDefaultSpinCycles);
        }
        __syncwarp();
    }

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if constexpr (CTAM) {
        // this warp's rows (reference maximum, sum, unnormalised O) go to its
        // own stage buffers (its copies are complete), then the CTA merges
        // the NW parts of each of the 16 rows: M = max m_w, L = sum l_w 2^(m_w - M),
        // O = sum o_w 2^(m_w - M) / L
        float *ml_s = reinterpret_cast<float *>(wsm);          // [2][16]: m, l
        float *o_s = ml_s + 32;                                 // [16][D]
        if (qc == 0) {
            ml_s[gr] = m0; ml_s[gr + 8] = m1;
            ml_s[16 + gr] = l0; ml_s[16 + gr + 8] = l1;
        }
#pragma unroll
        for (int nt = 0; nt < NT_D; ++nt) {
            const int c = nt * 8 + 2 * qc;
            *reinterpret_cast<float2 *>(o_s + gr * D + c) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2 *>(o_s + (gr + 8) * D + c) = make_float2(o[nt][2], o[nt][3]);
        }
        __syncthreads();
        for (int job = threadIdx.x; job < 16 * (D / 4); job += NW * 32) {
            const int r = job / (D / 4), c = (job % (D / 4)) * 4;
            const int hr = hc * 16 + r;
            if (hr >= p.G) continue;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NW; ++w) M = fmaxf(M, reinterpret_cast<const float *>(smem + w * WSTRIDE)[r]);
            float L = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    const float *wb = reinterpret_cast<const float *>(smem + w * WSTRIDE);
                    const float mw = wb[r];
                    const float f = mw == -INFINITY ? 0.f : ex2_fast(mw - M);
                    const float4 x = *reinterpret_cast<const float4 *>(wb + 32 + r * D + c);
                    L += f * wb[16 + r];
                    acc.x += f * x.x; acc.y += f * x.y; acc.z += f * x.z; acc.w += f * x.w;
                }
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
            const float lsev = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
            const long long orow = (long long)(b * p.Tq + t) * p.Hq + g * p.G + hr;
            if (p.n_split == 1) {
                if (p.out_f32) {
                    *reinterpret_cast<float4 *>(p.out_f32 + orow * D + c) =
                        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
                } else {
                    *reinterpret_cast<uint2 *>(p.out + orow * D + c) =
                        make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
                }
                if (p.lse && c == 0) p.lse[orow] = lsev;
            } else {
                const long long rows = (long long)p.B * p.Tq * p.Hq;
                *reinterpret_cast<float4 *>(p.part_o + ((long long)s * rows + orow) * D + c) =
                    make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
                if (c == 0) p.part_lse[s * rows + orow] = lsev;
            }
        }
        if (p.n_split > 1 && p.merge_cnt) {
            // the last CTA of the group to arrive merges every piece's rows
            // (the others only publish theirs): ticket after a fence, fence
            // before reading the other pieces' rows from L2
            __shared__ int last_s;
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) {
                int *ticket = p.merge_cnt + ((long long)(b * p.Tq + t) * p.Hkv + g) * p.n_hchunk + hc;
                const bool last = atomicAdd(ticket, 1) == p.n_split - 1;
                if (last) *ticket = 0;                      // ready for the next call
                last_s = last;
            }
            __syncthreads();
            if (last_s) {
                __threadfence();
                const long long rows = (long long)p.B * p.Tq * p.Hq;
                for (int job = threadIdx.x; job < 16 * (D / 4); job += NW * 32) {
                    const int r = job / (D / 4), c = (job % (D / 4)) * 4;
                    const int hr = hc * 16 + r;
                    if (hr >= p.G) continue;
                    const long long orow = (long long)(b * p.Tq + t) * p.Hq + g * p.G + hr;
                    float M = -INFINITY;
                    for (int q = 0; q < p.n_split; ++q) M = fmaxf(M, __ldcg(p.part_lse + q * rows + orow));
                    float den = 0.f;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (M != -INFINITY) {
                        for (int q = 0; q < p.n_split; ++q) {
                            const float lq = __ldcg(p.part_lse + q * rows + orow);
                            const float f = lq == -INFINITY ? 0.f : ex2_fast((lq - M) * kLog2e);
                            const float4 x = __ldcg(reinterpret_cast<const float4 *>(p.part_o + (q * rows + orow) * D + c));
                            den += f;
                            acc.x += f * x.x; acc.y += f * x.y; acc.z += f * x.z; acc.w += f * x.w;
                        }
                    }
                    const float inv = den > 0.f ? 1.f / den : 0.f;
                    *reinterpret_cast<uint2 *>(p.out + orow * D + c) =
                        make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
                    if (p.lse && c == 0) p.lse[orow] = den > 0.f ? M + log2f(den) * kLn2 : -INFINITY;
                }
            }
        }
        return;
    }
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
    const float lse0 = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
    const float lse1 = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;

    const long long orow0 = (long long)(b * p.Tq + tr0) * p.Hq + h0;
    const long long orow1 = (long long)(b * p.Tq + tr1) * p.Hq + h1;
    if (p.n_split == 1) {
        if (p.out_f32) {
#pragma unroll
            for (int nt = 0; nt < NT_D; ++nt) {
                const int dcol = nt * 8 + 2 * qc;
                if (v0) *reinterpret_cast<float2 *>(p.out_f32 + orow0 * D + dcol) =
                    make_float2(o[nt][0] * inv0, o[nt][1] * inv0);
                if (v1) *reinterpret_cast<float2 *>(p.out_f32 + orow1 * D + dcol) =
                    make_float2(o[nt][2] * inv1, o[nt][3] * inv1);
            }
        } else {
#pragma unroll
            for (int nt = 0; nt < NT_D; ++nt) {
                const int dcol = nt * 8 + 2 * qc;
                if (v0) *reinterpret_cast<unsigned *>(p.out + orow0 * D + dcol) =
                    pack_bf16(o[nt][0] * inv0, o[nt][1] * inv0);
                if (v1) *reinterpret_cast<unsigned *>(p.out + orow1 * D + dcol) =
                    pack_bf16(o[nt][2] * inv1, o[nt][3] * inv1);
            }
        }
        if (p.lse && qc == 0) {
            if (v0) p.lse[orow0] = lse0;
            if (v1) p.lse[orow1] = lse1;
        }
    } else {
        const long long rows = (long long)p.B * p.Tq * p.Hq;
        float *po = p.part_o + (long long)s * rows * D;
#pragma unroll
        for (int nt = 0; nt < NT_D; ++nt) {
            const int dcol = nt * 8 + 2 * qc;
            if (v0) *reinterpret_cast<float2 *>(po + orow0 * D + dcol) =
                make_float2(o[nt][0] * inv0, o[nt][1] * inv0);
            if (v1) *reinterpret_cast<float2 *>(po + orow1 * D + dcol) =
                make_float2(o[nt][2] * inv1, o[nt][3] * inv1);
        }
        if (qc == 0) {
            if (v0) p.part_lse[s * rows + orow0] = lse0;
            if (v1) p.part_lse[s * rows + orow1] = lse1;
        }
        if (p.merge_cnt) {
            // the last piece of the group to arrive merges all pieces (the
            // others only publish their partial rows): ticket after a fence,
            // fence before reading the other pieces' rows from L2
            __threadfence();
            __syncwarp();
            int last = 0;
            if (lane == 0) {
                int *ticket = p.merge_cnt + ((long long)(b * p.Tq + t) * p.Hkv + g) * p.n_hchunk + hc;
                last = atomicAdd(ticket, 1) == p.n_split - 1;
                if (last) *ticket = 0;                     // ready for the next call
            }
            if (__shfl_sync(0xffffffffu, last, 0)) {
                __threadfence();
                // lane l: head row l / 2 of the item, columns (l % 2) * D/2 .. + D/2
                const int hr = hc * 16 + (lane >> 1);
                if (hr < p.G) {
                    const long long row = (long long)(b * p.Tq + t) * p.Hq + g * p.G + hr;
                    merge_pieces_half<D>(p.part_o, p.part_lse, p.n_split, rows, row, (lane & 1) * (D / 2), p.out,
                                         (lane & 1) == 0 ? p.lse : nullptr);
                }
            }
        }
    }
}

template <int D, int STAGES, bool KLO = false, int NK = 32, int NW = 4, bool PR = false, bool BIAS = false,
          bool TMAB = false>
constexpr int gather_smem_bytes() {
    constexpr int SB = (KLO ? 3 : 2) * NK * D * 2;
    constexpr int KEYB = NK * ((PR ? 8 : 4) + (BIAS ? 12 : 0));
    return TMAB ? NW * STAGES * (SB + KEYB) + NW * STAGES * 8 + 1024
                : NW * (STAGES * SB + ((STAGES * KEYB + 255) & ~255)) + 256;
}

}  // namespace sa
