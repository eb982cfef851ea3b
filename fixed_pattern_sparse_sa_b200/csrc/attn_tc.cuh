// attn_tc.cuh -- gathered-KV sparse attention on the tcgen05 tensor cores.
//
// Same operation as gather_attn_kernel for explicit key lists (DSA top-k
// lists, NSA selected blocks): for each query t and KV group g, the G <= 16
// query heads of the group attend to the keys of their list,
//   o_h = sum_j softmax_j(scale * q_h . k_j) v_j,  lse_h = log sum_j exp(...)
// (IndexCache page, body: attention restricted to the indexer's top-k; NSA
// page, "Puntos Clave": attention over the selected blocks).
//
// One work item = (b, t, g, split piece); its keys are taken 128 at a time.
// With keys on the M side, both products are single 128-row MMAs:
//   S^T[128 keys x 16 heads] = K_tile[128 x D] . Q^T          (kind::f16)
//   O^T[D x 16 heads]       += V_tile^T[D x 128] . P^T[128 x 16]
// K and V rows are gathered with 16-byte cp.async copies (two whole 256-byte
// rows per warp instruction) into 128B-swizzled tiles that serve directly as
// the K-major A operand of the first MMA and the MN-major A operand of the
// second; the Q tile of an item is one TMA box load.
//
// Warp roles (288 threads, one persistent CTA per SM):
//   warps 0-3  producers: thread i validates list entry i of the tile; the
//              warps copy their 32 rows (a ring of ATC_STAGES K/V stages);
//              warp 0 also loads the Q tiles;
//   warp 4     MMA issuer (one thread) and TMEM owner;
//   warps 5-8  softmax + epilogue: thread r owns key row r of S^T (and row r
//              of O^T = output column d = r); per-head maxima are combined
//              across the four warps through shared memory.
// The running maximum is only raised (and O rescaled in TMEM) when some
// logit of a tile exceeds it by more than 2^60: one vote of the softmax
// group per tile, and the exact cross-warp max only on a tile that needs it
// (in practice an item's first).
// Every wait is bounded; on a timeout the kernel records ERR_TIMEOUT, stops
// issuing work, waits (bounded) for its own copies and frees its TMEM.
#pragma once

#include <cuda.h>

#include "attn_gather.cuh"
#include "tc_common.cuh"

namespace sa {

constexpr int ATC_STAGES = 3;               // K/V ring depth (64 KB per stage for D = 128)
constexpr int ATC_THREADS = 288;
constexpr int ATC_PRODUCERS = 128;          // producer threads (warps 0-3)
constexpr int ATC_MMA_WARP = 4;
constexpr int ATC_KEYS = 128;               // keys per tile
constexpr long long ATC_WAIT = 2000000000LL;   // ~1 s in SM clocks: drain waits
constexpr float ATC_RAISE = 60.f;           // log2 headroom of the running softmax max

struct AtcParams {
    GatherParams g;                         // shapes, list, outputs, scale, error word
    int n_items;                            // B * Tq * Hkv * n_split
};

// shared memory layout (offsets from a 1024-byte aligned base)
template <int D>
struct AtcSmem {
    static constexpr int KV_BYTES = ATC_KEYS * D * 2;            // one K (or V) tile
    static constexpr int STAGE = 2 * KV_BYTES;
    static constexpr int Q_BYTES = 16 * D * 2;
    static constexpr int P_BYTES = ATC_KEYS * 16 * 2;
    static constexpr int OFF_KV = 0;
    static constexpr int OFF_Q = OFF_KV + ATC_STAGES * STAGE;    // 2 buffers
    static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;            // 2 buffers
    static constexpr int OFF_KEYS = OFF_P + 2 * P_BYTES;         // [ATC_STAGES][128] int
    // reductions: per-warp maxima [4][16] (ints), combined maxima [16],
    // per-warp row sums [4][16] at float offset 128
    static constexpr int OFF_RED = OFF_KEYS + ATC_STAGES * ATC_KEYS * 4;
    static constexpr int OFF_BAR = OFF_RED + 1024;
    // barriers: kv_full[S], kv_empty[S], q_full[2], q_empty[2], s_full[2],
    // s_free[2], p_full[2], pv_done[2], o_full, o_free, drain, tma_full[S]
    static constexpr int N_BAR = 3 * ATC_STAGES + 12 + 3;
    static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;         // tmem slot, abort flag
    static constexpr int TOTAL = OFF_MISC + 16;
    static constexpr int ALLOC = TOTAL + 1024;                   // room to align the base
};

namespace atc {

__device__ __forceinline__ void expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(tc::smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(tc::smem_u32(bar)) : "memory");
}
// one arrival on `bar`, made by the hardware once every cp.async issued so
// far by this thread has completed
__device__ __forceinline__ void arrive_on_copies(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(tc::smem_u32(bar)) : "memory");
}
// box of a 2-D tensor map at (x, y)
__device__ __forceinline__ void load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(tc::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(tc::smem_u32(bar))
        : "memory");
}
// box of a 3-D tensor map at (x, y, z)
__device__ __forceinline__ void load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(tc::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(tc::smem_u32(bar))
        : "memory");
}
// shared-memory descriptor, 128-byte swizzle
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
// Named-barrier OR over the n threads of barrier `id` (same verdict for all).
__device__ __forceinline__ bool vote_any(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
// Named-barrier AND over the n threads of barrier `id`: every thread gets the
// same verdict, so a failed wait never leaves part of the group behind at a
// later barrier.
__device__ __forceinline__ bool agree(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
// order-preserving float <-> int map (for integer max reductions)
__device__ __forceinline__ int f2ord(float x) {
    const int i = __float_as_int(x);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float ord2f(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

// Bounded progress wait (spin_limit() clocks) that also gives up once
// another role has aborted.
__device__ __forceinline__ bool wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    const long long limit = spin_limit();
    for (unsigned n = 1;; ++n) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((n & 15u) == 0u && (*abort_flag || clock64() - t0 > limit)) return false;
    }
}

}  // namespace atc

// Item -> (b, t, g, split) in the gather kernel's order (split fastest).
__device__ __forceinline__ void atc_item(const GatherParams &p, int it, int &b, int &t, int &g, int &s) {
    int r = it;                                    // the item count fits in int (checked by the host)
    s = r % p.n_split; r /= p.n_split;
    g = r % p.Hkv; r /= p.Hkv;
    t = r % p.Tq; r /= p.Tq;
    b = r;
}

// SRC = KS_IDX gathers key rows with cp.async; SRC = KS_BLOCKS (NSA selected
// blocks of p.block consecutive keys) loads each block's K and V rows with TMA
// box loads (kmap / vmap: [B*Lk rows, Hkv, D] bf16, box = one block).
template <int D, int SRC>
__global__ void __launch_bounds__(ATC_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const AtcParams ap) {
    grid_dependency_sync();
    static_assert(D == 128, "the tensor-core gather path handles head dim 128");
    constexpr bool TMA = SRC == KS_BLOCKS;
    using L = AtcSmem<D>;
    const GatherParams &p = ap.g;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
    uint64_t *kv_full = bars, *kv_empty = bars + ATC_STAGES;
    uint64_t *q_full = bars + 2 * ATC_STAGES, *q_empty = q_full + 2;
    uint64_t *s_full = q_empty + 2, *s_free = s_full + 2;
    uint64_t *p_full = s_free + 2, *pv_done = p_full + 2;
    uint64_t *o_full = pv_done + 2, *o_free = o_full + 1, *drain = o_free + 1;
    uint64_t *tma_full = drain + 1;                 // KS_BLOCKS: bytes of a stage's TMA block loads
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);
    int *keys_s = reinterpret_cast<int *>(smem + L::OFF_KEYS);
    float *red_s = reinterpret_cast<float *>(smem + L::OFF_RED);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == ATC_MMA_WARP) {
        tc::tmem_alloc(tmem_slot, 64);   // S^T x2 (cols 0-31), O^T (cols 32-47)
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < ATC_STAGES; ++i) {
            // keys (and, with cp.async, copies) of a stage: every producer
            // thread arrives once for its keys_s entry and once more for its
            // copies; with TMA block loads the bytes complete tma_full instead
            tc::mbar_init(kv_full + i, (TMA ? 1 : 2) * ATC_PRODUCERS);
            tc::mbar_init(kv_empty + i, 1);
            tc::mbar_init(tma_full + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(q_full + i, 1); tc::mbar_init(q_empty + i, 1);
            tc::mbar_init(s_full + i, 1); tc::mbar_init(s_free + i, 128);
            tc::mbar_init(p_full + i, 128); tc::mbar_init(pv_done + i, 1);
        }
        tc::mbar_init(o_full, 1); tc::mbar_init(o_free, 128); tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const int per = p.per_split;
    auto n_tiles_of = [&](int s) -> int {
        const int e_beg = s * per;
        const int e_end = min(p.entries, e_beg + per);
        return e_end > e_beg ? (e_end - e_beg + ATC_KEYS - 1) / ATC_KEYS : 0;
    };
    auto fail = [&]() {
        raise_error(p.err, ERR_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp < ATC_PRODUCERS / 32) {
        // ---------------------------------------------------------- producer
        // List entries are loaded two tiles ahead of the copies that use them
        // (the lists stream from HBM); tiles are walked in this CTA's order
        // with a cursor, so the item decode happens once per item.
        struct Cur { int it, k, nt, b, t, g, s; };
        auto seek = [&](int from, Cur &c) {              // first non-empty item >= from
            for (c.it = from; c.it < ap.n_items; c.it += gridDim.x) {
                atc_item(p, c.it, c.b, c.t, c.g, c.s);
                c.nt = n_tiles_of(c.s);
                if (c.nt > 0) { c.k = 0; return; }
            }
            c.it = -1; c.k = 0; c.nt = 0;
        };
        auto advance = [&](Cur &c) {
            if (c.it < 0) return;
            if (c.k + 1 < c.nt) { ++c.k; return; }
            seek(c.it + (int)gridDim.x, c);
        };
        auto load_raw = [&](const Cur &c) -> int {
            if (c.it < 0) return KEY_NONE;
            const int e_beg = c.s * per, e_end = min(p.entries, e_beg + per);
            return key_raw<SRC>(p, c.b, c.t, c.g, p.q_pos0 + c.t, e_beg + c.k * ATC_KEYS + tid, e_end);
        };
        Cur pf0, pf1;
        seek((int)blockIdx.x, pf0);
        pf1 = pf0;
        advance(pf1);
        int pf_raw0 = load_raw(pf0), pf_raw1 = load_raw(pf1);
        const int hi = lane >> 4, ch = lane & 15;          // row of the pair, 16-byte chunk of the row
        const uint32_t ch_off = (uint32_t)(ch >> 3) * (ATC_KEYS * 128);   // 64-column half
        int tile = 0, qn = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < ap.n_items && ok; it += gridDim.x, ++qn) {
            int b, t, g, s;
            atc_item(p, it, b, t, g, s);
            const int nt = n_tiles_of(s);
            const long long pos = p.q_pos0 + t;
            if (warp == 0) {
                // Q rows of the group (16 rows; rows past the group are unused)
                const int qb = qn & 1;
                if (!__all_sync(0xffffffffu, atc::wait(q_empty + qb, ((qn >> 1) & 1) ^ 1, abort_flag))) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    atc::expect_tx(q_full + qb, L::Q_BYTES);
                    const int qrow = (b * p.Tq + t) * p.Hq + g * p.G;
                    unsigned char *qdst = smem + L::OFF_Q + qb * L::Q_BYTES;
                    atc::load_2d(qdst, &qmap, 0, qrow, q_full + qb);
                    atc::load_2d(qdst + 16 * 128, &qmap, 64, qrow, q_full + qb);
                }
            }
            const int e_beg = s * per;
            const long long row_base = (long long)b * p.Lk * p.Hkv + g;
            for (int k = 0; k < nt; ++k, ++tile) {
                const int st = tile % ATC_STAGES;
                int raw = pf_raw0;
                if (pf0.it != (int)it || pf0.k != k) {          // not expected; load it now
                    Cur c{(int)it, k, nt, b, t, g, s};
                    raw = load_raw(c);
                }
                // advance the prefetch ring: issue the load of the tile two ahead
                pf0 = pf1; pf_raw0 = pf_raw1;
                advance(pf1);
                pf_raw1 = load_raw(pf1);
                const int key = key_finish<SRC>(p, pos, raw, e_beg + k * ATC_KEYS + tid);
                if (!__all_sync(0xffffffffu, atc::wait(kv_empty + st, ((tile / ATC_STAGES) & 1) ^ 1, abort_flag))) {
                    ok = false;
                    break;
                }
                keys_s[st * ATC_KEYS + tid] = key;
                unsigned char *kdst = smem + L::OFF_KV + st * L::STAGE;
                unsigned char *vdst = kdst + L::KV_BYTES;
                if constexpr (TMA) {
                    // the tile's ATC_KEYS / block blocks, each one box load per
                    // 64-column half of K and of V; a slot with no valid block
                    // loads block 0 so that masked rows hold finite values
                    if (tid == 0) {
                        atc::expect_tx(tma_full + st, 2 * L::KV_BYTES);
                        const int32_t *list = p.idx + ((long long)(b * p.Tq + t) * p.Hkv + g) * p.K;
                        for (int i = 0; i < ATC_KEYS / p.block; ++i) {
                            const int e0 = e_beg + k * ATC_KEYS + i * p.block;
                            int blk = e0 < min(p.entries, e_beg + per) ? __ldg(list + e0 / p.block) : -1;
                            if (blk < 0 || (long long)blk * p.block >= p.Lk) blk = 0;
                            const int z = b * p.Lk + blk * p.block;
                            for (int h = 0; h < 2; ++h) {
                                const uint32_t off = (uint32_t)h * (ATC_KEYS * 128) + (uint32_t)(i * p.block) * 128;
                                atc::load_3d(kdst + off, &kmap, h * 64, g, z, tma_full + st);
                                atc::load_3d(vdst + off, &vmap, h * 64, g, z, tma_full + st);
                            }
                        }
                    }
                    atc::arrive(kv_full + st);                       // this thread's keys_s entry
                } else {
                    // this warp's 32 rows, two 256-byte rows per instruction
#pragma unroll 4
                    for (int j = 0; j < 16; ++j) {
                        const int rr = 2 * j + hi;                       // row within the warp's 32
                        const int kk = __shfl_sync(0xffffffffu, key, rr);
                        const int r = warp * 32 + rr;                    // row within the tile
                        const long long grow = row_base + (long long)(kk >= 0 ? kk : 0) * p.Hkv;
                        const uint32_t off = ch_off + (uint32_t)r * 128 + ((uint32_t)((ch & 7) ^ (r & 7)) << 4);
                        cp_async16(kdst + off, p.k + grow * D + ch * 8, kk >= 0 ? 16 : 0);
                        cp_async16(vdst + off, p.v + grow * D + ch * 8, kk >= 0 ? 16 : 0);
                    }
                    // the stage completes once every producer thread has arrived
                    // (releasing its keys_s entry) and the copies of every
                    // producer thread have landed
                    atc::arrive(kv_full + st);
                    atc::arrive_on_copies(kv_full + st);
                }
            }
        }
        cp_async_wait<0>();                                  // nothing of ours is still in flight
        if (TMA && tid == 0) {
            // the block loads of the last stages land before the CTA exits
            for (int i = 0; i < ATC_STAGES && i < tile; ++i) {
                const int ti = tile - 1 - i;
                tc::mbar_wait_bounded(tma_full + ti % ATC_STAGES, (ti / ATC_STAGES) & 1, ATC_WAIT);
            }
        }
        if (!ok && lane == 0) fail();
        if (warp == 0 && lane == 0) {
            for (int i = 0; i < 2 && i < qn; ++i) {
                const int qi = qn - 1 - i;
                tc::mbar_wait_bounded(q_full + (qi & 1), (qi >> 1) & 1, ATC_WAIT);
            }
        }
    } else if (warp == ATC_MMA_WARP) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t ID_S = tc::make_idesc(1, 1, 128, 16);
            constexpr uint32_t ID_O = tc::make_idesc(1, 1, 128, 16) | (1u << 15) | (1u << 16);
            int tile = 0, qn = 0;
            bool ok = true;
            // S^T(tile) = K . Q^T into S buffer tile & 1
            auto issue_s = [&](int tl, int st, int qb) -> bool {
                const int sb = tl & 1;
                if (!atc::wait((TMA ? tma_full : kv_full) + st, (tl / ATC_STAGES) & 1, abort_flag)) return false;
                if (!atc::wait(s_free + sb, ((tl >> 1) & 1) ^ 1, abort_flag)) return false;
                tc::fence_after_sync();
                tc::fence_proxy_async_smem();   // the copied K rows -> tensor-core reads
                const uint32_t ka = tc::smem_u32(smem + L::OFF_KV + st * L::STAGE);
                const uint32_t qa = tc::smem_u32(smem + L::OFF_Q + qb * L::Q_BYTES);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int h = ks / 4, kk = ks % 4;
                    const uint64_t ad = atc::desc_sw128(ka + h * (ATC_KEYS * 128) + kk * 32, 16, 1024);
                    const uint64_t bd = atc::desc_sw128(qa + h * (16 * 128) + kk * 32, 16, 1024);
                    tc::mma_bf16(tmem + sb * 16, ad, bd, ID_S, ks > 0 ? 1u : 0u);
                }
                tc::mma_commit(s_full + sb);
                return true;
            };
            for (int it = blockIdx.x; it < ap.n_items && ok; it += gridDim.x, ++qn) {
                int b, t, g, s;
                atc_item(p, it, b, t, g, s);
                const int nt = n_tiles_of(s);
                const int qb = qn & 1;
                if (!atc::wait(q_full + qb, (qn >> 1) & 1, abort_flag)) { ok = false; break; }
                if (nt > 0 && !issue_s(tile, tile % ATC_STAGES, qb)) { ok = false; break; }
                // the previous item's epilogue must have read O before it is overwritten
                if (nt > 0 && qn > 0 && !atc::wait(o_free, ((qn - 1) & 1), abort_flag)) { ok = false; break; }
                for (int k = 0; k < nt; ++k, ++tile) {
                    const int st = tile % ATC_STAGES, pb = tile & 1;
                    if (k + 1 < nt && !issue_s(tile + 1, (tile + 1) % ATC_STAGES, qb)) { ok = false; break; }
                    if (!atc::wait(p_full + pb, (tile >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t va = tc::smem_u32(smem + L::OFF_KV + st * L::STAGE + L::KV_BYTES);
                    const uint32_t pa = tc::smem_u32(smem + L::OFF_P + pb * L::P_BYTES);
#pragma unroll
                    for (int ks = 0; ks < ATC_KEYS / 16; ++ks) {
                        // V tile: MN-major, 64-column atoms 16 KB apart, 8-key groups 1 KB apart
                        const uint64_t ad = atc::desc_sw128(va + ks * 2048, ATC_KEYS * 128, 1024);
                        // P tile: MN-major without swizzle, 8-key core matrices 128 B apart,
                        // head groups 2 KB apart
                        const uint64_t bd = tc::desc_noswizzle(pa + ks * 256, 128, ATC_KEYS * 16);
                        tc::mma_bf16(tmem + 32, ad, bd, ID_O, (k > 0 || ks > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(kv_empty + st);
                    tc::mma_commit(pv_done + pb);
                    if (k + 1 == nt) {
                        tc::mma_commit(o_full);
                    }
                }
                if (!ok) break;
                tc::mma_commit(q_empty + qb);
                if (nt == 0) {
                    // an empty piece still hands its (zero) result to the epilogue
                    tc::mma_commit(o_full);
                }
            }
            if (!ok) fail();
            // every MMA issued here completes before TMEM is released
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, ATC_WAIT);
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- softmax warps
        const int quad = warp & 3;                 // TMEM lane quadrant of this warp
        const int r = quad * 32 + lane;            // key row of S^T / d row of O^T
        const uint32_t lrow = (uint32_t)(quad * 32) << 16;
        const int sw = warp - ATC_MMA_WARP - 1;    // 0..3 within the softmax group
        int tile = 0, qn = 0;
        bool ok = true;      // uniform over the four warps (decided by agree)
        bool bad = false;    // a wait of this thread failed since the last agreement
        for (int it = blockIdx.x; it < ap.n_items && ok; it += gridDim.x, ++qn) {
            int b, t, g, s;
            atc_item(p, it, b, t, g, s);
            const int nt = n_tiles_of(s);
            float m[16], l[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) { m[h] = -INFINITY; l[h] = 0.f; }
            for (int k = 0; k < nt; ++k, ++tile) {
                const int st = tile % ATC_STAGES, sb = tile & 1, pb = tile & 1;
                const bool w = atc::wait(s_full + sb, (tile >> 1) & 1, abort_flag) &&
                               atc::wait(kv_full + st, (tile / ATC_STAGES) & 1, abort_flag);
                if (!atc::agree(1, 128, w && !bad)) { ok = false; break; }
                tc::fence_after_sync();
                uint32_t sr[16];
                tc::tmem_ld16(tmem + lrow + sb * 16, sr);
                tc::tmem_ld_wait();
                tc::fence_before_sync();
                atc::arrive(s_free + sb);
                const bool valid = keys_s[st * ATC_KEYS + r] >= 0;
                float x[16];
                bool need = false;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    x[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
                    need |= x[h] > m[h] + ATC_RAISE;
                }
                // The running max m is only a reference point (softmax does not
                // depend on it) and stays put while no logit exceeds it by more
                // than 2^ATC_RAISE, which fp32 weights and sums absorb.  One vote
                // of the group per tile; the exact tile max (two exchanges
                // through shared memory) only when some logit is above that.
                if (atc::vote_any(1, 128, need)) {
                    int wm[16];
#pragma unroll
                    for (int h = 0; h < 16; ++h) wm[h] = __reduce_max_sync(0xffffffffu, atc::f2ord(x[h]));
                    if (lane == 0) {
#pragma unroll
                        for (int h = 0; h < 16; h += 4)
                            *reinterpret_cast<int4 *>(red_s + sw * 16 + h) = make_int4(wm[h], wm[h + 1], wm[h + 2], wm[h + 3]);
                    }
                    atc::named_sync(1, 128);
                    if (sw == 0 && lane < 16) {
                        const int* ri = reinterpret_cast<const int *>(red_s);
                        const int v = max(max(ri[lane], ri[16 + lane]), max(ri[32 + lane], ri[48 + lane]));
                        red_s[64 + lane] = atc::ord2f(v);
                    }
                    atc::named_sync(1, 128);
                    float mt[16];
#pragma unroll
                    for (int h = 0; h < 16; h += 4) {
                        const float4 v = *reinterpret_cast<const float4 *>(red_s + 64 + h);
                        mt[h] = v.x; mt[h + 1] = v.y; mt[h + 2] = v.z; mt[h + 3] = v.w;
                    }
                    float alpha[16];
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        const float mn = fmaxf(m[h], mt[h]);
                        alpha[h] = mn == -INFINITY ? 1.f : exp2f(m[h] - mn);
                        m[h] = mn;
                        l[h] *= alpha[h];
                    }
                    if (k > 0) {
                        // rescale O^T (row d = r) once the previous P.V is done
                        const int pt = tile - 1;
                        if (atc::wait(pv_done + (pt & 1), (pt >> 1) & 1, abort_flag)) {
                            tc::fence_after_sync();
                            uint32_t orow[16];
                            tc::tmem_ld16(tmem + lrow + 32, orow);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int h = 0; h < 16; ++h)
                                orow[h] = __float_as_uint(__uint_as_float(orow[h]) * alpha[h]);
                            atc::tmem_st16(tmem + lrow + 32, orow);
                            atc::tmem_st_wait();
                        } else {
                            bad = true;
                        }
                    }
                }
                uint32_t pk[8];
#pragma unroll
                for (int h = 0; h < 16; h += 2) {
                    const float mu0 = m[h] == -INFINITY ? 0.f : m[h];
                    const float mu1 = m[h + 1] == -INFINITY ? 0.f : m[h + 1];
                    const float p0 = exp2f(x[h] - mu0), p1 = exp2f(x[h + 1] - mu1);
                    l[h] += p0;
                    l[h + 1] += p1;
                    pk[h / 2] = pack_bf16(p0, p1);
                }
                // P buffer pb was last read by the P.V of tile - 2
                if (tile >= 2 && !atc::wait(pv_done + pb, ((tile >> 1) & 1) ^ 1, abort_flag)) bad = true;
                if (!bad) {
                    unsigned char *pd = smem + L::OFF_P + pb * L::P_BYTES;
                    *reinterpret_cast<uint4 *>(pd + r * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4 *>(pd + ATC_KEYS * 16 + r * 16) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    tc::fence_proxy_async_smem();
                    tc::fence_before_sync();
                    atc::arrive(p_full + pb);
                }
            }
            if (!ok) break;
            // ------------------------------------------------------ epilogue
            // per-head sums over the 128 key rows
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                float v = l[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                l[h] = v;
            }
            float *red_l = red_s + 128;
            // also orders this item's writes after the previous item's readers
            if (!atc::agree(1, 128, !bad)) { ok = false; break; }
            if (lane == 0) {
#pragma unroll
                for (int h = 0; h < 16; h += 4)
                    *reinterpret_cast<float4 *>(red_l + sw * 16 + h) = make_float4(l[h], l[h + 1], l[h + 2], l[h + 3]);
            }
            atc::named_sync(1, 128);
#pragma unroll
            for (int h = 0; h < 16; ++h) l[h] = red_l[h] + red_l[16 + h] + red_l[32 + h] + red_l[48 + h];
            uint32_t orow[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) orow[h] = 0u;
            if (atc::wait(o_full, qn & 1, abort_flag)) {
                if (nt > 0) {
                    tc::fence_after_sync();
                    tc::tmem_ld16(tmem + lrow + 32, orow);
                    tc::tmem_ld_wait();
                }
            } else {
                bad = true;
            }
            tc::fence_before_sync();
            atc::arrive(o_free);
            const long long orow0 = (long long)(b * p.Tq + t) * p.Hq + g * p.G;   // output row of head 0
            const long long rows = (long long)p.B * p.Tq * p.Hq;
            if (p.n_split == 1) {
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    if (h < p.G) {
                        const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
                        const float o = __uint_as_float(orow[h]) * inv;
                        if (p.out_f32) p.out_f32[(orow0 + h) * D + r] = o;
                        else p.out[(orow0 + h) * D + r] = __float2bfloat16_rn(o);
                    }
                }
                if (p.lse && r < p.G) {
                    float lv = 0.f, mv = 0.f;
#pragma unroll
                    for (int h = 0; h < 16; ++h) if (h == r) { lv = l[h]; mv = m[h]; }
                    p.lse[orow0 + r] = lv > 0.f ? (mv + log2f(lv)) * kLn2 : -INFINITY;
                }
            } else {
                float *po = p.part_o + (long long)s * rows * D;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    if (h < p.G) {
                        const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
                        po[(orow0 + h) * D + r] = __uint_as_float(orow[h]) * inv;
                    }
                }
                if (r < p.G) {
                    float lv = 0.f, mv = 0.f;
#pragma unroll
                    for (int h = 0; h < 16; ++h) if (h == r) { lv = l[h]; mv = m[h]; }
                    p.part_lse[s * rows + orow0 + r] = lv > 0.f ? (mv + log2f(lv)) * kLn2 : -INFINITY;
                }
            }
        }
        if (!ok || bad) fail();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == ATC_MMA_WARP) tc::tmem_dealloc(tmem, 64);
}

}  // namespace sa
