// probe_gather.cuh -- measurement kernel: the L2 -> shared-memory gather
// ceiling that bounds gathered-KV sparse attention.
//
// Gathered attention moves one K row and one V row (256 bytes each at head
// dim 128, bf16) per (query, selected key) from L2 into shared memory, and
// the selected keys of different queries barely overlap, so that movement
// cannot be shared.  This kernel does the movement alone, with no math:
// every CTA streams rows picked by a hash from a buffer (32 MiB = the K and V
// of a 65536-token sequence, resident in L2) into a per-warp ring of
// shared-memory stages, and nothing else.  Its bytes per second are the
// ceiling that gathered attention is measured against.
//   mode 0: 16-byte cp.async copies (a warp moves two 256-byte rows per
//           instruction), commit groups per stage;
//   mode 1: bulk copies (cp.async.bulk, the TMA engine), one 256-byte row per
//           copy, completion on one mbarrier per stage;
//   mode 2: bulk copies of whole 16 KB blocks (64 consecutive 256-byte rows,
//           the K or V tile of one NSA selection block) at random block
//           offsets, one copy per stage.
#pragma once

#include "sa_common.cuh"
#include "tc_common.cuh"

namespace sa {

constexpr int PROBE_ROW = 256;            // bytes per gathered row
constexpr int PROBE_ROWS_PER_STAGE = 16;  // rows per stage (a 16-key K or V chunk)
constexpr int PROBE_BLOCK = 16384;        // bytes per copy in mode 2
template <int MODE>
__host__ __device__ constexpr int probe_stage_bytes() {
    return MODE == 2 ? PROBE_BLOCK : PROBE_ROWS_PER_STAGE * PROBE_ROW;
}

struct ProbeParams {
    const unsigned char *buf;   // n_rows x 256 bytes
    unsigned n_rows;
    int warps, stages, iters;   // per CTA: warps x iters stages of 16 rows
    unsigned *sink;             // one word, keeps the copies observable
    unsigned *err;
};

__device__ __forceinline__ unsigned probe_hash(unsigned x) {
    x ^= x >> 16; x *= 0x7feb352du;
    x ^= x >> 15; x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

// STAGES: ring depth of the cp.async mode (the bulk mode takes p.stages).
template <int MODE, int STAGES>
__global__ void __launch_bounds__(512) probe_gather_kernel(const ProbeParams p) {
    grid_dependency_sync();
    extern __shared__ __align__(1024) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= p.warps) return;
    constexpr int SB = probe_stage_bytes<MODE>();
    unsigned char *ring = smem + (size_t)warp * p.stages * SB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)p.warps * p.stages * SB) + warp * 16;
    const unsigned seed = (blockIdx.x * 64u + warp) * 0x9e3779b9u;
    auto row_of = [&](int it, int r) -> unsigned {
        return probe_hash(seed + (unsigned)it * PROBE_ROWS_PER_STAGE + (unsigned)r) % p.n_rows;
    };
    if constexpr (MODE == 0) {
        const int hi = lane >> 4, ch = lane & 15;          // row of the pair, 16-byte chunk
        for (int it = 0; it < p.iters; ++it) {
            unsigned char *dst = ring + (it % STAGES) * SB;
#pragma unroll
            for (int j = 0; j < PROBE_ROWS_PER_STAGE / 2; ++j) {
                const int r = 2 * j + hi;
                const unsigned row = row_of(it, r);
                cp_async16(dst + r * PROBE_ROW + ch * 16, p.buf + (size_t)row * PROBE_ROW + ch * 16);
            }
            cp_async_commit();
            // keep STAGES - 1 stages in flight: the next stage's buffer is free
            cp_async_wait<STAGES - 1>();
        }
        cp_async_wait<0>();
    } else {
        // one lane per warp issues the bulk copies of a stage; bars[s] counts
        // its bytes
        if (lane == 0)
            for (int s = 0; s < p.stages; ++s) tc::mbar_init(bars + s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        __syncwarp();
        bool ok = true;
        if (lane == 0) {
            int issued = 0;                                // stages whose copies were issued
            for (int it = 0; it < p.iters; ++it) {
                const int s = it % p.stages;
                if (it >= p.stages && ok) {
                    // the stage's previous copies must have landed before reuse
                    ok = tc::mbar_wait_bounded(bars + s, ((it / p.stages) - 1) & 1, spin_limit());
                    if (!ok) raise_error(p.err, ERR_TIMEOUT);
                }
                if (!ok) break;
                unsigned char *dst = ring + s * SB;
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(tc::smem_u32(bars + s)),
                             "r"(SB)
                             : "memory");
                constexpr int NCOPY = MODE == 2 ? 1 : PROBE_ROWS_PER_STAGE;
                constexpr int CB = MODE == 2 ? PROBE_BLOCK : PROBE_ROW;
                const unsigned n_units = MODE == 2 ? p.n_rows / (PROBE_BLOCK / PROBE_ROW) : p.n_rows;
                for (int r = 0; r < NCOPY; ++r) {
                    const unsigned unit = probe_hash(seed + (unsigned)it * PROBE_ROWS_PER_STAGE + (unsigned)r) % n_units;
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                            tc::smem_u32(dst + r * CB)),
                        "l"(p.buf + (size_t)unit * CB), "r"(CB), "r"(tc::smem_u32(bars + s))
                        : "memory");
                }
                ++issued;
            }
            // drain (fixed long limit, also after a timeout): every issued
            // stage completes before the CTA exits
            for (int it = (issued > p.stages ? issued - p.stages : 0); it < issued; ++it)
                tc::mbar_wait_bounded(bars + it % p.stages, (it / p.stages) & 1, kDefaultSpinCycles);
        }
        __syncwarp();
    }
    if (lane == 0 && p.iters > 0) {
        // fold one byte the copies wrote into the sink so they are observable
        const int last = (p.iters - 1) % (MODE == 0 ? STAGES : p.stages);
        atomicAdd(p.sink, (unsigned)ring[(size_t)last * SB]);
    }
}

__host__ __device__ constexpr int probe_smem_bytes(int warps, int stages, int mode) {
    return warps * stages * (mode == 2 ? PROBE_BLOCK : PROBE_ROWS_PER_STAGE * PROBE_ROW) + warps * 16 * 8;
}

}  // namespace sa
