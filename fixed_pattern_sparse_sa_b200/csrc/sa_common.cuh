// sa_common.cuh -- device helpers shared by the library's kernels.
#pragma once

#include <type_traits>
#include <utility>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// Bits of the device error word (one word per device, owned by the API
// layer and passed to each kernel as a pointer).
enum : unsigned {
    ERR_BAD_INDEX = 1u,       // index outside [0, L) or after the query position
    ERR_BAD_BLOCK = 2u,       // NSA block id outside the sequence
    ERR_TIMEOUT = 4u,         // a bounded progress wait gave up (see spin_limit)
};

// Spin limit of the kernels' progress waits (a barrier a role waits on before
// it can go on), in SM clocks; the default is about one second.  Set per
// device by sa_debug_set_spin_limit().  Drain waits (letting the kernel's own
// copies and MMAs finish before it frees tensor memory and exits) never use
// it: they keep a fixed long limit, so a short debug limit cannot release
// memory that an operation in flight still writes.
constexpr long long kDefaultSpinCycles = 2000000000LL;
__device__ long long g_sa_spin_cycles = kDefaultSpinCycles;
__device__ __forceinline__ long long spin_limit() {
    return *reinterpret_cast<volatile long long *>(&g_sa_spin_cycles);
}

// Test hook set by sa_debug_inject_stall(): while nonzero, the NSA
// tensor-core branch kernels issue none of their loads, so the first
// progress wait of each CTA (on a barrier that nothing will complete) runs
// out after the spin limit and reports ERR_TIMEOUT.
__device__ int g_sa_debug_stall = 0;
__device__ __forceinline__ bool debug_stall() { return *reinterpret_cast<volatile int *>(&g_sa_debug_stall) != 0; }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 2^x on the special-function unit (the PTX ex2.approx instruction; results
// below the normal range flush to zero, which a softmax weight can ignore).
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Programmatic dependent launch: every kernel starts by waiting for the
// grid launched before it on the stream to complete (its results visible),
// then lets the next grid begin launching.  With the launch attribute set,
// the next kernel's blocks are scheduled while this grid's last blocks run
// and wait here, instead of launching after the stream drains; without it
// both instructions do nothing.  Nothing is read or written before the wait.
__device__ __forceinline__ void grid_dependency_sync() {
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

__device__ __forceinline__ void raise_error(unsigned *err, unsigned bit) {
    if (err) atomicOr(err, bit);
}

// ---------------------------------------------------------------- cp.async --
// 16-byte asynchronous global->shared copy; src_bytes = 0 zero-fills.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes = 16) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
                 "r"(src_bytes));
}
// f(integral_constant<int, 0>), ..., f(integral_constant<int, N-1>): a loop
// whose index is a compile-time constant (for immediate operands).
template <typename F, int... I>
__device__ __forceinline__ void static_for_impl(F &&f, std::integer_sequence<int, I...>) {
    (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F &&f) {
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

// 16-byte copy from gmem + GOFF bytes to shared address s + SOFF (s a 32-bit
// shared address): the offsets are immediates, so copies from one base share
// its registers.
template <int SOFF, int GOFF>
__device__ __forceinline__ void cp_async16_at(uint32_t s, const void *gmem, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0+%3], [%1+%4], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes),
                 "n"(SOFF), "n"(GOFF));
}
// 4-byte asynchronous global->shared copy (cached at all levels).
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}
// the same, zero-filled past src_bytes (0 or 4)
__device__ __forceinline__ void cp_async4_zfill(void *smem, const void *gmem, int src_bytes) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// --------------------------------------------------------------- ldmatrix --
__device__ __forceinline__ void ldsm_x4(unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3,
                                        const void *smem) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(s));
}
// The same two loads from a 32-bit shared-memory address.
__device__ __forceinline__ void ldsm_x4_a(unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3, uint32_t s) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(s));
}
__device__ __forceinline__ void ldsm_x4_ta(unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3, uint32_t s) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(s));
}
__device__ __forceinline__ void ldsm_x4_t(unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3,
                                          const void *smem) {
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(s));
}

// ---------------------------------------------------------------- mma.sync --
// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const unsigned (&a)[4],
                                               unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x32] * B[32x8], int8 inputs, int32 accumulators (exact).
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], unsigned a0, unsigned a1, unsigned a2,
                                             unsigned a3, unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ unsigned pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<unsigned *>(&v);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<unsigned>(b) << 16);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace sa
