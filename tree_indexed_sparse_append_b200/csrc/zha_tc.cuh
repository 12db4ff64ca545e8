// Tensor-core building blocks shared by the tcgen05 kernels of libzha (frontier
// scoring and gathered attention): tile geometry, the shared-memory operand
// layout and descriptors, the MMA issue, TMEM loads, mbarriers with bounded
// waits, and the copies that fill shared memory. Internal to the library.
//
// Operand layout: a 128-row tile of bf16 with K = 128 columns is stored K-major
// without swizzle as 8-row x 16-byte core matrices, consecutive along K (128 B
// apart), 8-row groups 2 KB apart; core_offset gives an element's byte offset.
#pragma once

#include <cstdint>

#include "zha_internal.cuh"

namespace zha {
namespace {

constexpr int TC_M = 128;                            // walks per A tile
constexpr int TC_N = 128;                            // columns (node x reference) per B tile
constexpr int TC_K = 128;                            // head dimension
constexpr int TC_PART = TC_N * TC_K * 2;             // bytes of one bf16 part of a B tile
constexpr int TC_BTILE = 3 * TC_PART + TC_N * 4;     // hi, mid, lo, biases
constexpr int TC_ATILE = TC_M * TC_K * 2;
constexpr int TC_MT = 2;                             // A tiles (of 128 walks) per CTA
constexpr int TC_SLOTS = 4;                          // B part slots in shared memory
constexpr int TC_SMEM = TC_MT * TC_ATILE + TC_SLOTS * TC_PART + 256;  // + barriers, TMEM address, flag
constexpr int TC_TMEM_COLS = 512;                    // TC_MT x 2 fp32 accumulators of 128 columns
constexpr int TC_THREADS = 9 * 32;                   // 8 epilogue warps + 1 producer warp
constexpr unsigned long long TC_WAIT_NS = 1000000000ull;  // a wait gives up after 1 s (unless the tree sets less)

// byte offset of element (row, k) in a 128-row K-major tile without swizzle:
// 8-row x 16-byte core matrices, consecutive along K (128 B apart), 8-row groups
// 2 KB apart
__host__ __device__ __forceinline__ int core_offset(int row, int k) {
    return (row >> 3) * 2048 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// shared memory matrix descriptor: K-major, no swizzle, LBO = 128 B (between the
// two K halves of an MMA's 16-element slice), SBO = 2 KB (between 8-row groups),
// descriptor version 1
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(2048 >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// instruction descriptor: D fp32, A and B bf16, both K-major, N = 128, M = 128
constexpr uint32_t TC_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TC_N >> 3) << 17) |
                              ((uint32_t)(TC_M >> 4) << 24);

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// bounded wait (at most limit_ns of %globaltimer); false when it gave up
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, phase)) return true;
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < limit_ns)
        if (mbar_try_wait(bar, phase)) return true;
    return false;
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(TC_IDESC), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// 16-byte global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

}  // namespace
}  // namespace zha
