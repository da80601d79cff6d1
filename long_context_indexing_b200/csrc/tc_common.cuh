// tc_common.cuh -- tcgen05 / TMA wrappers shared by the tensor-core scoring
// kernels over 64-wide bf16 rows (bucket scorer and per-key indexer): a 2-D
// TMA tile load, the 128-byte-swizzled K-major shared-memory descriptor, the
// kind::f16 MMA (bf16 A and B, fp32 accumulators in TMEM), its commit, the
// tcgen05 fences and TMEM loads of 32 or 64 consecutive columns of the
// calling thread's lane.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "ptx.cuh"

namespace lsa {

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(ptx::smem_addr(dst)),
        "l"((uint64_t)map), "r"(ptx::smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

// A tile of 128-byte rows (64 bf16), 128-byte swizzle, 8-row core groups.
__device__ __forceinline__ uint64_t sw128_desc(const void* smem_tile)
{
    const uint64_t a = ptx::smem_addr(smem_tile);
    return ((a >> 4) & 0x3FFFull)   // start address
           | (1ull << 16)           // leading byte offset (unused for 128B-swizzled K-major)
           | (64ull << 32)          // stride byte offset: 8 rows x 128 B = 1024 B
           | (1ull << 46)           // descriptor version (tcgen05)
           | (2ull << 61);          // 128-byte swizzle
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
// K-major, M x N.
__host__ __device__ constexpr uint32_t tc_idesc_bf16(int m, int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     ptx::smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

#define LSA_TMEM_LD32(R, ADDR)                                                                   \
    asm volatile(                                                                                \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "  \
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "  \
        "%28, %29, %30, %31}, [%32];"                                                            \
        : "=r"((R)[0]), "=r"((R)[1]), "=r"((R)[2]), "=r"((R)[3]), "=r"((R)[4]), "=r"((R)[5]),    \
          "=r"((R)[6]), "=r"((R)[7]), "=r"((R)[8]), "=r"((R)[9]), "=r"((R)[10]),                 \
          "=r"((R)[11]), "=r"((R)[12]), "=r"((R)[13]), "=r"((R)[14]), "=r"((R)[15]),             \
          "=r"((R)[16]), "=r"((R)[17]), "=r"((R)[18]), "=r"((R)[19]), "=r"((R)[20]),             \
          "=r"((R)[21]), "=r"((R)[22]), "=r"((R)[23]), "=r"((R)[24]), "=r"((R)[25]),             \
          "=r"((R)[26]), "=r"((R)[27]), "=r"((R)[28]), "=r"((R)[29]), "=r"((R)[30]),             \
          "=r"((R)[31])                                                                          \
        : "r"(ADDR))

// 32 consecutive columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v)
{
    uint32_t r[32];
    LSA_TMEM_LD32(r, taddr);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// Two 32-column loads in flight, one wait: 64 consecutive columns of this
// thread's TMEM lane.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v)
{
    uint32_t r[64];
    LSA_TMEM_LD32(r, taddr);
    LSA_TMEM_LD32(r + 32, taddr + 32u);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 64; ++j) v[j] = __uint_as_float(r[j]);
}

}  // namespace lsa
