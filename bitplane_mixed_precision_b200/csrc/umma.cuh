// Fifth-generation tensor-core (tcgen05) helpers for sm_100a: tensor-memory
// allocation, shared-memory matrix descriptors, the f16 MMA with an fp32
// accumulator in tensor memory, completion through an mbarrier, and loads of
// accumulator columns back to registers.
//
// Operand layout used throughout (K-major, no swizzle): a matrix of R rows and
// 32 k (one "k-step") of 16-bit elements is stored as 8x8 core matrices of 16
// bytes per row; element (r, k) sits at byte
//     (r % 8) * 16 + (r / 8) * 512 + (k / 8) * 128 + (k % 8) * 2,
// i.e. the four k-groups of a row group are adjacent (leading byte offset 128)
// and row groups follow every 512 bytes (stride byte offset 512). One MMA
// consumes k 0..15 (descriptor at the base) or k 16..31 (base + 256).
#pragma once

#include <cstdint>

#include "pipe.cuh"

namespace pmoe {
namespace umma {

constexpr uint32_t kLBO = 128; // bytes between the two k-groups of one MMA (K direction)
constexpr uint32_t kSBO = 512; // bytes between 8-row groups (M / N direction)

// element (r, k) of a k-step block in the layout above
__host__ __device__ constexpr uint32_t kstep_offset(int r, int k)
{
    return (uint32_t)((r % 8) * 16 + (r / 8) * 512 + (k / 8) * 128 + (k % 8) * 2);
}

// Shared-memory matrix descriptor: start address >> 4 in bits 0-13, leading
// byte offset >> 4 in bits 16-29, stride byte offset >> 4 in bits 32-45,
// descriptor version 1 in bits 46-47, no swizzle (bits 61-63 zero).
__device__ __forceinline__ uint64_t smem_desc(const void *p)
{
    const uint32_t a = pipe::smem_u32(p);
    return (uint64_t)((a >> 4) & 0x3fffu) | ((uint64_t)(kLBO >> 4) << 16) | ((uint64_t)(kSBO >> 4) << 32) |
           (1ull << 46);
}

// The A operand (128 rows, written by threads) uses the 32-byte-swizzled K-major layout instead: per
// MMA K slice kh (16 elements) a 4 KB block of 128 rows x 32 bytes, row r at 32 r, its two 16-byte
// chunks (k 0..7, 8..15 of the slice) swapped on rows with bit 2 set (address bit 4 ^= bit 7). Eight
// lanes that store 8 bytes of 4 consecutive rows then hit 32 distinct banks per half-warp.
__host__ __device__ constexpr uint32_t a_offset_sw32(int r, int k)
{
    return (uint32_t)((k / 16) * 4096 + r * 32 + ((((k % 16) / 8) ^ ((r >> 2) & 1)) << 4) + (k % 8) * 2);
}

// Descriptor of one K slice of that layout (start 256-byte aligned): leading byte offset 16 (unused by
// swizzled K-major layouts), stride byte offset 256 (8 rows x 32 bytes), layout type 6 (32-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw32(const void *p)
{
    const uint32_t a = pipe::smem_u32(p);
    return (uint64_t)((a >> 4) & 0x3fffu) | (1ull << 16) | ((uint64_t)(256 >> 4) << 32) | (1ull << 46) |
           (6ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// f16 (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 in bits
// 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N)
{
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// One warp (all lanes): allocates ncols columns (a power of two >= 32) of
// tensor memory; the address lands in *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(pipe::smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Makes this thread's generic-proxy writes to shared memory visible to the
// tensor cores (async proxy) once a barrier orders them.
__device__ __forceinline__ void fence_smem_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A * B^T, M x N x 16, f16 inputs, fp32 accumulator; accumulate = false overwrites.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        bool accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
                 : "memory");
}

// The mbarrier receives one arrival once every tcgen05 operation this thread issued so far completed.
__device__ __forceinline__ void commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     pipe::smem_u32(bar))
                 : "memory");
}

// 16 consecutive fp32 columns of this thread's tensor-memory lane (the warp reads lanes 32*(warp%4) ..),
// waited for inside the same asm block so that no copy of the destination registers can be made before
// the load has landed.
__device__ __forceinline__ void ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

// The same 16 columns of four accumulators at column offsets 0, d1, 2*d1, 3*d1 (one wait for all four).
__device__ __forceinline__ void ld16x4(uint32_t taddr, uint32_t d1, float (&v)[4][16])
{
    uint32_t r[64];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%64];\n\t"
                 "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%65];\n\t"
                 "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47}, [%66];\n\t"
                 "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%67];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]),
                   "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
                   "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
                   "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
                   "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
                 : "r"(taddr), "r"(taddr + d1), "r"(taddr + 2 * d1), "r"(taddr + 3 * d1)
                 : "memory");
#pragma unroll
    for (int d = 0; d < 4; ++d)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            v[d][i] = __uint_as_float(r[16 * d + i]);
}

// The same 16 columns of two accumulators at column offsets 0 and d1 (one wait for both).
__device__ __forceinline__ void ld16x2(uint32_t taddr, uint32_t d1, float (&v)[2][16])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
                 "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr), "r"(taddr + d1)
                 : "memory");
#pragma unroll
    for (int d = 0; d < 2; ++d)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            v[d][i] = __uint_as_float(r[16 * d + i]);
}

} // namespace umma
} // namespace pmoe
