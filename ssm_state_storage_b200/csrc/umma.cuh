// umma.cuh -- 5th-generation tensor-core (tcgen05) primitives for sm_100a,
// inline PTX: tensor-memory allocation, shared-memory matrix descriptors,
// the bf16 MMA with an fp32 accumulator in tensor memory, completion through
// an mbarrier, and tensor-memory loads.
//
// Operand layout used here: K-major, no swizzle.  A matrix of R rows and 16
// bf16 columns (one MMA's K) is stored as core matrices of 8 rows x 16 bytes
// (8 rows x 8 bf16, 128 contiguous bytes, rows 16 bytes apart): element
// (r, k) lives at byte
//     (r / 8) * kSBO + (k / 8) * kLBO + (r % 8) * 16 + (k % 8) * 2
// with kLBO = 128 (the two K halves of a core-matrix row pair are adjacent)
// and kSBO = 256 (consecutive 8-row groups).  A K-slab of R rows therefore
// takes R * 32 bytes; further K-slabs follow at multiples of that.
//
// Accumulator layout (M = 128, cta_group::1): row m of D is tensor-memory
// lane m, column n is tensor-memory column base + n (fp32).  A warp may
// access only lanes 32 * (warp % 4) .. + 31.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "pipeline.cuh"

namespace rssm {
namespace umma {

constexpr uint32_t kLBO = 128;  // bytes between the two K halves of a core-matrix pair
constexpr uint32_t kSBO = 256;  // bytes between consecutive 8-row groups

// Byte offset of element (r, k), k < 16, inside one K-slab.
__host__ __device__ __forceinline__ uint32_t kmajor_offset(int r, int k) {
  return (uint32_t)(r >> 3) * kSBO + (uint32_t)(k >> 3) * kLBO + (uint32_t)(r & 7) * 16u +
         (uint32_t)(k & 7) * 2u;
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading
// and stride byte offsets (all >> 4), descriptor version 1 (bits 46-47),
// base offset 0, swizzle mode 0 (none, bits 61-63).
__device__ __forceinline__ uint64_t smem_desc(const void *base) {
  const uint64_t a = (smem_addr(base) >> 4) & 0x3FFFu;
  return a | ((uint64_t)(kLBO >> 4) << 16) | ((uint64_t)(kSBO >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16 with bf16 A and B (both K-major), fp32
// D, dense, no negation: D format bits 4-5 = 1 (F32), A format bits 7-9 = 1
// (BF16), B format bits 10-12 = 1 (BF16), N >> 3 at bits 17-22, M >> 4 at bits
// 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B^T for one K = 16 slab, issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate), "r"(0u), "r"(0u), "r"(0u),
      "r"(0u)
      : "memory");
}

// Arrive once on `bar` when every MMA issued so far by this thread completes.
__device__ __forceinline__ void commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Tensor-memory allocation by one whole warp; the base address is written to
// *slot (shared memory).  ncols: a power of two, 32..512.
__device__ __forceinline__ void alloc(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// 32 consecutive fp32 columns of this thread's lane (warp-collective).
__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Split an fp32 value into three bf16 terms whose sum reproduces it to about
// 2^-24 relative (each term carries the next 8 significant bits of the
// remainder; every subtraction is exact).  Used so that a bf16 MMA of an
// fp32 operand with a bf16 operand keeps fp32 accuracy: each partial product
// of two bf16 values is exact in the fp32 accumulator.
__device__ __forceinline__ void split3_bf16(float v, __nv_bfloat16 &hi, __nv_bfloat16 &mid,
                                            __nv_bfloat16 &lo) {
  hi = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);
  lo = __float2bfloat16_rn(r2);
}

}  // namespace umma
}  // namespace rssm
