// Blackwell (sm_100a) tensor-core and bulk-copy helpers of the LAMP attention
// kernels: tcgen05.mma with operands in shared memory and the accumulator in
// tensor memory (TMEM), and TMA tile loads (cp.async.bulk.tensor) that complete
// on an mbarrier. Every form here is single-CTA (cta_group::1) and loads only
// this GPU's own memory; nothing is multicast.
//
// P.V is the one dense contraction of the method ("LAMP: Look-Ahead
// Mixed-Precision Inference of Large Language Models", technical summary,
// gist.science paper 2601.21623, section "Theoretical basis": f = softmax and
// its consumer). The kernels compute it transposed, O^T = V^T P^T:
//   A = V^T  (M = head dimension, K = keys): the V tile exactly as a TMA load with
//            128-byte swizzle leaves it ([key][64 dims] rows of 128 bytes), which is
//            the MN-major 128-byte-swizzled operand layout;
//   B = P^T  (N = 32: the 16 query rows' bf16 "hi" parts, then their "lo" parts;
//            K = keys), K-major with 128-byte swizzle, written by the softmax pass
//            over the score rows in place (see sw_at / p_at in lamp_ws_common.cuh);
//   D        fp32 in TMEM: lane = head dimension (M = 128), or the 16-lane
//            quarters of the M = 64 shape; column n < 16 holds sum_j P_hi[n][j] V[j],
//            column 16 + n the same with P_lo.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "lamp_device.cuh"

namespace lamp {

// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor (64 bits), 128-byte swizzle:
//   bits  0-13  start address >> 4
//   bits 16-29  leading-dimension byte offset >> 4
//   bits 32-45  stride-dimension byte offset >> 4
//   bits 46-47  descriptor version (1 on sm_100)
//   bits 61-63  layout: 2 = 128-byte swizzle
// K-major operand: rows of 128 bytes, 8-row groups SBO apart (LBO unused).
// MN-major operand: 64-element blocks of the M/N dimension LBO apart, groups of 8
// K rows SBO apart. The swizzle is a function of the address bits, so each
// 8-row atom must start on a 1024-byte boundary; a K step inside an atom moves
// the start address by 32 bytes (16 bf16).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits 4-5 =
// 1), A and B bf16 (bits 7-9 and 10-12 = 1), A MN-major (bit 15), B K-major
// (bit 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// The mbarrier receives one arrival when every tcgen05.mma this thread issued
// before has completed (its shared-memory operands may then be overwritten and
// its TMEM result read).
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// TMEM allocation (whole warp): the base address goes to *slot in shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Ordering of tcgen05 operations against thread synchronisation.
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Generic-proxy shared-memory writes become visible to the tensor core and TMA.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Eight consecutive 32-bit TMEM columns of this warp's 32 lanes (lane i of the
// warp reads TMEM lane base + i); complete after tmem_wait_ld().
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&r)[8]) {
  uint32_t u[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = __uint_as_float(u[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// TMA tile loads. The tensor maps describe a [B*H][n][d] bf16 tensor (this
// GPU's memory); boxes past n read as zero. x, the innermost coordinate, is a
// multiple of 8 elements (16 bytes).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Offset (bytes) that moves a dynamic shared-memory base up to a 1024-byte boundary.
__device__ __forceinline__ uint32_t smem_align1k_pad(const void* base) {
  return (1024u - (smem_u32(base) & 1023u)) & 1023u;
}

}  // namespace lamp
