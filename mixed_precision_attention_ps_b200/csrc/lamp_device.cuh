// Device helpers shared by the LAMP attention kernels (sm_100a).
//
// Method: "LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models"
// (technical summary, gist.science paper 2601.21623). PS(mu) is the simulated
// float of section "Experimental results"; the rounding contract is stated in
// include/lamp.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace lamp {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// Packed binary32 pairs. sm_100 executes fma/mul/add on float pairs as one
// instruction that occupies the FP32 pipe for two lanes' worth of work; one
// issue slot per pair leaves issue bandwidth for loads and bookkeeping while the
// FP32 pipe stays saturated. Each lane of the pair is an ordinary IEEE
// round-to-nearest-even operation.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// ---------------------------------------------------------------------------
// PS(mu) rounding. s = 23 - mu fraction bits are dropped, round to nearest,
// ties to even, binary32 exponent range.
//
// Exact form (any input): on the bit pattern, add half of the dropped range
// minus one plus the lowest kept bit, then clear the dropped bits; a carry
// moves into the exponent (and to infinity past the largest finite value).
// Infinities and NaNs pass through.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ps_round_exact(float x, int s) {
  uint32_t u = __float_as_uint(x);
  if (s == 0 || ((u >> 23) & 0xFFu) == 0xFFu) return x;
  u += ((1u << (s - 1)) - 1u) + ((u >> s) & 1u);
  u &= ~((1u << s) - 1u);
  return __uint_as_float(u);
}

// Two-instruction form (Veltkamp/Dekker-style splitting, T. J. Dekker, "A
// floating-point technique for extending the available precision", Numer.
// Math. 18, 1971): with g = fl(-(2^s - 1) * x), the value fl(2^s * x + g)
// (one fused multiply-add, exact because 2^s * x + g is representable) is x
// rounded to 24 - s significant bits. Ties go to even because, for s >= 2, a
// tie forces the dropped pattern 10..0, so the rounding of g resolves the tie on
// the kept bits alone. Using 2^s - 1 (not 2^s + 1) keeps 2^s * x - x in or
// below the binade of 2^s * x; the lower-binade case only arises for x within
// 2^-s of a power of two, where rounding at twice the resolution agrees as long
// as s >= mu + 2, i.e. mu <= 10. Valid for mu in [1, 10], x = +0, and normal x
// with |x| < 2^(127 - s); checked against the exact form over every binary32
// pattern in that domain. The kernels use it only when the inputs' exponent
// range keeps every partial sum inside the domain.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ps_round_fast(float x, float neg_c, float pow2s) {
  float g = __fmul_rn(x, neg_c);
  return __fmaf_rn(x, pow2s, g);
}

__device__ __forceinline__ float2 ps_round_fast2(float2 x, float2 neg_c, float2 pow2s) {
  return fma2(x, pow2s, mul2(x, neg_c));
}

// ---------------------------------------------------------------------------
// bfloat16 helpers (inputs are raw 16-bit patterns).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);  // quiet NaN
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// P = hi + lo with hi = bf16(P) and lo = bf16(P - hi): two bf16 values that
// carry about 16 significant bits of P into the bf16 tensor-core product.
__device__ __forceinline__ void split_bf16(float p, uint16_t& hi, uint16_t& lo) {
  hi = f32_to_bf16_rne(p);
  float r = __fsub_rn(p, __uint_as_float((uint32_t)hi << 16));
  lo = f32_to_bf16_rne(r);
}

// ---------------------------------------------------------------------------
// Warp reductions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
// Warp-wide maximum of binary32 values in one instruction (redux.sync, sm_100a);
// NaN inputs are ignored, as by fmaxf.
__device__ __forceinline__ float warp_max_redux(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ int warp_min_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Shared-memory addressing and cp.async staging.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

// ---------------------------------------------------------------------------
// Per-(b,h) exponent statistics written by the preparation kernel. All four
// are maxima of non-negative integers so that partial results combine by max:
//   [0] largest exponent field of Q, [1] 255 - smallest "lsb field" of a nonzero
//   Q element (lsb field = max(exponent field, 1); 0 when Q is all zero),
//   [2], [3] the same for K.
// ---------------------------------------------------------------------------
struct HeadStats {
  int v[4];
};

// True when every partial sum of every PS(mu) score of the head stays inside the
// domain of ps_round_fast and every product q_k * k_k is exact in binary32, so
// that fma(q, k, acc) equals fl(acc + fl(q * k)).
//   emax_sum_limit: largest allowed e_q + e_k (unbiased exponents), computed on
//   the host from mu and d (see lamp_api.cu).
__device__ __forceinline__ bool head_fast_ok(const int* partials, int nchunk, int emax_sum_limit) {
  int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
  for (int c = 0; c < nchunk; ++c) {
    s0 = max(s0, partials[4 * c + 0]);
    s1 = max(s1, partials[4 * c + 1]);
    s2 = max(s2, partials[4 * c + 2]);
    s3 = max(s3, partials[4 * c + 3]);
  }
  if (s1 == 0 || s3 == 0) return (s0 < 255 && s2 < 255);  // an all-zero side: every product is +-0
  int eq = s0 - 127, ek = s2 - 127;
  int lq = (255 - s1) - 134, lk = (255 - s3) - 134;  // exponent of the lowest set bit a nonzero value can have
  return (eq + ek <= emax_sum_limit) && (lq + lk >= -126);
}


constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// 64-bit packed pairs of binary32 (low word = first element).
// ---------------------------------------------------------------------------
typedef unsigned long long u64;

__device__ __forceinline__ u64 fma2u(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ u64 mul2u(u64 a, u64 b) {
  u64 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 pack2(float lo, float hi) {
  return (u64)__float_as_uint(lo) | ((u64)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float lo_f(u64 v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f(u64 v) { return __uint_as_float((uint32_t)(v >> 32)); }

enum StepMode { kStepFast = 0, kStepF32 = 1, kStepExact = 2 };

// One accumulation step of a pair of scores.
template <int MODE>
__device__ __forceinline__ u64 ps_step(u64 q, u64 k, u64 acc, u64 negc, u64 pow2s, int s) {
  if (MODE == kStepFast) {
    const u64 x = fma2u(q, k, acc);
    return fma2u(x, pow2s, mul2u(x, negc));
  } else if (MODE == kStepF32) {
    return fma2u(q, k, acc);
  } else {
    const float x0 = __fadd_rn(lo_f(acc), __fmul_rn(lo_f(q), lo_f(k)));
    const float x1 = __fadd_rn(hi_f(acc), __fmul_rn(hi_f(q), hi_f(k)));
    return pack2(ps_round_exact(x0, s), ps_round_exact(x1, s));
  }
}

// P_j stored in place of the score as one 32-bit word: bf16(P) in the low half
// (the "hi" part) and bf16(P - hi) in the high half (the "lo" part), so that a
// tensor-core step over k = 2j, 2j+1 against V row j twice yields (hi + lo) V_j.
__device__ __forceinline__ uint32_t p_pair(float pj) {
  const uint32_t hi = f32_to_bf16_rne(pj);
  const float rest = __fsub_rn(pj, __uint_as_float(hi << 16));
  return hi | ((uint32_t)f32_to_bf16_rne(rest) << 16);
}

__device__ __forceinline__ float exp_fast(float x) {  // 2^(x log2 e), approximate
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * kLog2e));
  return y;
}


// ---------------------------------------------------------------------------
// mbarriers in shared memory and bounded waits. A wait gives up after about two
// seconds of wall time (%globaltimer), so that a protocol error ends the kernel
// with an error status instead of a hang.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// One wait attempt; the thread may sleep in hardware for up to hint_ns while the
// phase is incomplete (it wakes when the phase completes), so waiting warps take
// no issue slots from the working ones.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Wait until the phase with the given parity has completed; false after the limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity, 20000u)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity, 20000u)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Named-barrier helpers for warp groups.
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// OR of a predicate over the n threads of barrier id (all of them wait).
__device__ __forceinline__ int named_or(int id, int n, int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %3, 0;\n\t"
      "bar.red.or.pred q, %1, %2, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(n), "r"(pred)
      : "memory");
  return r;
}

// bf16 pair of P: low half bf16(P), high half bf16(P - bf16(P)).
__device__ __forceinline__ uint32_t p_pair_cvt(float pj) {
  unsigned short h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(pj));
  const float rest = __fsub_rn(pj, __uint_as_float((uint32_t)h << 16));
  uint32_t packed;  // high half bf16(rest), low half bf16(pj)
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(packed) : "f"(rest), "f"(pj));
  return packed;
}
}  // namespace lamp
