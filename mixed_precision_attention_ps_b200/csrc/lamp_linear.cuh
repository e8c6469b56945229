// Pieces shared by the linear-map operators (GELU and LayerNorm after a PS(mu)
// linear map): the sequential binary32 recompute of one output.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace lamp {

// The sequential binary32 dot of two bf16 rows of K values (K a multiple of 8,
// rows 16-byte aligned): one binary32 multiply and one add a step, in order.
// Both rows stream through a ring of R 16-byte loads per operand, so that R * 8
// steps of the dependent chain cover the latency of the loads behind them.
// R = 0: a plain loop (the compiler overlaps about four loads), for kernels whose
// other warps hide the latency and whose registers are tight.
template <int R>
__device__ __forceinline__ float fp32_dot_bf16(const uint16_t* a, const uint16_t* b, int K) {
  const uint4* aq = reinterpret_cast<const uint4*>(a);
  const uint4* bq = reinterpret_cast<const uint4*>(b);
  const int n = K >> 3;
  if (R == 0) {
    float s = 0.f;
#pragma unroll 4
    for (int k = 0; k < n; ++k) {
      const uint4 u = __ldg(aq + k), v = __ldg(bq + k);
      const uint32_t uw[4] = {u.x, u.y, u.z, u.w}, vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s = __fadd_rn(s, __fmul_rn(__uint_as_float(uw[j] << 16), __uint_as_float(vw[j] << 16)));
        s = __fadd_rn(s, __fmul_rn(__uint_as_float(uw[j] & 0xFFFF0000u), __uint_as_float(vw[j] & 0xFFFF0000u)));
      }
    }
    return s;
  }
  constexpr int RR = R > 0 ? R : 1;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  uint4 ra[RR], rb[RR];
#pragma unroll
  for (int i = 0; i < RR; ++i) {
    ra[i] = i < n ? __ldg(aq + i) : z;
    rb[i] = i < n ? __ldg(bq + i) : z;
  }
  float s = 0.f;
  for (int base = 0; base < n; base += RR) {
#pragma unroll
    for (int i = 0; i < RR; ++i) {
      if (base + i < n) {
        const uint4 u = ra[i], v = rb[i];
        const int nx = base + i + RR;
        ra[i] = nx < n ? __ldg(aq + nx) : z;
        rb[i] = nx < n ? __ldg(bq + nx) : z;
        const uint32_t uw[4] = {u.x, u.y, u.z, u.w}, vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s = __fadd_rn(s, __fmul_rn(__uint_as_float(uw[j] << 16), __uint_as_float(vw[j] << 16)));
          s = __fadd_rn(s, __fmul_rn(__uint_as_float(uw[j] & 0xFFFF0000u), __uint_as_float(vw[j] & 0xFFFF0000u)));
        }
      }
    }
  }
  return s;
}

}  // namespace lamp
