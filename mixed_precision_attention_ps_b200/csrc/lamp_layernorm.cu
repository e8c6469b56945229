// LAMP on LayerNorm after a PS(mu) linear map, the per-row half: the greedy
// selection by sorted magnitude, the binary32 recompute of the selected
// outputs, and LayerNorm of the mixed row.
// LAMP summary (gist.science paper 2601.21623): "Theoretical basis" item 3 (for
// layer normalisation a nearly sparsest recompute set is found greedily by
// sorting the input magnitudes) and "Implementation strategy" steps 2-3.
//
// The bound: LayerNorm's Jacobian is a projection over sigma, so relative errors
// u on the outputs that are not recomputed move the normalised row by at most
// u ||(1 - q) o y||_2 / sigma to first order. The fewest recomputes that bring
// ||(1 - q) o y_hat||_2 / sigma_hat to tau or below are the largest magnitudes
// (equal magnitudes in ascending index order), taken one at a time here.
//
// One warp per row; the row (binary32) and its selection words live in shared
// memory. Row statistics are summed in double.
#include <cuda_runtime.h>

#include <cstdint>

#include "lamp.h"
#include "lamp_device.cuh"
#include "lamp_kernels.h"
#include "lamp_linear.cuh"

namespace lamp {
namespace {

constexpr int LN_WPB = 4;    // rows (warps) per CTA
constexpr int LN_CAND = 512; // candidate list entries per warp

__device__ __forceinline__ u64 warp_max_u64(u64 v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const u64 w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Words of the valid-column mask of a row of N bits (the last word partial).
__device__ __forceinline__ uint32_t full_word(int w, int nw, int N) {
  return (w == nw - 1 && (N & 31)) ? (1u << (N & 31)) - 1u : 0xFFFFFFFFu;
}

__global__ void __launch_bounds__(LN_WPB * 32) ln_rows_kernel(const LnProblem p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * LN_WPB + warp;
  if (row >= p.M) return;  // the kernel has no CTA-wide barrier
  const int N = p.N, nw = (N + 31) >> 5;
  float* yr = reinterpret_cast<float*>(smem_raw) + (size_t)warp * (N + nw + LN_CAND);
  uint32_t* sw = reinterpret_cast<uint32_t*>(yr + N);

  // the low-precision row and its statistics
  const float* src = p.yhat + (size_t)row * N;
  double s1 = 0.0;
#pragma unroll 8
  for (int j = lane; j < N; j += 32) {
    const float v = __ldcg(src + j);
    yr[j] = v;
    s1 += (double)v;
  }
  const double mean_hat = warp_sum_d(s1) / N;
  double s2 = 0.0, sq = 0.0;
  for (int j = lane; j < N; j += 32) {
    const double v = (double)yr[j], dv = v - mean_hat;
    s2 += dv * dv;
    sq += v * v;
  }
  const double sigma_hat = sqrt(warp_sum_d(s2) / N + (double)p.eps);
  double rest = warp_sum_d(sq);

  // step 2: the recompute set
  int k = 0;
  if (p.variant == LAMP_GIVEN_MASK) {
    for (int w = lane; w < nw; w += 32) {
      const uint32_t m = __ldg(p.mask_in + (size_t)row * nw + w) & full_word(w, nw, N);
      sw[w] = m;
      k += __popc(m);
    }
    k = warp_sum_i(k);
  } else if (!(p.tau >= 0.f)) {  // tau < 0: no set meets the bound, so every output
    for (int w = lane; w < nw; w += 32) sw[w] = full_word(w, nw, N);
    k = N;
  } else {
    for (int w = lane; w < nw; w += 32) sw[w] = 0u;
    __syncwarp();
    const double bound = (double)p.tau * sigma_hat;
    auto met = [&]() { return sqrt(fmax(rest, 0.0)) <= bound; };
    // the largest magnitude not yet selected among idx(t), t < n; equal magnitudes:
    // the lowest index. Returns -1 when only zeros are left.
    auto take = [&](auto idx, int n) {
      u64 best = 0ull;
      for (int t = lane; t < n; t += 32) {
        const int j = idx(t);
        if ((sw[j >> 5] >> (j & 31)) & 1u) continue;
        const u64 key = ((u64)(__float_as_uint(yr[j]) & 0x7FFFFFFFu) << 32) | (u64)(0xFFFFFFFFu - (uint32_t)j);
        best = key > best ? key : best;
      }
      best = warp_max_u64(best);
      if ((best >> 32) == 0ull) return -1;  // only zeros: their squares add nothing
      const int j = (int)(0xFFFFFFFFu - (uint32_t)best);
      __syncwarp();
      if (lane == 0) sw[j >> 5] |= 1u << (j & 31);
      __syncwarp();
      const double v = (double)yr[j];
      rest -= v * v;
      ++k;
      return j;
    };
    if (!met()) {
      // Candidates: the outputs at or above the largest magnitude probe t_i whose
      // squares alone carry the mass to remove (with a margin for rounding); the
      // greedy takes the largest first, so it stops inside that set.
      constexpr int NPROBE = 7;
      const double probe[NPROBE] = {4.0, 3.0, 2.5, 2.0, 1.5, 1.0, 0.5};
      const double rms = sqrt(rest / N), need = (rest - bound * bound) * (1.0 + 1e-6);
      double cum[NPROBE];
#pragma unroll
      for (int i = 0; i < NPROBE; ++i) cum[i] = 0.0;
      for (int j = lane; j < N; j += 32) {
        const double v = (double)yr[j], a = fabs(v), q = v * v;
#pragma unroll
        for (int i = 0; i < NPROBE; ++i) cum[i] += a >= probe[i] * rms ? q : 0.0;
      }
      double thr = -1.0;
#pragma unroll
      for (int i = NPROBE - 1; i >= 0; --i)
        if (warp_sum_d(cum[i]) >= need) thr = probe[i] * rms;
      if (thr >= 0.0) {
        int* cand = reinterpret_cast<int*>(sw + nw);
        int nc = 0;
        for (int base = 0; base < N; base += 32) {
          const int j = base + lane;
          const bool c = j < N && fabs((double)yr[j]) >= thr;
          const uint32_t b = __ballot_sync(0xFFFFFFFFu, c);
          if (c) cand[nc + __popc(b & ((1u << lane) - 1u))] = j;
          nc += __popc(b);
          if (nc > LN_CAND - 32) { nc = -1; break; }
        }
        __syncwarp();
        if (nc >= 0)
          while (!met() && take([&](int t) { return cand[t]; }, nc) >= 0) {
          }
      }
    }
    // the whole row, when the candidates did not suffice (or there were too many)
    while (k < N && !met() && take([](int t) { return t; }, N) >= 0) {
    }
  }
  __syncwarp();

  // step 3: recompute the selected outputs in binary32. Their indices are gathered
  // into the candidate list (LN_CAND at a time), then taken 32 per round, one per
  // lane.
  const uint16_t* xr = p.x + (size_t)row * p.K;
  int* list = reinterpret_cast<int*>(sw + nw);
  int w0 = 0, carry = 0;  // words gathered so far; bits of word w0 already listed
  while (w0 < nw) {
    int nl = 0;
    while (w0 < nw && nl + 32 <= LN_CAND) {  // one word per pass, all lanes
      uint32_t word = sw[w0] & ~carry;
      const int c = __popc(word);
      if (nl + c > LN_CAND) {  // the list is full: keep the rest of the word for later
        int keep = LN_CAND - nl;
        uint32_t part = 0u;
        for (uint32_t b = word; keep > 0; --keep) { const uint32_t low = b & (0u - b); part |= low; b ^= low; }
        word = part;
      }
      if ((word >> lane) & 1u) list[nl + __popc(word & ((1u << lane) - 1u))] = w0 * 32 + lane;
      nl += __popc(word);
      carry |= (int)word;
      if ((uint32_t)carry == sw[w0]) { ++w0; carry = 0; }
    }
    __syncwarp();
    for (int base = 0; base < nl; base += 32) {
      if (base + lane < nl) {
        const int j = list[base + lane];
        yr[j] = __fmul_rn(p.scale, fp32_dot_bf16<16>(xr, p.W + (size_t)j * p.K, p.K));
      }
    }
    __syncwarp();
  }
  __syncwarp();

  // LayerNorm of the mixed row
  double t1 = 0.0;
  for (int j = lane; j < N; j += 32) t1 += (double)yr[j];
  const double mean = warp_sum_d(t1) / N;
  double t2 = 0.0;
  for (int j = lane; j < N; j += 32) {
    const double dv = (double)yr[j] - mean;
    t2 += dv * dv;
  }
  const double inv_sigma = 1.0 / sqrt(warp_sum_d(t2) / N + (double)p.eps);
  const size_t o = (size_t)row * N;
  for (int j = lane; j < N; j += 32) {
    const float y = yr[j];
    const float f = (float)(((double)y - mean) * inv_sigma);
    if (p.out_f32) p.out_f32[o + j] = f;
    p.out[o + j] = f32_to_bf16_rne(f);
    if (p.mixed_out) p.mixed_out[o + j] = y;
  }
  if (p.mask_out)
    for (int w = lane; w < nw; w += 32) p.mask_out[(size_t)row * nw + w] = sw[w];
  if (p.nsel_out && lane == 0 && k) atomicAdd(p.nsel_out, (unsigned long long)k);
}

}  // namespace

cudaError_t launch_ln_rows(const LnProblem& p, cudaStream_t st) {
  const int nw = (p.N + 31) >> 5;
  const size_t smem = (size_t)LN_WPB * (p.N + nw + LN_CAND) * 4;
  cudaError_t e = cudaFuncSetAttribute(ln_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ln_rows_kernel<<<(p.M + LN_WPB - 1) / LN_WPB, LN_WPB * 32, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace lamp
