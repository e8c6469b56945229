// Preparation kernel and the PS(mu) rounding utility kernel.
//
// The preparation kernel runs before every attention launch on the same stream:
//   - it writes, per (b, h) and per chunk of that head's rows, the exponent
//     statistics the score kernels use to decide whether the two-instruction
//     PS(mu) rounding is exact for every partial sum of that head;
//   - it resets the persistent kernels' work counters and the caller's
//     selected-count word.
// Reading Q and K once costs far less than one pass of the score emulation.
#include "lamp_device.cuh"
#include "lamp_kernels.h"

namespace lamp {
namespace {

constexpr int kPrepThreads = 256;

// Fold the exponent statistics of 8 bf16 values (one uint4) into the running maxima.
__device__ __forceinline__ void fold8(uint4 w, int& emax, int& lsbinv) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t b = (words[i] >> (16 * h)) & 0xFFFFu;
      int e = (int)((b >> 7) & 0xFFu);
      emax = max(emax, e);
      if (b & 0x7FFFu) lsbinv = max(lsbinv, 255 - max(e, 1));
    }
  }
}

// grid: (nchunk, B*H). Block (c, bh) covers rows [c*rq, (c+1)*rq) of Q and of K of head bh.
__global__ void __launch_bounds__(kPrepThreads) prep_kernel(const uint16_t* __restrict__ Q,
                                                            const uint16_t* __restrict__ K, int n_q,
                                                            int n_k, int d, int nchunk, int* stats,
                                                            uint32_t* counters,
                                                            unsigned long long* nsel_out) {
  const int c = blockIdx.x, bh = blockIdx.y;
  if (c == 0 && bh == 0 && threadIdx.x < 4) counters[threadIdx.x] = 0u;
  if (c == 0 && bh == 0 && threadIdx.x == 0 && nsel_out) *nsel_out = 0ull;
  int st[4] = {0, 0, 0, 0};
  const int vec_per_row = d / 8;
  // Q
  {
    const int rq = (n_q + nchunk - 1) / nchunk;
    const int r0 = c * rq, r1 = min(n_q, r0 + rq);
    const uint4* base = reinterpret_cast<const uint4*>(Q + (size_t)bh * n_q * d);
    for (long long v = (long long)r0 * vec_per_row + threadIdx.x; v < (long long)r1 * vec_per_row;
         v += kPrepThreads)
      fold8(__ldg(base + v), st[0], st[1]);
  }
  // K
  {
    const int rk = (n_k + nchunk - 1) / nchunk;
    const int r0 = c * rk, r1 = min(n_k, r0 + rk);
    const uint4* base = reinterpret_cast<const uint4*>(K + (size_t)bh * n_k * d);
    for (long long v = (long long)r0 * vec_per_row + threadIdx.x; v < (long long)r1 * vec_per_row;
         v += kPrepThreads)
      fold8(__ldg(base + v), st[2], st[3]);
  }
  __shared__ int red[kPrepThreads / 32][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int v = st[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5][i] = v;
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    int v = 0;
    for (int w = 0; w < kPrepThreads / 32; ++w) v = max(v, red[w][threadIdx.x]);
    stats[((size_t)bh * nchunk + c) * 4 + threadIdx.x] = v;
  }
}

__global__ void ps_round_kernel(const float* __restrict__ x, float* __restrict__ y, size_t n, int mu,
                                int path) {
  const int s = 23 - mu;
  const float neg_c = -(float)((1u << s) - 1u);
  const float pow2s = (float)(1u << s);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    float v = x[i];
    y[i] = (path == 1 && s > 0) ? ps_round_fast(v, neg_c, pow2s) : ps_round_exact(v, s);
  }
}

}  // namespace

cudaError_t launch_prep(const Problem& p, const Workspace& ws, char* base, cudaStream_t st) {
  dim3 grid(ws.nchunk, p.B * p.H);
  prep_kernel<<<grid, kPrepThreads, 0, st>>>(p.Q, p.K, p.n_q, p.n_k, p.d, ws.nchunk,
                                             reinterpret_cast<int*>(base + ws.stats),
                                             reinterpret_cast<uint32_t*>(base + ws.counters),
                                             p.nsel_out);
  return cudaGetLastError();
}

cudaError_t launch_ps_round(const float* x, float* y, size_t n, int mu, int path, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  ps_round_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, y, n, mu, path);
  return cudaGetLastError();
}

}  // namespace lamp
