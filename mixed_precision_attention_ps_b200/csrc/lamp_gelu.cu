// LAMP on an elementwise activation: out = GELU(y), y = scale * x W^T with the
// linear map accumulated in PS(mu), and the outputs whose component-wise
// condition number exceeds tau recomputed in binary32 before the activation.
// LAMP summary (gist.science paper 2601.21623): "Theoretical basis" item 3 (an
// activation has a diagonal Jacobian, so each output's sensitivity is its own
// condition number kappa_j = |y_j f'(y_j) / f(y_j)|) and "Implementation
// strategy" steps 1-3 (low-precision g, look-ahead selection, recompute).
//
// One CTA of 256 threads computes a 64 x (32 NM) tile of outputs over the whole
// K (NM = 4, or 2 when 128-wide tiles would leave SMs idle): warp w owns rows
// 8w .. 8w+7 of the tile, lane l the columns l + 32m (m < NM), so that a ballot
// over a (row, m) is one mask word. Slices of 32 dimensions of
// x and W are staged global -> registers -> shared memory as binary32 (W as
// (w, w) pairs), one slice ahead; a step is packed over two rows: fma.rn.f32x2
// of the exact bf16 products, then the PS(mu) rounding of the pair.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "lamp.h"
#include "lamp_device.cuh"
#include "lamp_kernels.h"
#include "lamp_linear.cuh"

namespace lamp {
namespace {

constexpr int GL_BM = 64, GL_KS = 32, GL_T = 256;
constexpr float kGeluC = 0.7978845608028654f;   // sqrt(2 / pi)
constexpr float kGeluA = 0.044715f;
constexpr double kGeluCd = 0.7978845608028654;  // sqrt(2 / pi) in double
constexpr double kGeluAd = 0.044715;
// |kappa_f32 - kappa| <= 2e-5 (1 + |v|) for the binary32 evaluation below (v the
// term added to 1): inside twice that band the test is taken again in double.
constexpr float kKappaBand = 4e-5f;

template <int NM>
struct GeluSmem {
  float xs[2][GL_KS][GL_BM];   // x slice: [dim][row], so a row pair is one 8-byte word
  u64 ws[2][GL_KS][32 * NM];   // W slice: [dim][col] as (w, w)
};

struct GeluArgs {
  GeluProblem p;
  u64 negc, pow2s;  // the two-instruction rounding's constants, as pairs
  int s;            // 23 - mu
  int num_sms;      // of the device (host side: the tile-width choice)
  long long tile0;  // first tile of this launch, in row-major (row tile, column tile) order
  int ctiles;       // column tiles per row tile at this launch's width
};

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// bf16 bits -> binary32 bits, for the low and high halves of a word
__device__ __forceinline__ uint32_t lo_bits(uint32_t w) { return w << 16; }
__device__ __forceinline__ uint32_t hi_bits(uint32_t w) { return w & 0xFFFF0000u; }

// Largest magnitude and (smallest nonzero magnitude - 1) of the staged values, as
// binary32 bit patterns compared as integers (a zero wraps to 0xFFFFFFFF).
__device__ __forceinline__ void fold(uint32_t& mx, uint32_t& mn, uint32_t bits) {
  const uint32_t a = bits & 0x7FFFFFFFu;
  mx = max(mx, a);
  mn = min(mn, a - 1u);
}

// kappa(y) = |1 + y u'(y) (1 - tanh u)|, u = c (y + a y^3), in double, with the
// operations in the order of the definition (no contraction).
__device__ __noinline__ double kappa_d(float yf) {
  const double y = (double)yf;
  const double y2 = __dmul_rn(y, y);
  const double u = __dmul_rn(kGeluCd, __dadd_rn(y, __dmul_rn(__dmul_rn(kGeluAd, y), y2)));
  const double du = __dmul_rn(kGeluCd, __dadd_rn(1.0, __dmul_rn(__dmul_rn(3.0 * kGeluAd, y), y)));
  const double omt = 2.0 / __dadd_rn(1.0, exp(__dmul_rn(2.0, u)));
  return fabs(__dadd_rn(1.0, __dmul_rn(__dmul_rn(y, du), omt)));
}

// The same in binary32: returns kappa and the term v (kappa = |1 + v|).
__device__ __forceinline__ float kappa_f(float y, float& v) {
  const float y2 = y * y;
  const float u = kGeluC * fmaf(kGeluA * y2, y, y);
  const float du = kGeluC * fmaf(3.f * kGeluA, y2, 1.f);
  const float omt = 2.f / (1.f + expf(2.f * u));
  v = y * du * omt;
  return fabsf(1.f + v);
}

__device__ __forceinline__ float gelu_f(float y) {
  const float u = kGeluC * fmaf(kGeluA * y * y, y, y);
  return 0.5f * y * (1.f + tanhf(u));
}

// The K loop: acc[p][m] accumulates rows (8w + 2p, 8w + 2p + 1) of the tile
// against column lane + 32m, in PS(mu) steps of the given mode, sequentially
// over k. FOLD collects the operands' magnitude range for the rounding test.
template <int MODE, bool FOLD, int NM>
__device__ __forceinline__ void gelu_mainloop(const GeluArgs& A, GeluSmem<NM>& sm, int m0, int n0,
                                              u64 (&acc)[4][NM], uint32_t (&rng)[4]) {
  constexpr int BN = 32 * NM, WL = NM / 2;  // W: each thread stages WL groups of 8 dimensions
  const GeluProblem& p = A.p;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int xr = t & 63, xc = t >> 6;                // x: row xr, dims 8 xc .. 8 xc + 7 of a slice
  const int wc = t % BN, wq = (t / BN) * WL;         // W: col wc, dims 8 wq .. 8 (wq + WL) - 1
  const bool xin = m0 + xr < p.M, win = n0 + wc < p.N;
  const uint16_t* xp = p.x + (size_t)(xin ? m0 + xr : 0) * p.K + 8 * xc;
  const uint16_t* wp = p.W + (size_t)(win ? n0 + wc : 0) * p.K + 8 * wq;
  const int nsl = (p.K + GL_KS - 1) / GL_KS;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
  uint4 rx, rw[WL];
  auto load = [&](int sl) {
    const int k = sl * GL_KS;
    rx = (xin && k + 8 * xc < p.K) ? ldg16(xp + k) : z4;
#pragma unroll
    for (int g = 0; g < WL; ++g) rw[g] = (win && k + 8 * (wq + g) < p.K) ? ldg16(wp + k + 8 * g) : z4;
  };
  auto store = [&](int buf) {
    const uint32_t xw[4] = {rx.x, rx.y, rx.z, rx.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a = lo_bits(xw[j]), b = hi_bits(xw[j]);
      sm.xs[buf][8 * xc + 2 * j][xr] = __uint_as_float(a);
      sm.xs[buf][8 * xc + 2 * j + 1][xr] = __uint_as_float(b);
      if (FOLD) { fold(rng[0], rng[1], a); fold(rng[0], rng[1], b); }
    }
#pragma unroll
    for (int g = 0; g < WL; ++g) {
      const uint32_t ww[4] = {rw[g].x, rw[g].y, rw[g].z, rw[g].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t a = lo_bits(ww[j]), b = hi_bits(ww[j]);
        sm.ws[buf][8 * (wq + g) + 2 * j][wc] = ((u64)a << 32) | a;
        sm.ws[buf][8 * (wq + g) + 2 * j + 1][wc] = ((u64)b << 32) | b;
        if (FOLD) { fold(rng[2], rng[3], a); fold(rng[2], rng[3], b); }
      }
    }
  };
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < NM; ++m) acc[i][m] = 0ull;
  load(0);
  store(0);
  __syncthreads();
  for (int sl = 0; sl < nsl; ++sl) {
    const int buf = sl & 1;
    if (sl + 1 < nsl) load(sl + 1);
#pragma unroll 8
    for (int k = 0; k < GL_KS; ++k) {
      const ulonglong2 xa = *reinterpret_cast<const ulonglong2*>(&sm.xs[buf][k][8 * warp]);
      const ulonglong2 xb = *reinterpret_cast<const ulonglong2*>(&sm.xs[buf][k][8 * warp + 4]);
      const u64 xq[4] = {xa.x, xa.y, xb.x, xb.y};
      u64 wd[NM];
#pragma unroll
      for (int m = 0; m < NM; ++m) wd[m] = sm.ws[buf][k][lane + 32 * m];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < NM; ++m) acc[i][m] = ps_step<MODE>(xq[i], wd[m], acc[i][m], A.negc, A.pow2s, A.s);
    }
    // buf ^ 1 was last read before the barrier that ended the previous slice
    if (sl + 1 < nsl) store(buf ^ 1);
    __syncthreads();
  }
}

// The two-instruction rounding is exact when every partial sum is 0 or a normal
// number below 2^(127 - s): partial sums are multiples of the smallest product
// grid 2^(e_x,min - 7) 2^(e_w,min - 7), and bounded by the growth limit the host
// computes from mu and K.
__device__ __forceinline__ bool gelu_fast_ok(const uint32_t (&r)[4], int emax_sum_limit) {
  const int ex = (int)(r[0] >> 23), ew = (int)(r[2] >> 23);
  if (ex >= 255 || ew >= 255) return false;  // an infinity or NaN: the exact rounding
  if (r[1] == 0xFFFFFFFFu || r[3] == 0xFFFFFFFFu) return true;  // one operand all zero: every product is 0
  const int lx = max((int)((r[1] + 1u) >> 23), 1) - 134, lw = max((int)((r[3] + 1u) >> 23), 1) - 134;
  return (ex - 127) + (ew - 127) <= emax_sum_limit && lx + lw >= -126;
}

// EPI_GELU: the whole LAMP GELU op. EPI_STORE: only the PS(mu) linear map, its
// outputs written to p.ps_out (the first half of the LayerNorm op).
enum { EPI_GELU = 0, EPI_STORE = 1 };

template <int RND, int EPI, int NM>
__global__ void __launch_bounds__(GL_T, NM == 4 ? 2 : 3) gelu_kernel(const GeluArgs A) {
  constexpr int BN = 32 * NM;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GeluSmem<NM>& sm = *reinterpret_cast<GeluSmem<NM>*>(smem_raw);
  __shared__ uint32_t red[GL_T / 32][4];
  __shared__ int fast_sh;
  const GeluProblem& p = A.p;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const long long tile = A.tile0 + blockIdx.x;
  const int n0 = (int)(tile % A.ctiles) * BN, m0 = (int)(tile / A.ctiles) * GL_BM;
  u64 acc[4][NM];
  uint32_t rng[4] = {0u, 0xFFFFFFFFu, 0u, 0xFFFFFFFFu};

  // step 1: the low-precision linear map. The fused forms (the two-instruction
  // rounding for mu <= 10, a fused multiply-add for mu = 23) are taken first and
  // checked against the operands' magnitude range; a tile outside it (products
  // that are not exact in binary32, partial sums outside the rounding's domain)
  // is computed again with one binary32 multiply, add and exact rounding a step.
  if (RND == kRndExact) {
    gelu_mainloop<kStepExact, false, NM>(A, sm, m0, n0, acc, rng);
  } else {
    if (RND == kRndNone) gelu_mainloop<kStepF32, true, NM>(A, sm, m0, n0, acc, rng);
    else gelu_mainloop<kStepFast, true, NM>(A, sm, m0, n0, acc, rng);
    rng[0] = __reduce_max_sync(0xFFFFFFFFu, rng[0]);
    rng[1] = __reduce_min_sync(0xFFFFFFFFu, rng[1]);
    rng[2] = __reduce_max_sync(0xFFFFFFFFu, rng[2]);
    rng[3] = __reduce_min_sync(0xFFFFFFFFu, rng[3]);
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][i] = rng[i];
    }
    __syncthreads();
    if (t == 0) {
      uint32_t r[4] = {0u, 0xFFFFFFFFu, 0u, 0xFFFFFFFFu};
      for (int w = 0; w < GL_T / 32; ++w) {
        r[0] = max(r[0], red[w][0]); r[1] = min(r[1], red[w][1]);
        r[2] = max(r[2], red[w][2]); r[3] = min(r[3], red[w][3]);
      }
      fast_sh = gelu_fast_ok(r, p.emax_sum_limit) ? 1 : 0;
    }
    __syncthreads();
    if (!fast_sh)  // outside the two-instruction rounding's domain: again, exactly
      gelu_mainloop<kStepExact, false, NM>(A, sm, m0, n0, acc, rng);
  }

  // step 2: the condition number of each output, and the selection
  const u64 sc2 = pack2(p.scale, p.scale);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < NM; ++m) acc[i][m] = mul2u(acc[i][m], sc2);
  const int row0 = m0 + 8 * warp;
  if (EPI == EPI_STORE) {
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const int row = row0 + r, col = n0 + lane + 32 * m;
        if (row < p.M && col < p.N)
          p.ps_out[(size_t)row * p.N + col] = (r & 1) ? hi_f(acc[r >> 1][m]) : lo_f(acc[r >> 1][m]);
      }
    return;
  }
  const int nw = (p.N + 31) >> 5;
  uint32_t myword = 0u;  // lane NM r + m keeps the ballot of (row r, column group m)
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int row = row0 + r;
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      const int col = n0 + lane + 32 * m;
      const float y = (r & 1) ? hi_f(acc[r >> 1][m]) : lo_f(acc[r >> 1][m]);
      const bool valid = row < p.M && col < p.N;
      bool sel;
      if (p.variant == LAMP_GIVEN_MASK) {
        sel = valid && ((__ldg(p.mask_in + (size_t)row * nw + (col >> 5)) >> lane) & 1u);
      } else if (!isfinite(y)) {
        sel = valid && p.tau < INFINITY;  // kappa = +inf
      } else {
        float v;
        const float kf = kappa_f(y, v);
        sel = kf > p.tau;
        if (fabsf(kf - p.tau) <= kKappaBand * (1.f + fabsf(v))) sel = kappa_d(y) > (double)p.tau;
        sel = sel && valid;
      }
      const uint32_t b = __ballot_sync(0xFFFFFFFFu, sel);
      if (lane == NM * r + m) myword = b;
      if (valid) {
        const size_t o = (size_t)row * p.N + col;
        if (p.ps_out) p.ps_out[o] = y;
        if (!sel) {  // step 3 for the others: the activation of the low-precision output
          if (p.mixed_out) p.mixed_out[o] = y;
          const float f = gelu_f(y);
          if (p.out_f32) p.out_f32[o] = f;
          p.out[o] = f32_to_bf16_rne(f);
        }
      }
    }
  }
  {
    const int r = lane / NM, m = lane % NM;
    if (p.mask_out && lane < 8 * NM && row0 + r < p.M && (n0 >> 5) + m < nw)
      p.mask_out[(size_t)(row0 + r) * nw + (n0 >> 5) + m] = myword;
  }

  // step 3: recompute the selected outputs in binary32, 32 per round over the warp
  const int cnt = __popc(myword);
  int incl = cnt;  // inclusive scan of the counts over the lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  if (p.nsel_out && lane == 0 && total) atomicAdd(p.nsel_out, (unsigned long long)total);
  for (int base = 0; base < total; base += 32) {
    const int slot = base + lane;
    // the word holding this slot: the first lane whose inclusive count passes it
    int lo = 0, hi = 31;
#pragma unroll
    for (int it = 0; it < 5; ++it) {
      const int mid = (lo + hi) >> 1;
      const int v = __shfl_sync(0xFFFFFFFFu, incl, mid);
      if (v > slot) hi = mid; else lo = mid + 1;
    }
    const int owner = lo;
    const uint32_t word = __shfl_sync(0xFFFFFFFFu, myword, owner);
    const int before = __shfl_sync(0xFFFFFFFFu, incl - cnt, owner);
    if (slot < total) {
      const int c = __fns(word, 0, slot - before + 1);
      const int r = owner / NM, m = owner % NM;
      const int row = row0 + r, col = n0 + c + 32 * m;
      const float s = fp32_dot_bf16<0>(p.x + (size_t)row * p.K, p.W + (size_t)col * p.K, p.K);
      const float y = __fmul_rn(p.scale, s);
      const size_t o = (size_t)row * p.N + col;
      if (p.mixed_out) p.mixed_out[o] = y;
      const float f = gelu_f(y);
      if (p.out_f32) p.out_f32[o] = f;
      p.out[o] = f32_to_bf16_rne(f);
    }
  }
}

template <int RND, int EPI, int NM>
cudaError_t gelu_launch_nm(GeluArgs A, long long t_begin, long long t_end, cudaStream_t st) {
  const size_t smem = sizeof(GeluSmem<NM>);
  cudaError_t e =
      cudaFuncSetAttribute(gelu_kernel<RND, EPI, NM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  A.tile0 = t_begin;
  A.ctiles = (A.p.N + 32 * NM - 1) / (32 * NM);
  gelu_kernel<RND, EPI, NM><<<(unsigned)(t_end - t_begin), GL_T, smem, st>>>(A);
  return cudaGetLastError();
}

// Tile width. The 128-wide tiles run two CTAs per SM, the 64-wide ones three at
// about 8 % less work per output. Whole problems take the narrower tiles when
// they cut the largest per-SM share of the outputs (whole tiles a SM runs, times
// the tile's size) by an eighth or more. Otherwise the 128-wide tiles fill whole
// rounds of 2 x num_sms CTAs and, when a last partial round would be left, its
// outputs go to a second launch of 64-wide tiles, which spreads them over three
// CTAs per SM (the same rows and columns, so the two launches write disjoint
// outputs).
template <int RND, int EPI>
cudaError_t gelu_launch_one(const GeluArgs& A, cudaStream_t st) {
  const long long rt = (A.p.M + GL_BM - 1) / GL_BM;
  const long long c4 = (A.p.N + 127) / 128, c2 = (A.p.N + 63) / 64;
  const long long t4 = rt * c4, t2 = rt * c2;
  const long long share4 = (t4 + A.num_sms - 1) / A.num_sms * 2, share2 = (t2 + A.num_sms - 1) / A.num_sms;
  if (8 * share2 <= 7 * share4) return gelu_launch_nm<RND, EPI, 2>(A, 0, t2, st);
  const long long round4 = 2LL * A.num_sms, full = t4 / round4 * round4, rest = t4 - full;
  if (full > 0 && rest > 0 && rest < round4 && c2 == 2 * c4) {
    cudaError_t e = gelu_launch_nm<RND, EPI, 4>(A, 0, full, st);
    if (e != cudaSuccess) return e;
    return gelu_launch_nm<RND, EPI, 2>(A, 2 * full, t2, st);
  }
  return gelu_launch_nm<RND, EPI, 4>(A, 0, t4, st);
}

template <int EPI>
cudaError_t gelu_launch(const GeluProblem& p, cudaStream_t st) {
  GeluArgs A;
  A.p = p;
  A.s = 23 - p.mu;
  int dev = 0;
  A.num_sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&A.num_sms, cudaDevAttrMultiProcessorCount, dev);
  const float c = -(float)((1 << A.s) - 1), q = (float)(1 << A.s);
  uint32_t cb, qb;
  std::memcpy(&cb, &c, 4);
  std::memcpy(&qb, &q, 4);
  A.negc = ((u64)cb << 32) | cb;
  A.pow2s = ((u64)qb << 32) | qb;
  if (p.mu == 23) return gelu_launch_one<kRndNone, EPI>(A, st);
  if (p.mu <= 10) return gelu_launch_one<kRndFast, EPI>(A, st);
  return gelu_launch_one<kRndExact, EPI>(A, st);
}

}  // namespace

int gelu_max_rows() { return 65535 * GL_BM; }

cudaError_t launch_gelu(const GeluProblem& p, cudaStream_t st) {
  if (p.nsel_out) {
    cudaError_t e = cudaMemsetAsync(p.nsel_out, 0, sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
  }
  return gelu_launch<EPI_GELU>(p, st);
}

cudaError_t launch_linear_ps(const GeluProblem& p, cudaStream_t st) { return gelu_launch<EPI_STORE>(p, st); }

}  // namespace lamp
