// LAMP attention for decode shapes: a few query rows (n_q <= 4 per head) against
// long key rows, split over the keys so that every SM streams K and V.
//
// Method ("LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models",
// technical summary, gist.science paper 2601.21623): section "Implementation
// strategy", steps 1-3; section "Theoretical basis", item 3, softmax bullet (the
// strict test 2 z (1 - z) |y| > tau); section "Experimental results" (PS(mu), the
// relaxed relative-threshold test, the random-selection control). The tests are
// the same as in the whole-row kernels; only the work is split differently.
//
// A row is cut into 512-key chunks, one CTA of 256 threads per (chunk, b, h):
//   1. scores: the chunk's K rows go to shared memory by TMA, 16 dimensions of
//      the 512 keys per load (two boxes of 256 keys x 32 bytes, 32-byte swizzle, so
//      that a thread's two 16-byte reads of a key hit all 32 banks across a
//      quarter warp); a thread computes two keys as one packed pair per PS(mu) step. The low-precision scores go to a scratch buffer (L2
//      resident), with per (row, chunk) statistics: maximum, first argmax and
//      S = sum of exp(y - max) over the chunk's other keys (binary32 expf summed in
//      double).
//   2. selection: the strict test takes the row's maximum, first argmax and
//      S_rest combined exactly from the chunk records (in double); the relaxed
//      test continues the running maximum over 64-key tiles across the chunks
//      before it. Selected keys are recomputed in binary32 (one key per lane,
//      compacted from the ballot words), then the chunk's softmax numerators
//      against its own maximum, their sum, and the partial output sum_j p_j V_j
//      in binary32 (CUDA cores: one row needs no tensor cores).
//   3. combine: the last chunk of a row to finish (a per-row counter) rescales
//      the row's chunk partials to the row maximum, adds them in chunk order and
//      divides by the normaliser.
// Memory traffic is K once, V once and the small scratch: the split keeps HBM
// busy, which bounds this shape. Each CTA asks for its chunk of K (scores) or V
// (selection) towards L2 with one bulk prefetch when it starts.
#include <cfloat>

#include "lamp.h"
#include "lamp_device.cuh"
#include "lamp_kernels.h"
#include "lamp_umma.cuh"

namespace lamp {
namespace {

constexpr int DC_T = 256;            // threads per CTA
constexpr int DC_CK = kDecodeChunk;  // keys per chunk
constexpr int DC_MAXQ = kDecodeMaxQ;

struct DecStat {
  float m;   // chunk maximum of the low-precision scores (-inf if none valid)
  int am;    // its first key (absolute)
  double s;  // sum over the chunk's other valid keys of exp(y - m)
};

struct DecArgs {
  Problem p;
  int n_ch;          // key chunks per row
  float* scores;     // [BH][n_q][n_ch * DC_CK]
  DecStat* cstat;    // [BH][n_q][n_ch]
  float* part;       // [BH][n_q][n_ch][2 + d]
  int* cfast;        // [BH][n_ch]: the chunk's products are exact (the recompute may fuse)
  unsigned* rowdone; // [BH][n_q]: chunks of the row whose partials are written
};

__device__ __forceinline__ int dec_valid(int i, const Problem& p) {
  if (!p.causal) return p.n_k;
  return min(p.n_k, max(0, i + 1 + (p.n_k - p.n_q)));
}

// Block-wide reductions over DC_T threads through a small shared array (fixed
// order, so the results do not depend on timing).
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max_redux(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < DC_T / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}
__device__ __forceinline__ int block_min_i(int v, int* red) {
  v = __reduce_min_sync(0xFFFFFFFFu, v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  int r = red[0];
#pragma unroll
  for (int i = 1; i < DC_T / 32; ++i) r = min(r, red[i]);
  return r;
}
__device__ __forceinline__ double block_sum_d(double v, double* red) {
  v = warp_sum_d(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  double r = red[0];
#pragma unroll
  for (int i = 1; i < DC_T / 32; ++i) r += red[i];
  return r;
}
__device__ __forceinline__ float block_sum_f(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < DC_T / 32; ++i) r += red[i];
  return r;
}

// ---------------------------------------------------------------------------
// 1. Scores and chunk statistics. grid (n_ch, B*H).
// K comes in slices of 16 dimensions of all 512 keys through a ring of DC_NR
// slots, one TMA load of two boxes (keys k0 .. k0 + 255 and k0 + 256 .. + 511, 32
// bytes of each) per slice, completing on the slot's mbarrier. Thread t computes
// keys t and t + 256 for the NQ query rows at once; a slice's 16 values of each Q
// row sit in registers. Keys past the row read as zero from the TMA and are
// replaced by 1.0 (their scores are masked; 1.0 leaves the magnitude test below
// unchanged). The two-instruction rounding is taken optimistically: the largest
// and smallest magnitudes of the chunk's K values are folded on the way (binary32
// max / min of the widened values), and a chunk outside the rounding's domain (or
// holding an exact zero, conservatively) is computed again with the exact rounding.
// ---------------------------------------------------------------------------
constexpr int DC_NR = 4;                           // K slices in the ring
constexpr uint32_t DC_SLICE = DC_CK * 16 * 2;      // bytes of a slice (16 dimensions of 512 keys)

template <int D>
__host__ __device__ constexpr size_t dec_scores_smem() {  // ring, Q rows, 1024-byte alignment slack
  return (size_t)DC_NR * DC_SLICE + (size_t)DC_MAXQ * D * 4 + 1024;
}

__device__ __forceinline__ int f32_exp(float v) { return (int)((__float_as_uint(v) >> 23) & 0xFFu); }

// The rounding-domain test of the exponent-statistics kernel, from the largest
// and smallest nonzero magnitudes of Q and of K (exponent fields).
__device__ __forceinline__ bool dec_fast_ok(float qmax, float qmin, float kmax, float kmin, int emax_sum_limit) {
  if (!(kmin > 0.f) || !(qmin > 0.f)) return false;  // a zero (or NaN): take the exact rounding
  const int s0 = f32_exp(qmax), s2 = f32_exp(kmax);
  if (s0 >= 255 || s2 >= 255) return false;
  const int eq = s0 - 127, ek = s2 - 127;
  const int lq = max(f32_exp(qmin), 1) - 134, lk = max(f32_exp(kmin), 1) - 134;
  return (eq + ek <= emax_sum_limit) && (lq + lk >= -126);
}

// The slices of one pass over the chunk. g counts the slices this CTA has taken
// through the ring (slot g % DC_NR, phase (g / DC_NR) & 1) across passes; ok turns
// false when a wait gave up (the pass then skips the waits that follow).
template <int D, int NQ, int MODE, bool FOLD>
__device__ __forceinline__ void dec_slices(const CUtensorMap* tmK, int bh, int k0, int n_k, const float* sQf,
                                           unsigned char* ring, uint64_t* bars, int& g, u64 (&acc)[NQ],
                                           float& kmax, float& kmin, u64 negc, u64 pow2s, int s, bool& ok) {
  constexpr int NSL = D / 16;
  const int t = threadIdx.x;
  auto issue = [&](int sl) {  // thread 0
    if (sl < NSL) {
      const int gs = g + sl;
      unsigned char* slot = ring + (gs % DC_NR) * DC_SLICE;
      uint64_t* bar = bars + gs % DC_NR;
      mbar_expect_tx(bar, DC_SLICE);
      tma_load_3d(slot, tmK, 16 * sl, k0, bh, bar);
      tma_load_3d(slot + DC_SLICE / 2, tmK, 16 * sl, k0 + DC_T, bh, bar);
    }
  };
  const bool va = k0 + t < n_k, vb = k0 + t + DC_T < n_k;
  const int sw = 16 * ((t >> 2) & 1);  // the 32-byte swizzle: 16-byte half c of row t sits at 16 c ^ sw
  const uint4 one = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
#pragma unroll
  for (int i = 0; i < NQ; ++i) acc[i] = 0ull;
  if (t == 0)
    for (int sl = 0; sl < DC_NR - 1; ++sl) issue(sl);
  for (int sl = 0; sl < NSL; ++sl) {
    const int gs = g + sl;
    if (ok) ok = mbar_wait(bars + gs % DC_NR, (gs / DC_NR) & 1);
    __syncthreads();  // slice sl has landed; every thread is done with slice sl - 1, whose slot is refilled
    if (t == 0) issue(sl + DC_NR - 1);
    const unsigned char* slot = ring + (gs % DC_NR) * DC_SLICE;
    uint4 a0 = *reinterpret_cast<const uint4*>(slot + 32 * t + sw);
    uint4 a1 = *reinterpret_cast<const uint4*>(slot + 32 * t + (16 ^ sw));
    uint4 b0 = *reinterpret_cast<const uint4*>(slot + DC_SLICE / 2 + 32 * t + sw);
    uint4 b1 = *reinterpret_cast<const uint4*>(slot + DC_SLICE / 2 + 32 * t + (16 ^ sw));
    if (!va) a0 = a1 = one;
    if (!vb) b0 = b1 = one;
    const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    float q[NQ][16];
#pragma unroll
    for (int i = 0; i < NQ; ++i)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 f = *reinterpret_cast<const float4*>(sQf + i * D + sl * 16 + 4 * v);
        q[i][4 * v] = f.x; q[i][4 * v + 1] = f.y; q[i][4 * v + 2] = f.z; q[i][4 * v + 3] = f.w;
      }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t xa = (e & 1) ? (wa[e >> 1] & 0xFFFF0000u) : (wa[e >> 1] << 16);
      const uint32_t xb = (e & 1) ? (wb[e >> 1] & 0xFFFF0000u) : (wb[e >> 1] << 16);
      if (FOLD) {
        const float fa = fabsf(__uint_as_float(xa)), fb = fabsf(__uint_as_float(xb));
        kmax = fmaxf(kmax, fmaxf(fa, fb));
        kmin = fminf(kmin, fminf(fa, fb));
      }
      const u64 kp = (u64)xa | ((u64)xb << 32);
#pragma unroll
      for (int i = 0; i < NQ; ++i) acc[i] = ps_step<MODE>(pack2(q[i][e], q[i][e]), kp, acc[i], negc, pow2s, s);
    }
  }
  __syncthreads();  // the ring may be refilled
  g += NSL;
}

template <int D, int RND, int NQ>
__global__ void __launch_bounds__(DC_T) dec_scores_kernel(const DecArgs a, const __grid_constant__ CUtensorMap tmK) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = smem_raw + smem_align1k_pad(smem_raw);
  float* sQf = reinterpret_cast<float*>(ring + DC_NR * DC_SLICE);
  __shared__ __align__(8) uint64_t bars[DC_NR];
  __shared__ float redf[DC_T / 32];
  __shared__ int redi[DC_T / 32];
  __shared__ double redd[DC_T / 32];
  const Problem& p = a.p;
  const int c = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int k0 = c * DC_CK;
  const uint16_t* Kh = p.K + (size_t)bh * p.n_k * D;
  if (t == 0) {  // the whole chunk of K towards L2 at once; the ring then reads it from there
    const int nk = min(DC_CK, p.n_k - k0);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(Kh + (size_t)k0 * D), "r"(nk * D * 2) : "memory");
    for (int i = 0; i < DC_NR; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
  }
  if (c == 0 && t < NQ) a.rowdone[(size_t)bh * NQ + t] = 0;  // the selection kernel counts finished chunks
  if (c == 0 && bh == 0 && t == 0 && p.nsel_out) *p.nsel_out = 0ull;
  // Q rows, binary32, and their largest and smallest magnitudes
  float qmax = 0.f, qmin = INFINITY;
  for (int u = t; u < NQ * D; u += DC_T) {
    const float q = __uint_as_float((uint32_t)p.Q[(size_t)bh * NQ * D + u] << 16);
    sQf[u] = q;
    qmax = fmaxf(qmax, fabsf(q));
    qmin = fminf(qmin, fabsf(q));
  }
  const int s = 23 - p.mu;
  const u64 negc = pack2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const u64 pow2s = pack2((float)(1u << s), (float)(1u << s));
  const u64 scale2 = pack2(p.scale, p.scale);
  u64 acc[NQ];
  float kmax = 0.f, kmin = INFINITY;
  int fast = 0;
  int g = 0;       // slices taken through the ring
  bool ok = true;  // no wait gave up
  __syncthreads();  // the barriers are initialised, Q is in place
  if (RND == kRndExact) {
    dec_slices<D, NQ, kStepExact, false>(&tmK, bh, k0, p.n_k, sQf, ring, bars, g, acc, kmax, kmin, negc, pow2s, s, ok);
  } else {
    dec_slices<D, NQ, RND == kRndFast ? kStepFast : kStepF32, true>(&tmK, bh, k0, p.n_k, sQf, ring, bars, g, acc,
                                                                    kmax, kmin, negc, pow2s, s, ok);
    qmax = block_max(qmax, redf);
    qmin = -block_max(-qmin, redf);
    kmax = block_max(kmax, redf);
    kmin = -block_max(-kmin, redf);
    fast = dec_fast_ok(qmax, qmin, kmax, kmin, p.emax_sum_limit) ? 1 : 0;
    if (!fast)  // outside the two-instruction rounding's domain: the exact rounding
      dec_slices<D, NQ, kStepExact, false>(&tmK, bh, k0, p.n_k, sQf, ring, bars, g, acc, kmax, kmin, negc, pow2s, s,
                                           ok);
  }
  if (!ok && p.status_out) atomicExch(p.status_out, LAMP_ERR_TIMEOUT);
  if (t == 0) a.cfast[(size_t)bh * a.n_ch + c] = fast;
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    const u64 y2 = mul2u(acc[i], scale2);
    const int nv = dec_valid(i, p);
    const float y0 = k0 + t < nv ? lo_f(y2) : -INFINITY;
    const float y1 = k0 + t + DC_T < nv ? hi_f(y2) : -INFINITY;
    const size_t row = (size_t)bh * NQ + i;
    float* yrow = a.scores + row * ((size_t)a.n_ch * DC_CK) + k0;
    yrow[t] = y0;
    yrow[t + DC_T] = y1;
    // chunk statistics: maximum, first argmax, and the sum over the other keys
    const float m = block_max(fmaxf(y0, y1), redf);
    int li = 0x7FFFFFFF;
    if (m > -INFINITY) li = y0 == m ? k0 + t : (y1 == m ? k0 + t + DC_T : 0x7FFFFFFF);
    const int am = block_min_i(li, redi);
    double sl = 0.0;
    if (m > -INFINITY) {
      if (k0 + t != am) sl += (double)expf(__fsub_rn(y0, m));
      if (k0 + t + DC_T != am) sl += (double)expf(__fsub_rn(y1, m));
    }
    const double sc = block_sum_d(sl, redd);
    if (t == 0) {
      DecStat st;
      st.m = m;
      st.am = am;
      st.s = sc;
      a.cstat[row * a.n_ch + c] = st;
    }
  }
}

// ---------------------------------------------------------------------------
// 2. Selection, recompute, chunk softmax and partial P.V. grid (n_ch, B*H).
// Thread t takes keys t and t + 256 of the chunk, so the ballots of warp w are the
// chunk's mask words w and 8 + w.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ float dec_recompute(const float* qf, const uint16_t* krow, float scale, bool fused) {
  float acc = 0.f;
#pragma unroll 4
  for (int kk = 0; kk < D; kk += 8) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(krow + kk));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float k0 = bf16_lo(ws[e]), k1 = bf16_hi(ws[e]);
      if (fused) {
        acc = __fmaf_rn(qf[kk + 2 * e], k0, acc);
        acc = __fmaf_rn(qf[kk + 2 * e + 1], k1, acc);
      } else {
        acc = __fadd_rn(acc, __fmul_rn(qf[kk + 2 * e], k0));
        acc = __fadd_rn(acc, __fmul_rn(qf[kk + 2 * e + 1], k1));
      }
    }
  }
  return __fmul_rn(scale, acc);
}

template <int D, int VAR>
__global__ void __launch_bounds__(DC_T) dec_select_kernel(const DecArgs a) {
  constexpr int G = DC_T / (D / 8);  // key groups of the partial P.V (a thread: 8 value columns)
  __shared__ float ys[DC_CK];        // mixed scores of the chunk (current row)
  __shared__ float ps[DC_CK];        // softmax numerators against the chunk maximum
  __shared__ float qf[D];            // the current row of Q, binary32
  __shared__ float ro[G][D];         // partial outputs of the key groups
  __shared__ float half[16];         // relaxed: maxima of half 64-key tiles
  __shared__ float redf[DC_T / 32];
  __shared__ int redi[DC_T / 32];
  __shared__ double redd[DC_T / 32];
  const Problem& p = a.p;
  const int c = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int k0 = c * DC_CK;
  const int nwords = (p.n_k + 31) >> 5;
  const bool fast = a.cfast[(size_t)bh * a.n_ch + c] != 0;
  const bool refine_ok = VAR != LAMP_GIVEN_MASK && isfinite(p.tau) && p.tau >= 0.f;
  const float band = 8e-6f * p.tau;
  const float tlo = refine_ok ? p.tau - band : INFINITY;
  const float thi = refine_ok ? (p.tau == 0.f ? 1e-30f : p.tau + band) : -INFINITY;
  const uint16_t* Kh = p.K + (size_t)bh * p.n_k * D;
  const uint16_t* Vh = p.V + (size_t)bh * p.n_k * D;
  if (t == 0) {  // the chunk's V rows towards L2 while the selection runs
    const int nk = min(DC_CK, p.n_k - k0);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(Vh + (size_t)k0 * D), "r"(nk * D * 2) : "memory");
  }
  __shared__ float wgt[DC_T];  // combine: chunk weights
  __shared__ int last;
  long long nsel = 0;
  for (int i = 0; i < p.n_q; ++i) {
    const size_t row = (size_t)bh * p.n_q + i;
    const int nv = dec_valid(i, p);
    const DecStat* cs = a.cstat + row * a.n_ch;
    const float* yrow = a.scores + row * ((size_t)a.n_ch * DC_CK) + k0;
    for (int u = t; u < D; u += DC_T)
      qf[u] = __uint_as_float((uint32_t)p.Q[row * D + u] << 16);
    float y[2] = {yrow[t], yrow[t + DC_T]};
    bool sel[2] = {false, false};
    if (VAR == LAMP_STRICT) {
      // the row's maximum, first argmax and S_rest from the chunk records
      float lm = -INFINITY;
      for (int cc = t; cc < a.n_ch; cc += DC_T) lm = fmaxf(lm, cs[cc].m);
      const float m = block_max(lm, redf);
      int li = 0x7FFFFFFF;
      if (m > -INFINITY)
        for (int cc = t; cc < a.n_ch; cc += DC_T)
          if (cs[cc].m == m) li = min(li, cs[cc].am);
      const int am = block_min_i(li, redi);
      double sl = 0.0;
      for (int cc = t; cc < a.n_ch; cc += DC_T) {
        const DecStat st = cs[cc];
        if (st.m > -INFINITY) sl += (st.s + (st.am == am ? 0.0 : 1.0)) * exp((double)st.m - (double)m);
      }
      const double srest = block_sum_d(sl, redd);
      const double Sd = 1.0 + srest;
      const float Sf = (float)Sd, srest_f = (float)srest, c2 = (float)(2.0 / (Sd * Sd));
      const float mL = m * kLog2e;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int g = k0 + t + DC_T * e;
        float ex;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ex) : "f"(fmaf(y[e], kLog2e, -mL)));
        float cr = (fabsf(y[e]) * ex) * (__fsub_rn(Sf, ex) * c2);
        if (g == am) cr = fabsf(y[e]) * (srest_f * c2);  // z = 1 / S, 1 - z = S_rest / S
        sel[e] = cr > p.tau;
        if (cr >= tlo && cr <= thi) {  // close to tau: the test again in double
          const double yd = (double)y[e];
          const double ed = g == am ? 1.0 : exp(yd - (double)m);
          const double z = ed / Sd;
          const double omz = g == am ? srest / Sd : (Sd - ed) / Sd;
          sel[e] = 2.0 * z * omz * fabs(yd) > (double)p.tau;
        }
      }
    } else if (VAR == LAMP_RELAXED) {
      // running maximum over 64-key tiles from key 0: the chunks before this one,
      // then this chunk's tiles in order
      float lm = -INFINITY;
      for (int cc = t; cc < c; cc += DC_T) lm = fmaxf(lm, cs[cc].m);
      const float mprev = block_max(lm, redf);
      const float h0 = warp_max_redux(y[0]), h1 = warp_max_redux(y[1]);
      if (lane == 0) {
        half[w] = h0;
        half[8 + w] = h1;
      }
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tile = 4 * e + (t >> 6);  // 64-key tile of the key within the chunk
        float mt = mprev;
        for (int tt = 0; tt <= tile; ++tt) mt = fmaxf(mt, fmaxf(half[2 * tt], half[2 * tt + 1]));
        float ex;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ex) : "f"(fmaf(y[e], kLog2e, -(mt * kLog2e))));
        const float cr = 2.f * fabsf(y[e]) * ex;
        sel[e] = cr > p.tau;
        if (cr >= tlo && cr <= thi) {
          const double yd = (double)y[e];
          sel[e] = 2.0 * exp(yd - (double)mt) * fabs(yd) > (double)p.tau;
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int g = k0 + t + DC_T * e;
        const uint32_t word = (g >> 5) < nwords ? __ldg(p.mask_in + row * nwords + (g >> 5)) : 0u;
        sel[e] = ((word >> (g & 31)) & 1u) && g < nv;
      }
    }
    // mask words, then the selected keys recomputed one per lane (warp-local)
    const uint32_t b0 = __ballot_sync(0xFFFFFFFFu, sel[0]), b1 = __ballot_sync(0xFFFFFFFFu, sel[1]);
    if (p.mask_out && lane == 0) {
      const int wd0 = (k0 >> 5) + w, wd1 = (k0 >> 5) + 8 + w;
      if (wd0 < nwords) p.mask_out[row * nwords + wd0] = b0;
      if (wd1 < nwords) p.mask_out[row * nwords + wd1] = b1;
    }
    nsel += __popc(b0) + __popc(b1);
    ys[t] = y[0];
    ys[t + DC_T] = y[1];
    __syncthreads();  // q row in shared memory for the recompute
    const int n0 = __popc(b0), tot = n0 + __popc(b1);
    for (int base = 0; base < tot; base += 32) {
      const int e = base + lane;
      if (e < tot) {
        const int kk = e < n0 ? 32 * w + __fns(b0, 0, e + 1) : DC_T + 32 * w + __fns(b1, 0, e - n0 + 1);
        ys[kk] = dec_recompute<D>(qf, Kh + (size_t)(k0 + kk) * D, p.scale, fast);
      }
    }
    __syncthreads();
    const float z0 = ys[t], z1 = ys[t + DC_T];
    if (p.ps_out) {
      if (k0 + t < p.n_k) p.ps_out[row * p.n_k + k0 + t] = y[0];
      if (k0 + t + DC_T < p.n_k) p.ps_out[row * p.n_k + k0 + t + DC_T] = y[1];
    }
    if (p.mixed_out) {
      if (k0 + t < p.n_k) p.mixed_out[row * p.n_k + k0 + t] = z0;
      if (k0 + t + DC_T < p.n_k) p.mixed_out[row * p.n_k + k0 + t + DC_T] = z1;
    }
    // the chunk's softmax numerators against its own maximum, their sum
    const float mc = block_max(fmaxf(z0, z1), redf);
    const float mcL = mc == -INFINITY ? 0.f : mc * kLog2e;
    float p0, p1;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p0) : "f"(fmaf(z0, kLog2e, -mcL)));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p1) : "f"(fmaf(z1, kLog2e, -mcL)));
    ps[t] = p0;
    ps[t + DC_T] = p1;
    const float lc = block_sum_f(p0 + p1, redf);  // its barriers also publish ps
    // partial output: key group gq of thread t takes keys gq, gq + G, ... and the
    // value columns 8 dq .. 8 dq + 7 (one 16-byte load per key)
    {
      const int dq = t % (D / 8), gq = t / (D / 8);
      const int kend = min(DC_CK, nv - k0);
      const uint4* vcol = reinterpret_cast<const uint4*>(Vh + (size_t)k0 * D) + dq;
      float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      auto add = [&](float pj, uint4 v) {
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o[2 * e] = fmaf(pj, bf16_lo(w4[e]), o[2 * e]);
          o[2 * e + 1] = fmaf(pj, bf16_hi(w4[e]), o[2 * e + 1]);
        }
      };
      int j = gq;
      for (; j + 3 * G < kend; j += 4 * G) {  // four 16-byte loads in flight per thread
        uint4 v4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v4[u] = __ldg(vcol + (size_t)(j + u * G) * (D / 8));
#pragma unroll
        for (int u = 0; u < 4; ++u) add(ps[j + u * G], v4[u]);
      }
      for (; j < kend; j += G) add(ps[j], __ldg(vcol + (size_t)j * (D / 8)));
#pragma unroll
      for (int e = 0; e < 8; ++e) ro[gq][8 * dq + e] = o[e];
    }
    __syncthreads();
    float* pr = a.part + (row * a.n_ch + c) * (2 + D);
    for (int u = t; u < D; u += DC_T) {
      float o = ro[0][u];
#pragma unroll
      for (int g = 1; g < G; ++g) o += ro[g][u];
      pr[2 + u] = o;
    }
    if (t == 0) {
      pr[0] = mc;
      pr[1] = lc;
    }
    // the last chunk of the row to finish adds up the row's partials (chunk order)
    __threadfence();
    __syncthreads();
    if (t == 0) last = atomicAdd(a.rowdone + row, 1u) == (unsigned)(a.n_ch - 1);
    __syncthreads();
    if (last) {
      __threadfence();
      const float* p0 = a.part + row * a.n_ch * (2 + D);
      float lm = -INFINITY;
      for (int cc = t; cc < a.n_ch; cc += DC_T) lm = fmaxf(lm, __ldcg(p0 + (size_t)cc * (2 + D)));
      const float m = block_max(lm, redf);
      float l = 0.f, o = 0.f;
      for (int c0 = 0; c0 < a.n_ch; c0 += DC_T) {
        const int nc = min(DC_T, a.n_ch - c0);
        __syncthreads();
        if (t < nc) {
          const float mcc = __ldcg(p0 + (size_t)(c0 + t) * (2 + D));
          wgt[t] = (m == -INFINITY || mcc == -INFINITY) ? 0.f : expf(__fsub_rn(mcc, m));
        }
        __syncthreads();
        if (t < D) {
#pragma unroll 8
          for (int cc = 0; cc < nc; ++cc) {
            const float* q = p0 + (size_t)(c0 + cc) * (2 + D);
            l = fmaf(__ldcg(q + 1), wgt[cc], l);
            o = fmaf(__ldcg(q + 2 + t), wgt[cc], o);
          }
        }
      }
      if (t < D) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float v = o * inv;
        p.out[row * D + t] = f32_to_bf16_rne(v);
        if (p.out_f32) p.out_f32[row * D + t] = v;
        if (t == 0 && p.lse_out) p.lse_out[row] = nv > 0 ? m + logf(l) : -INFINITY;
      }
    }
    __syncthreads();  // shared arrays are reused by the next row
  }
  if (lane == 0 && nsel && p.nsel_out) atomicAdd(p.nsel_out, (unsigned long long)nsel);
}

template <int D, int RND, int NQ>
cudaError_t dec_launch_scores(const DecArgs& a, const CUtensorMap& tmK, dim3 grid, cudaStream_t st) {
  const size_t smem = dec_scores_smem<D>();
  cudaError_t e = cudaFuncSetAttribute(dec_scores_kernel<D, RND, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dec_scores_kernel<D, RND, NQ><<<grid, DC_T, smem, st>>>(a, tmK);
  return cudaGetLastError();
}

template <int D, int RND>
cudaError_t dec_launch_rnd(const DecArgs& a, const CUtensorMap& tmK, dim3 grid, cudaStream_t st) {
  switch (a.p.n_q) {
    case 1: return dec_launch_scores<D, RND, 1>(a, tmK, grid, st);
    case 2: return dec_launch_scores<D, RND, 2>(a, tmK, grid, st);
    case 3: return dec_launch_scores<D, RND, 3>(a, tmK, grid, st);
    default: return dec_launch_scores<D, RND, 4>(a, tmK, grid, st);
  }
}

template <int D>
cudaError_t dec_launch(const DecArgs& a, int rnd, cudaStream_t st) {
  const dim3 grid((unsigned)a.n_ch, (unsigned)(a.p.B * a.p.H));
  // K slices: boxes of 16 dimensions x 256 keys of one (b, h), 32-byte swizzle
  CUtensorMap tmK;
  cudaError_t e = make_tmap_bf16(&tmK, a.p.K, D, a.p.n_k, a.p.B * a.p.H, 16, DC_T, 32);
  if (e != cudaSuccess) return e;
  if (rnd == kRndFast) e = dec_launch_rnd<D, kRndFast>(a, tmK, grid, st);
  else if (rnd == kRndNone) e = dec_launch_rnd<D, kRndNone>(a, tmK, grid, st);
  else e = dec_launch_rnd<D, kRndExact>(a, tmK, grid, st);
  if (e != cudaSuccess) return e;
  if (a.p.variant == LAMP_STRICT) dec_select_kernel<D, LAMP_STRICT><<<grid, DC_T, 0, st>>>(a);
  else if (a.p.variant == LAMP_RELAXED) dec_select_kernel<D, LAMP_RELAXED><<<grid, DC_T, 0, st>>>(a);
  else dec_select_kernel<D, LAMP_GIVEN_MASK><<<grid, DC_T, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const Problem& p, const Workspace& ws, char* base, cudaStream_t st) {
  DecArgs a;
  a.p = p;
  a.n_ch = ws.dec_chunks;
  a.scores = reinterpret_cast<float*>(base + ws.dec_scores);
  a.cstat = reinterpret_cast<DecStat*>(base + ws.dec_stat);
  a.part = reinterpret_cast<float*>(base + ws.dec_part);
  a.cfast = reinterpret_cast<int*>(base + ws.dec_flag);
  a.rowdone = reinterpret_cast<unsigned*>(base + ws.dec_done);
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  return p.d == 64 ? dec_launch<64>(a, rnd, st) : dec_launch<128>(a, rnd, st);
}

}  // namespace lamp
