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
//   1. scores: the chunk's K rows go to shared memory by cp.async (16-byte pieces
//      swizzled against bank conflicts); a thread computes two keys as one packed
//      pair per PS(mu) step. The low-precision scores go to a scratch buffer (L2
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
//   3. combine: per row, the chunk partials rescaled to the row maximum, summed in
//      chunk order and divided by the normaliser.
// Memory traffic is K once, V once and the small scratch: the split keeps HBM
// busy, which bounds this shape.
#include <cfloat>

#include "lamp.h"
#include "lamp_device.cuh"
#include "lamp_kernels.h"

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
  const int* stats;  // per-(b, h) exponent statistics
  int nchunk;        // their records per head
  int n_ch;          // key chunks per row
  float* scores;     // [BH][n_q][n_ch * DC_CK]
  DecStat* cstat;    // [BH][n_q][n_ch]
  float* part;       // [BH][n_q][n_ch][2 + d]
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
// Shared memory: K chunk [DC_CK keys][D/8 pieces] uint4 (piece c of key j at
// c ^ ((j >> 1) & 7)), then Q as packed pairs {q, q} [n_q][D] u64.
// ---------------------------------------------------------------------------
template <int D>
__host__ __device__ constexpr size_t dec_scores_smem() {
  return (size_t)DC_CK * D * 2 + (size_t)DC_MAXQ * D * 8;
}

template <int D, int RND>
__global__ void __launch_bounds__(DC_T) dec_scores_kernel(const DecArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int NP = D / 8;  // 16-byte pieces per K row
  uint4* sK = reinterpret_cast<uint4*>(smem);
  u64* sQ = reinterpret_cast<u64*>(smem + (size_t)DC_CK * D * 2);
  __shared__ float redf[DC_T / 32];
  __shared__ int redi[DC_T / 32];
  __shared__ double redd[DC_T / 32];
  const Problem& p = a.p;
  const int c = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int k0 = c * DC_CK;
  const uint16_t* Kh = p.K + (size_t)bh * p.n_k * D;
  for (int u = t; u < DC_CK * NP; u += DC_T) {
    const int j = u / NP, pc = u % NP;
    uint4* dst = sK + j * NP + (pc ^ ((j >> 1) & 7));
    if (k0 + j < p.n_k) cp_async16(dst, Kh + (size_t)(k0 + j) * D + pc * 8);
    else *dst = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();
  for (int u = t; u < p.n_q * D; u += DC_T) {
    const int i = u / D, dd = u % D;
    const float q = __uint_as_float((uint32_t)p.Q[((size_t)bh * p.n_q + i) * D + dd] << 16);
    sQ[u] = pack2(q, q);
  }
  const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)bh * a.nchunk * 4, a.nchunk,
                                                        p.emax_sum_limit);
  const int s = 23 - p.mu;
  const u64 negc = pack2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const u64 pow2s = pack2((float)(1u << s), (float)(1u << s));
  const u64 scale2 = pack2(p.scale, p.scale);
  cp_async_wait<0>();
  __syncthreads();
  const int j0 = 2 * t, sw = t & 7;  // keys j0, j0 + 1 of the chunk (same swizzle)
  const uint4* ka = sK + j0 * NP;
  const uint4* kb = sK + (j0 + 1) * NP;
  for (int i = 0; i < p.n_q; ++i) {
    u64 acc = 0ull;
    const u64* qrow = sQ + i * D;
#pragma unroll 2
    for (int pc = 0; pc < NP; ++pc) {
      const uint4 va = ka[pc ^ sw], vb = kb[pc ^ sw];
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t xa = (e & 1) ? (wa[e >> 1] & 0xFFFF0000u) : (wa[e >> 1] << 16);
        const uint32_t xb = (e & 1) ? (wb[e >> 1] & 0xFFFF0000u) : (wb[e >> 1] << 16);
        const u64 kp = (u64)xa | ((u64)xb << 32);
        const u64 q = qrow[pc * 8 + e];
        if (RND == kRndFast && fast) acc = ps_step<kStepFast>(q, kp, acc, negc, pow2s, s);
        else if (RND == kRndNone && fast) acc = ps_step<kStepF32>(q, kp, acc, negc, pow2s, s);
        else acc = ps_step<kStepExact>(q, kp, acc, negc, pow2s, s);
      }
    }
    const u64 y2 = mul2u(acc, scale2);
    const int nv = dec_valid(i, p);
    const float y0 = k0 + j0 < nv ? lo_f(y2) : -INFINITY;
    const float y1 = k0 + j0 + 1 < nv ? hi_f(y2) : -INFINITY;
    const size_t row = (size_t)bh * p.n_q + i;
    *reinterpret_cast<float2*>(a.scores + row * ((size_t)a.n_ch * DC_CK) + k0 + j0) = make_float2(y0, y1);
    // chunk statistics: maximum, first argmax, and the sum over the other keys
    const float lm = fmaxf(y0, y1);
    const float m = block_max(lm, redf);
    int li = 0x7FFFFFFF;
    if (m > -INFINITY) li = y0 == m ? k0 + j0 : (y1 == m ? k0 + j0 + 1 : 0x7FFFFFFF);
    const int am = block_min_i(li, redi);
    double sl = 0.0;
    if (m > -INFINITY) {
      if (k0 + j0 != am) sl += (double)expf(__fsub_rn(y0, m));
      if (k0 + j0 + 1 != am) sl += (double)expf(__fsub_rn(y1, m));
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
__global__ void __launch_bounds__(DC_T) dec_select_kernel(const DecArgs a, int rnd) {
  constexpr int G = DC_T / (D / 2);  // key groups of the partial P.V
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
  const bool fast = (rnd != kRndExact) && head_fast_ok(a.stats + (size_t)bh * a.nchunk * 4, a.nchunk,
                                                        p.emax_sum_limit);
  const bool refine_ok = VAR != LAMP_GIVEN_MASK && isfinite(p.tau) && p.tau >= 0.f;
  const float band = 8e-6f * p.tau;
  const float tlo = refine_ok ? p.tau - band : INFINITY;
  const float thi = refine_ok ? (p.tau == 0.f ? 1e-30f : p.tau + band) : -INFINITY;
  const uint16_t* Kh = p.K + (size_t)bh * p.n_k * D;
  const uint16_t* Vh = p.V + (size_t)bh * p.n_k * D;
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
    // value columns 2 dp, 2 dp + 1
    {
      const int dp = t % (D / 2), gq = t / (D / 2);
      const int kend = min(DC_CK, nv - k0);
      float o0 = 0.f, o1 = 0.f;
      for (int j = gq; j < kend; j += G) {
        const float pj = ps[j];
        if (pj != 0.f) {
          const uint32_t v2 = __ldg(reinterpret_cast<const uint32_t*>(Vh + (size_t)(k0 + j) * D) + dp);
          o0 = fmaf(pj, bf16_lo(v2), o0);
          o1 = fmaf(pj, bf16_hi(v2), o1);
        }
      }
      ro[gq][2 * dp] = o0;
      ro[gq][2 * dp + 1] = o1;
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
    __syncthreads();  // shared arrays are reused by the next row
  }
  if (lane == 0 && nsel && p.nsel_out) atomicAdd(p.nsel_out, (unsigned long long)nsel);
}

// ---------------------------------------------------------------------------
// 3. Combine: per row, the chunk partials rescaled to the row maximum, summed in
// chunk order, divided by the normaliser. grid (B*H*n_q), D threads.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(D) dec_combine_kernel(const DecArgs a) {
  const Problem& p = a.p;
  const size_t row = blockIdx.x;
  const int t = threadIdx.x;
  const float* pr = a.part + row * a.n_ch * (2 + D);
  float m = -INFINITY;
  for (int c = 0; c < a.n_ch; ++c) m = fmaxf(m, pr[(size_t)c * (2 + D)]);
  float l = 0.f, o = 0.f;
  if (m > -INFINITY) {
    for (int c = 0; c < a.n_ch; ++c) {
      const float* q = pr + (size_t)c * (2 + D);
      if (q[0] == -INFINITY) continue;
      const float wgt = expf(__fsub_rn(q[0], m));
      l = fmaf(q[1], wgt, l);
      o = fmaf(q[2 + t], wgt, o);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float v = o * inv;
  p.out[row * D + t] = f32_to_bf16_rne(v);
  if (p.out_f32) p.out_f32[row * D + t] = v;
  if (t == 0 && p.lse_out) {
    const int i = (int)(row % p.n_q);
    p.lse_out[row] = dec_valid(i, p) > 0 ? m + logf(l) : -INFINITY;
  }
}

template <int D>
cudaError_t dec_launch(const DecArgs& a, int rnd, cudaStream_t st) {
  const dim3 grid((unsigned)a.n_ch, (unsigned)(a.p.B * a.p.H));
  const size_t smem1 = dec_scores_smem<D>();
  cudaError_t e;
  if (rnd == kRndFast) {
    e = cudaFuncSetAttribute(dec_scores_kernel<D, kRndFast>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e == cudaSuccess) dec_scores_kernel<D, kRndFast><<<grid, DC_T, smem1, st>>>(a);
  } else if (rnd == kRndNone) {
    e = cudaFuncSetAttribute(dec_scores_kernel<D, kRndNone>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e == cudaSuccess) dec_scores_kernel<D, kRndNone><<<grid, DC_T, smem1, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(dec_scores_kernel<D, kRndExact>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e == cudaSuccess) dec_scores_kernel<D, kRndExact><<<grid, DC_T, smem1, st>>>(a);
  }
  if (e != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.p.variant == LAMP_STRICT) dec_select_kernel<D, LAMP_STRICT><<<grid, DC_T, 0, st>>>(a, rnd);
  else if (a.p.variant == LAMP_RELAXED) dec_select_kernel<D, LAMP_RELAXED><<<grid, DC_T, 0, st>>>(a, rnd);
  else dec_select_kernel<D, LAMP_GIVEN_MASK><<<grid, DC_T, 0, st>>>(a, rnd);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dec_combine_kernel<D><<<(unsigned)(a.p.B * a.p.H * a.p.n_q), D, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const Problem& p, const Workspace& ws, char* base, cudaStream_t st) {
  DecArgs a;
  a.p = p;
  a.stats = reinterpret_cast<const int*>(base + ws.stats);
  a.nchunk = ws.nchunk;
  a.n_ch = ws.dec_chunks;
  a.scores = reinterpret_cast<float*>(base + ws.dec_scores);
  a.cstat = reinterpret_cast<DecStat*>(base + ws.dec_stat);
  a.part = reinterpret_cast<float*>(base + ws.dec_part);
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  return p.d == 64 ? dec_launch<64>(a, rnd, st) : dec_launch<128>(a, rnd, st);
}

}  // namespace lamp
