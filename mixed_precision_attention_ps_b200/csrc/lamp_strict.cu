// Strict LAMP attention (and the given-mask variant), one fused persistent kernel.
//
// Method ("LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models",
// technical summary, gist.science paper 2601.21623):
//   section "Implementation strategy", steps 1-3, and section "Theoretical
//   basis", item 3 (softmax bullet): y_hat in PS(mu), the strict test
//   2 z (1 - z) |y_hat| > tau on the softmax of the whole low-precision row,
//   FP32 recompute of the selected scores, then softmax and P.V. The strict test
//   needs the whole row of probabilities ("Significance and claims",
//   limitations), so this kernel keeps a block of complete score rows resident.
//
// Work item = (b, h, block of 32 query rows); items are handed out heaviest
// first (causal) through a counter, one CTA per SM. Per item:
//   1. scores: the CTA stages 128-key tiles of K as binary32 pairs in shared
//      memory; warp w owns rows 4w..4w+3 and each lane two key pairs of the tile,
//      so a lane carries 8 packed accumulators. Every step is one packed fma plus
//      the two-instruction PS(mu) rounding (when the head's exponent range
//      allows it; otherwise the exact integer rounding). Rows stay in shared
//      memory (or in an L2-resident global slab when n_k is too long).
//   2. selection: per row (warp-private), max and first argmax, S_rest with a
//      double accumulator, the criterion in binary32 with a double-precision
//      re-evaluation for entries within 8e-6 of tau, ballot into mask words,
//      warp-aggregated compaction of the selected keys and FP32 recompute by
//      full warps.
//   3. softmax of the mixed row; P is written back in place as bf16 hi + lo.
//   4. P.V on tensor cores (mma.sync m16n8k16 bf16, fp32 accumulation), V tiles
//      staged by cp.async; output bf16 (and optional fp32).
#include <cfloat>

#include "lamp_device.cuh"
#include "lamp_kernels.h"

namespace lamp {
namespace {

constexpr int BM = kStrictBM;   // query rows per item
constexpr int NT = kStrictThreads;
constexpr int NW = NT / kWarp;  // 8 warps
constexpr int RPW = BM / NW;    // 4 rows per warp
constexpr int BN = 128;         // keys per score tile (64 pairs)
constexpr int LIST = 64;        // per-warp recompute list capacity
constexpr int VT = 64;          // keys per V tile
constexpr float kBand = 8e-6f;  // relative band around tau re-evaluated in double

struct StrictArgs {
  Problem p;
  const int* stats;
  int nchunk;
  uint32_t* counter;
  float* spill;
  int nkp;
  int rows_on_chip;
  int n_items;
  int n_rb;
};

__host__ __device__ constexpr size_t q_bytes(int D) { return (size_t)BM * D * 8; }
__host__ __device__ constexpr size_t k_bytes(int D) { return (size_t)64 * (D + 2) * 8; }
__host__ __device__ constexpr size_t list_bytes() { return (size_t)NW * LIST * 4; }

enum ScoreMode { kModeFast = 0, kModeF32 = 1, kModeExact = 2 };

// One 128-key (or 64-key, NP = 1) tile of PS scores for the warp's 4 rows.
// sQ4: Q rows as duplicated pairs {q_k, q_k, q_k+1, q_k+1} (float4 per 2 steps);
// sK4: K as key pairs {k_a,k, k_b,k, k_a,k+1, k_b,k+1} (float4 per 2 steps).
template <int D, int NP, int MODE>
__device__ __forceinline__ void score_tile(const float4* __restrict__ sQ4, const float4* __restrict__ sK4,
                                           int lane, int s, float2 neg_c2, float2 pow2s2,
                                           float2 (&acc)[RPW][2]) {
  constexpr int QS = D / 2;        // float4 per Q row
  constexpr int KS = (D + 2) / 2;  // float4 per K pair (padded)
#pragma unroll
  for (int i = 0; i < RPW; ++i)
#pragma unroll
    for (int c = 0; c < 2; ++c) acc[i][c] = make_float2(0.f, 0.f);
#pragma unroll 8
  for (int kk2 = 0; kk2 < D / 2; ++kk2) {
    float4 qv[RPW], kv[NP];
#pragma unroll
    for (int i = 0; i < RPW; ++i) qv[i] = sQ4[i * QS + kk2];
#pragma unroll
    for (int c = 0; c < NP; ++c) kv[c] = sK4[(lane + 32 * c) * KS + kk2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
#pragma unroll
        for (int c = 0; c < NP; ++c) {
          const float2 q2 = h ? make_float2(qv[i].z, qv[i].w) : make_float2(qv[i].x, qv[i].y);
          const float2 k2 = h ? make_float2(kv[c].z, kv[c].w) : make_float2(kv[c].x, kv[c].y);
          if (MODE == kModeFast) {
            const float2 x = fma2(q2, k2, acc[i][c]);
            acc[i][c] = ps_round_fast2(x, neg_c2, pow2s2);
          } else if (MODE == kModeF32) {
            acc[i][c] = fma2(q2, k2, acc[i][c]);
          } else {
            float x0 = __fadd_rn(acc[i][c].x, __fmul_rn(q2.x, k2.x));
            float x1 = __fadd_rn(acc[i][c].y, __fmul_rn(q2.y, k2.y));
            acc[i][c] = make_float2(ps_round_exact(x0, s), ps_round_exact(x1, s));
          }
        }
      }
    }
  }
}

// FP32 recompute of one score: the sequential binary32 sum, then the scale.
template <int D>
__device__ __forceinline__ float recompute_fp32(const float2* __restrict__ qrow,
                                                const uint16_t* __restrict__ krow, float scale,
                                                bool fused) {
  float acc = 0.f;
#pragma unroll
  for (int kk = 0; kk < D; kk += 8) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(krow + kk));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float k0 = bf16_lo(ws[e]), k1 = bf16_hi(ws[e]);
      const float q0 = qrow[kk + 2 * e].x, q1 = qrow[kk + 2 * e + 1].x;
      if (fused) {
        acc = __fmaf_rn(q0, k0, acc);
        acc = __fmaf_rn(q1, k1, acc);
      } else {
        acc = __fadd_rn(acc, __fmul_rn(q0, k0));
        acc = __fadd_rn(acc, __fmul_rn(q1, k1));
      }
    }
  }
  return __fmul_rn(scale, acc);
}

__device__ __forceinline__ int n_valid_keys(int i, const Problem& p) {
  if (!p.causal) return p.n_k;
  return min(p.n_k, max(0, i + 1 + (p.n_k - p.n_q)));
}

template <int D, int RND>
__global__ void __launch_bounds__(NT, 1) strict_kernel(const StrictArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2* sQ = reinterpret_cast<float2*>(smem);
  float2* sK = reinterpret_cast<float2*>(smem + q_bytes(D));
  uint16_t* sV = reinterpret_cast<uint16_t*>(smem + q_bytes(D));  // phase 4 reuses the K area
  int* sList = reinterpret_cast<int*>(smem + q_bytes(D) + k_bytes(D));
  float* sRows = reinterpret_cast<float*>(smem + q_bytes(D) + k_bytes(D) + list_bytes());
  __shared__ int sItem;

  const Problem& p = a.p;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nkp = a.nkp;
  float* S = a.rows_on_chip ? sRows : a.spill + (size_t)blockIdx.x * BM * nkp;
  const int BH = p.B * p.H;
  const int nwords = (p.n_k + 31) >> 5;
  const int s = 23 - p.mu;
  const float2 neg_c2 = make_float2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const float2 pow2s2 = make_float2((float)(1u << s), (float)(1u << s));
  const float2 scale2 = make_float2(p.scale, p.scale);
  const bool given = (p.variant == 2);
  const bool relaxed = (p.variant == 1);
  const bool strict = (p.variant == 0);
  const uint32_t lanemask_lt = (1u << lane) - 1u;
  constexpr int QV = D / 64;   // uint4 per thread for the Q tile
  constexpr int KV = D / 32;   // uint4 per key per thread for a K tile

  for (;;) {
    if (tid == 0) sItem = (int)atomicAdd(a.counter, 1u);
    __syncthreads();
    const int item = sItem;
    if (item >= a.n_items) break;
    const int rb = p.causal ? a.n_rb - 1 - item / BH : item / BH;
    const int bh = item % BH;
    const int i0 = rb * BM;
    const int rows = min(BM, p.n_q - i0);
    const int kv_end = p.causal ? min(p.n_k, max(0, i0 + rows + (p.n_k - p.n_q))) : p.n_k;
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)bh * p.n_k * D;
    const uint16_t* Vh = p.V + (size_t)bh * p.n_k * D;

    // ---- Q rows as duplicated binary32 pairs --------------------------------
    {
      const int r = tid >> 3, seg = (tid & 7) * (D / 8);
      const uint16_t* src = p.Q + ((size_t)bh * p.n_q + i0 + r) * D + seg;
#pragma unroll
      for (int v = 0; v < QV; ++v) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (r < rows) w = __ldg(reinterpret_cast<const uint4*>(src + 8 * v));
        float4* dst = reinterpret_cast<float4*>(sQ + (size_t)r * D + seg + 8 * v);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_float4(bf16_lo(ws[e]), bf16_lo(ws[e]), bf16_hi(ws[e]), bf16_hi(ws[e]));
      }
    }

    // ---- phase 1: PS(mu) scores -----------------------------------------------
    const int ntiles = (kv_end + BN - 1) / BN;
    const int kp = tid >> 2, kseg = (tid & 3) * (D / 4);
    uint4 ra[KV], rbv[KV];
    auto load_k = [&](int t) {
      const int ka = t * BN + 2 * kp;
#pragma unroll
      for (int v = 0; v < KV; ++v) {
        ra[v] = make_uint4(0u, 0u, 0u, 0u);
        rbv[v] = make_uint4(0u, 0u, 0u, 0u);
        if (ka < kv_end) ra[v] = __ldg(reinterpret_cast<const uint4*>(Kh + (size_t)ka * D + kseg + 8 * v));
        if (ka + 1 < kv_end)
          rbv[v] = __ldg(reinterpret_cast<const uint4*>(Kh + (size_t)(ka + 1) * D + kseg + 8 * v));
      }
    };
    auto store_k = [&]() {
#pragma unroll
      for (int v = 0; v < KV; ++v) {
        const uint32_t wa[4] = {ra[v].x, ra[v].y, ra[v].z, ra[v].w};
        const uint32_t wb[4] = {rbv[v].x, rbv[v].y, rbv[v].z, rbv[v].w};
        float4* dst = reinterpret_cast<float4*>(sK + (size_t)kp * (D + 2) + kseg + 8 * v);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_float4(bf16_lo(wa[e]), bf16_lo(wb[e]), bf16_hi(wa[e]), bf16_hi(wb[e]));
      }
    };
    if (ntiles > 0) load_k(0);
    const int r0 = warp * RPW;
    for (int t = 0; t < ntiles; ++t) {
      __syncthreads();
      store_k();
      __syncthreads();
      if (t + 1 < ntiles) load_k(t + 1);
      if (r0 < rows) {
        const int k0 = t * BN;
        const int tile_keys = min(BN, kv_end - k0);
        const float4* q4 = reinterpret_cast<const float4*>(sQ) + (size_t)r0 * (D / 2);
        const float4* k4 = reinterpret_cast<const float4*>(sK);
        float2 acc[RPW][2];
        if (tile_keys > 64) {
          if (RND == kRndFast && fast) score_tile<D, 2, kModeFast>(q4, k4, lane, s, neg_c2, pow2s2, acc);
          else if (RND == kRndNone && fast) score_tile<D, 2, kModeF32>(q4, k4, lane, s, neg_c2, pow2s2, acc);
          else score_tile<D, 2, kModeExact>(q4, k4, lane, s, neg_c2, pow2s2, acc);
        } else {
          if (RND == kRndFast && fast) score_tile<D, 1, kModeFast>(q4, k4, lane, s, neg_c2, pow2s2, acc);
          else if (RND == kRndNone && fast) score_tile<D, 1, kModeF32>(q4, k4, lane, s, neg_c2, pow2s2, acc);
          else score_tile<D, 1, kModeExact>(q4, k4, lane, s, neg_c2, pow2s2, acc);
        }
        const int npairs = tile_keys > 64 ? 2 : 1;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
          const int r = r0 + i;
          if (r >= rows) continue;
          const int nv = n_valid_keys(i0 + r, p);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (c >= npairs) continue;
            const int j = k0 + 2 * (lane + 32 * c);
            float2 y = mul2(acc[i][c], scale2);
            if (j >= nv) y.x = -INFINITY;
            if (j + 1 >= nv) y.y = -INFINITY;
            *reinterpret_cast<float2*>(S + (size_t)r * nkp + j) = y;
          }
        }
      }
    }
    __syncwarp();

    // ---- phases 2 and 3, per row of the warp ---------------------------------
    long long warp_nsel = 0;
    for (int ri = 0; ri < RPW; ++ri) {
      const int r = r0 + ri;
      if (r >= rows) break;
      const int i = i0 + r;
      const int nv = n_valid_keys(i, p);
      float* row = S + (size_t)r * nkp;
      const size_t grow = (size_t)bh * p.n_q + i;
      if (p.ps_out)
        for (int j = lane; j < p.n_k; j += 32) p.ps_out[grow * p.n_k + j] = j < nv ? row[j] : -INFINITY;
      uint32_t* mrow = p.mask_out ? p.mask_out + grow * nwords : nullptr;
      const int nch = (nv + 31) >> 5;
      if (nv == 0) {
        if (mrow)
          for (int w = lane; w < nwords; w += 32) mrow[w] = 0u;
        if (p.mixed_out)
          for (int j = lane; j < p.n_k; j += 32) p.mixed_out[grow * p.n_k + j] = -INFINITY;
        if (p.lse_out && lane == 0) p.lse_out[grow] = -INFINITY;
        // zero P for the tensor-core pass
        uint16_t* rb16 = reinterpret_cast<uint16_t*>(row);
        for (int c = 0; c * 32 < kv_end; ++c) {
          rb16[64 * c + lane] = 0;
          rb16[64 * c + 32 + lane] = 0;
        }
        continue;
      }
      // (a) row maximum and its first index
      float m = -INFINITY;
      int am = 0x7FFFFFFF;
      for (int j = lane; j < nv; j += 32) {
        const float v = row[j];
        if (v > m) { m = v; am = j; }
      }
      {
        const float mw = warp_max(m);
        am = warp_min_i(m == mw ? am : 0x7FFFFFFF);
        m = mw;
        if (am == 0x7FFFFFFF) am = 0;
      }
      // (b) S_rest = sum over j != argmax of exp(y_j - m) (strict only)
      double srest = 0.0;
      if (strict) {
        for (int j = lane; j < nv; j += 32)
          if (j != am) srest += (double)expf(__fsub_rn(row[j], m));
        srest = warp_sum_d(srest);
      }
      const double Sd = 1.0 + srest;
      const float Sf = (float)Sd, srest_f = (float)srest;
      const float invS2 = (float)(1.0 / (Sd * Sd));
      const bool refine_ok = isfinite(p.tau) && p.tau >= 0.f;
      // (c) criterion, mask, compaction and recompute
      int* list = sList + warp * LIST;
      int list_n = 0;
      uint32_t myword = 0u;
      int row_nsel = 0;
      const float2* qrow = sQ + (size_t)r * D;
      float mrun = -INFINITY;  // relaxed: running maximum of y_hat over 64-key tiles
      for (int t = 0; t < nch; ++t) {
        const int j = 32 * t + lane;
        if (relaxed && (t & 1) == 0) {
          const float v0 = j < nv ? row[j] : -INFINITY;
          const float v1 = j + 32 < nv ? row[j + 32] : -INFINITY;
          mrun = fmaxf(mrun, warp_max(fmaxf(v0, v1)));
        }
        bool sel = false;
        if (j < nv) {
          if (given) {
            sel = (__ldg(p.mask_in + grow * nwords + t) >> lane) & 1u;
          } else if (relaxed) {
            const float y = row[j];
            const float c = 2.f * expf(__fsub_rn(y, mrun)) * fabsf(y);
            sel = c > p.tau;
            if (refine_ok && (fabsf(c - p.tau) <= kBand * p.tau || (p.tau == 0.f && c < 1e-30f))) {
              const double cd = 2.0 * exp((double)y - (double)mrun) * fabs((double)y);
              sel = cd > (double)p.tau;
            }
          } else {
            const float y = row[j];
            const float e = (j == am) ? 1.f : expf(__fsub_rn(y, m));
            const float om = (j == am) ? srest_f : __fsub_rn(Sf, e);
            const float c = 2.f * fabsf(y) * e * om * invS2;
            sel = c > p.tau;
            if (refine_ok && (fabsf(c - p.tau) <= kBand * p.tau || (p.tau == 0.f && c < 1e-30f))) {
              const double ed = (j == am) ? 1.0 : exp((double)y - (double)m);
              const double z = ed / Sd;
              const double omz = (j == am) ? srest / Sd : (Sd - ed) / Sd;
              const double cd = 2.0 * z * omz * fabs((double)y);
              sel = cd > (double)p.tau;
            }
          }
        }
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, sel);
        if ((t & 31) == lane) myword = bal;
        if ((t & 31) == 31 || t == nch - 1) {
          const int g = t & ~31;
          if (mrow && g + lane <= t) mrow[g + lane] = myword;
        }
        row_nsel += __popc(bal);
        if (sel) list[list_n + __popc(bal & lanemask_lt)] = j;
        list_n += __popc(bal);
        __syncwarp();
        if (list_n >= 32) {
          const int jj = list[lane];
          const float y32 = recompute_fp32<D>(qrow, Kh + (size_t)jj * D, p.scale, fast);
          __syncwarp();
          const int rest = list_n - 32;
          if (lane < rest) list[lane] = list[32 + lane];
          row[jj] = y32;
          list_n = rest;
          __syncwarp();
        }
      }
      if (list_n > 0) {
        if (lane < list_n) {
          const int jj = list[lane];
          row[jj] = recompute_fp32<D>(qrow, Kh + (size_t)jj * D, p.scale, fast);
        }
        list_n = 0;
      }
      __syncwarp();
      if (mrow)
        for (int w = nch + lane; w < nwords; w += 32) mrow[w] = 0u;
      warp_nsel += row_nsel;
      if (p.mixed_out)
        for (int j = lane; j < p.n_k; j += 32) p.mixed_out[grow * p.n_k + j] = j < nv ? row[j] : -INFINITY;
      // phase 3: softmax of the mixed row, P written in place as bf16 hi/lo
      float mm = -INFINITY;
      for (int j = lane; j < nv; j += 32) mm = fmaxf(mm, row[j]);
      mm = warp_max(mm);
      float l = 0.f;
      for (int j = lane; j < nv; j += 32) {
        const float pj = __expf(__fsub_rn(row[j], mm));
        row[j] = pj;
        l += pj;
      }
      l = warp_sum(l);
      const float inv_l = 1.f / l;
      if (p.lse_out && lane == 0) p.lse_out[grow] = mm + logf(l);
      __syncwarp();
      uint16_t* rb16 = reinterpret_cast<uint16_t*>(row);
      for (int c = 0; c * 32 < kv_end; ++c) {
        const int j = 32 * c + lane;
        const float pj = (j < nv) ? row[j] * inv_l : 0.f;
        __syncwarp();
        uint16_t hi, lo;
        split_bf16(pj, hi, lo);
        rb16[64 * c + lane] = hi;
        rb16[64 * c + 32 + lane] = lo;
        __syncwarp();
      }
    }
    if (p.nsel_out && lane == 0 && warp_nsel) atomicAdd(p.nsel_out, (unsigned long long)warp_nsel);

    // ---- phase 4: O = P.V on tensor cores -----------------------------------
    __syncthreads();
    {
      constexpr int VS = D + 8;                 // padded V row (bf16)
      constexpr int NG = D / 64;                // n16 groups per warp
      const int mt = warp & 1;                  // rows 16*mt .. 16*mt+15
      const int ng0 = warp >> 1;                // n16 groups ng0 + 4*g
      float accO[NG][2][4];
#pragma unroll
      for (int g = 0; g < NG; ++g)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int e = 0; e < 4; ++e) accO[g][h][e] = 0.f;
      const int nvt = (kv_end + VT - 1) / VT;
      auto load_v = [&](int vt, int buf) {
        uint16_t* dstb = sV + (size_t)buf * VT * VS;
        constexpr int CH = D / 8;  // 16-byte chunks per key row
        for (int idx = tid; idx < VT * CH; idx += NT) {
          const int key = idx / CH, ch = idx % CH;
          const int gk = vt * VT + key;
          uint16_t* dst = dstb + key * VS + ch * 8;
          if (gk < p.n_k) cp_async16(dst, Vh + (size_t)gk * D + ch * 8);
          else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        cp_async_commit();
      };
      if (nvt > 0) load_v(0, 0);
      const int g_ = lane >> 2, t4 = lane & 3;
      const uint16_t* Prow0 = reinterpret_cast<const uint16_t*>(S + (size_t)(16 * mt + g_) * nkp);
      const uint16_t* Prow8 = reinterpret_cast<const uint16_t*>(S + (size_t)(16 * mt + g_ + 8) * nkp);
      for (int vt = 0; vt < nvt; ++vt) {
        if (vt + 1 < nvt) {
          load_v(vt + 1, (vt + 1) & 1);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        __syncthreads();
        const uint16_t* vb = sV + (size_t)(vt & 1) * VT * VS;
#pragma unroll
        for (int ks = 0; ks < VT / 16; ++ks) {
          const int kb = vt * VT + ks * 16;
          if (kb >= kv_end) break;
          // A fragments (P hi and lo) straight from the row store
          const int c32 = kb >> 5, off = (kb & 31) + 2 * t4;
          const int hi0 = 64 * c32 + off, lo0 = hi0 + 32;
          uint32_t ah[4], al[4];
          ah[0] = *reinterpret_cast<const uint32_t*>(Prow0 + hi0);
          ah[1] = *reinterpret_cast<const uint32_t*>(Prow8 + hi0);
          ah[2] = *reinterpret_cast<const uint32_t*>(Prow0 + hi0 + 8);
          ah[3] = *reinterpret_cast<const uint32_t*>(Prow8 + hi0 + 8);
          al[0] = *reinterpret_cast<const uint32_t*>(Prow0 + lo0);
          al[1] = *reinterpret_cast<const uint32_t*>(Prow8 + lo0);
          al[2] = *reinterpret_cast<const uint32_t*>(Prow0 + lo0 + 8);
          al[3] = *reinterpret_cast<const uint32_t*>(Prow8 + lo0 + 8);
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const int n0 = 16 * (ng0 + 4 * g);
            const int krow = ks * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ncol = n0 + 8 * (lane >> 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(smem_u32(vb + krow * VS + ncol), b0, b1, b2, b3);
            mma_bf16_16816(accO[g][0], ah[0], ah[1], ah[2], ah[3], b0, b1);
            mma_bf16_16816(accO[g][0], al[0], al[1], al[2], al[3], b0, b1);
            mma_bf16_16816(accO[g][1], ah[0], ah[1], ah[2], ah[3], b2, b3);
            mma_bf16_16816(accO[g][1], al[0], al[1], al[2], al[3], b2, b3);
          }
        }
        __syncthreads();
      }
      // store O
#pragma unroll
      for (int g = 0; g < NG; ++g) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int col = 16 * (ng0 + 4 * g) + 8 * h + 2 * t4;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int r = 16 * mt + g_ + 8 * half;
            if (r >= rows) continue;
            const size_t o = ((size_t)bh * p.n_q + i0 + r) * D + col;
            const float v0 = accO[g][h][2 * half], v1 = accO[g][h][2 * half + 1];
            const uint32_t packed = (uint32_t)f32_to_bf16_rne(v0) | ((uint32_t)f32_to_bf16_rne(v1) << 16);
            *reinterpret_cast<uint32_t*>(p.out + o) = packed;
            if (p.out_f32) *reinterpret_cast<float2*>(p.out_f32 + o) = make_float2(v0, v1);
          }
        }
      }
    }
    __syncthreads();
  }
}

template <int D, int RND>
cudaError_t launch_one(const StrictArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto k = strict_kernel<D, RND>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, NT, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t strict_smem_bytes(int d, int nkp, bool rows_on_chip) {
  size_t b = q_bytes(d) + k_bytes(d) + list_bytes();
  if (rows_on_chip) b += (size_t)BM * nkp * 4;
  return b;
}

cudaError_t launch_strict(const Problem& p, const Workspace& ws, char* base, int num_sms,
                          size_t smem_optin, cudaStream_t st) {
  (void)smem_optin;
  StrictArgs a;
  a.p = p;
  a.stats = reinterpret_cast<const int*>(base + ws.stats);
  a.nchunk = ws.nchunk;
  a.counter = reinterpret_cast<uint32_t*>(base + ws.counters);
  a.spill = ws.spill_rows ? reinterpret_cast<float*>(base + ws.spill) : nullptr;
  a.nkp = ws.nkp;
  a.rows_on_chip = ws.spill_rows ? 0 : 1;
  a.n_rb = (p.n_q + BM - 1) / BM;
  a.n_items = a.n_rb * p.B * p.H;
  const int grid = ws.spill_rows ? ws.grid : (a.n_items < num_sms ? a.n_items : num_sms);
  const size_t smem = strict_smem_bytes(p.d, ws.nkp, !ws.spill_rows);
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  if (p.d == 64) {
    if (rnd == kRndFast) return launch_one<64, kRndFast>(a, grid, smem, st);
    if (rnd == kRndNone) return launch_one<64, kRndNone>(a, grid, smem, st);
    return launch_one<64, kRndExact>(a, grid, smem, st);
  }
  if (rnd == kRndFast) return launch_one<128, kRndFast>(a, grid, smem, st);
  if (rnd == kRndNone) return launch_one<128, kRndNone>(a, grid, smem, st);
  return launch_one<128, kRndExact>(a, grid, smem, st);
}

}  // namespace lamp
