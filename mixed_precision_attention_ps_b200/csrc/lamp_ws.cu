// LAMP attention, warp-specialised row kernel (strict, relaxed, given mask) for
// rows short enough that two blocks of 16 complete score rows fit in shared
// memory at once (n_k up to about a thousand keys; the GPT-2 XL attention shape).
//
// Method ("LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models",
// technical summary, gist.science paper 2601.21623): section "Implementation
// strategy", steps 1-3; section "Theoretical basis", item 3, softmax bullet (the
// strict test 2 z (1 - z) |y| > tau on the whole probability row); section
// "Experimental results" (PS(mu), relaxed relative threshold, random control).
//
// One persistent CTA of 512 threads per SM works through a fixed sequence of
// items (b, h, block of 16 query rows), heaviest causal blocks first, in a snake
// order over the CTAs. Two row buffers alternate between two warp groups:
//
//   producers (warps 0-7): PS(mu) scores of item k into buffer k & 1. The item's
//     keys are cut into 32-key units dealt round-robin to the producer warps,
//     continuing across items, so no warp idles at the end of an item. Each warp
//     stages its own K slices (16 head dimensions x 32 keys, binary32, double
//     buffered) and needs no block-wide barrier; a lane holds 4 rows x 4 keys as
//     packed binary32 pairs; one accumulation step is fma.rn.f32x2 plus the
//     two-instruction PS(mu) rounding (or the exact integer rounding).
//   consumers (warps 8-15): for item k, two rows per warp processed together:
//     row maximum and first argmax, S_rest in double (strict), the criterion with
//     a double re-evaluation near tau, mask words, warp-compacted FP32 recompute,
//     softmax numerators of the mixed row written in place as bf16 hi/lo pairs;
//     then P.V on tensor cores (mma.sync, V staged by cp.async) and the output.
//
// Hand-offs use named barriers: "full[b]" (producers arrive, consumers wait) and
// "empty[b]" (consumers arrive, producers wait), so each side blocks only when
// the other is a whole item behind.
#include <cfloat>

#include "lamp_device.cuh"
#include "lamp_kernels.h"

namespace lamp {
namespace {

constexpr int WS_BM = 16;              // query rows per item
constexpr int WS_NT = kWsThreads;      // 512
constexpr int WS_NP = 8;               // producer warps
constexpr int WS_NC = 8;               // consumer warps
constexpr int WS_UNIT = 32;            // keys per producer unit
constexpr int WS_DS = 16;              // head dimensions per K slice
constexpr int WS_LIST = 64;            // per-warp recompute list capacity
constexpr float WS_BAND = 8e-6f;       // relative band around tau re-evaluated in double

// named barriers (0 is __syncthreads, unused after the split)
constexpr int BAR_EMPTY0 = 1;          // + buffer
constexpr int BAR_FULL0 = 3;           // + buffer
constexpr int BAR_PROD = 5;            // producers only
constexpr int BAR_CONS = 6;            // consumers only

__device__ __forceinline__ void bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

template <int D>
__host__ __device__ constexpr int ws_vkeys() { return D == 64 ? 128 : 64; }

struct WsSmem {
  int q;      // Q pairs [2][D][16] u64
  int ks;     // producer K slices [8 warps][2][16][32] f32
  int v;      // consumer V chunks [2][VK][D + 8] bf16, later the output sums [16][D] f32
  int list;   // consumer recompute lists [8][64] int
  int stats;  // per buffer and row: softmax max, normaliser [2][16][2] f32
  int rows;   // score rows [2][16][nkp] f32
  int total;
};

template <int D>
__host__ __device__ inline WsSmem ws_plan(int nkp) {
  WsSmem s{};
  s.q = 0;
  s.ks = s.q + 2 * D * WS_BM * 8;
  s.v = s.ks + WS_NP * 2 * WS_DS * WS_UNIT * 4;
  const int vb = 2 * ws_vkeys<D>() * (D + 8) * 2;
  const int ob = WS_BM * D * 4;
  s.list = s.v + (vb > ob ? vb : ob);
  s.stats = s.list + WS_NC * WS_LIST * 4;
  s.rows = s.stats + 2 * WS_BM * 2 * 4;
  s.total = s.rows + 2 * WS_BM * nkp * 4;
  return s;
}

struct WsArgs {
  Problem p;
  const int* stats;  // per-(b, h) exponent statistics
  int nchunk;
  int nkp;           // row stride in floats
  int n_items;
  int n_rb;
};

// Row r (0..15) of the Q pair layout: lane group gr reads rows 4gr + 2h and
// 4gr + 2h + 1 with one 16-byte load at h * 8 + 2gr.
__device__ __forceinline__ int ws_qpos(int r) { return ((r >> 1) & 1) * 8 + (r >> 2) * 2 + (r & 1); }

// The k-th item of CTA b (snake order over heaviest-first items), or -1.
__device__ __forceinline__ int ws_item(int k, int b, int G, int n_items) {
  const int q = (k & 1) ? (k + 1) * G - 1 - b : k * G + b;
  return q < n_items ? q : -1;
}

struct ItemInfo {
  int bh, i0, rows, kv_end;
};

__device__ __forceinline__ ItemInfo ws_decode(int q, const WsArgs& a) {
  const Problem& p = a.p;
  const int BH = p.B * p.H;
  ItemInfo it;
  const int rb = p.causal ? a.n_rb - 1 - q / BH : q / BH;
  it.bh = q % BH;
  it.i0 = rb * WS_BM;
  it.rows = min(WS_BM, p.n_q - it.i0);
  it.kv_end = p.causal ? min(p.n_k, max(0, it.i0 + it.rows + (p.n_k - p.n_q))) : p.n_k;
  return it;
}

__device__ __forceinline__ int ws_valid_keys(int i, const Problem& p) {
  if (!p.causal) return p.n_k;
  return min(p.n_k, max(0, i + 1 + (p.n_k - p.n_q)));
}

// WS_DS accumulation steps of a lane's 4 x 4 score tile (16-row items).
//   qs: Q pairs of this slice, [WS_DS][16] u64; ks: warp's K slice, [WS_DS][32] f32.
template <int MODE>
__device__ __forceinline__ void score_slice_ws(const u64* __restrict__ qs, const float* __restrict__ ks, int qoff,
                                               int koff, u64 (&acc)[4][2], u64 negc, u64 pow2s, int s) {
#pragma unroll 4
  for (int dd = 0; dd < WS_DS; ++dd) {
    const ulonglong2 qa = *reinterpret_cast<const ulonglong2*>(qs + dd * WS_BM + qoff);
    const ulonglong2 qb = *reinterpret_cast<const ulonglong2*>(qs + dd * WS_BM + 8 + qoff);
    const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(ks + dd * WS_UNIT + koff);
    const u64 q[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      acc[r][0] = ps_step<MODE>(q[r], kk.x, acc[r][0], negc, pow2s, s);
      acc[r][1] = ps_step<MODE>(q[r], kk.y, acc[r][1], negc, pow2s, s);
    }
  }
}

// ---------------------------------------------------------------------------
// Producers: PS(mu) scores of every item into the item's row buffer.
// ---------------------------------------------------------------------------
template <int D, int RND>
__device__ __forceinline__ void ws_producer(const WsArgs& a, unsigned char* smem, const WsSmem& L, int warp,
                                            int lane) {
  constexpr int NSL = D / WS_DS;  // K slices per unit
  const Problem& p = a.p;
  const int tidp = warp * 32 + lane;
  const int G = gridDim.x, cta = blockIdx.x;
  const int s = 23 - p.mu;
  const u64 negc = pack2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const u64 pow2s = pack2((float)(1u << s), (float)(1u << s));
  const u64 scale2 = pack2(p.scale, p.scale);
  float* ksw = reinterpret_cast<float*>(smem + L.ks) + warp * 2 * WS_DS * WS_UNIT;
  const int gr = lane & 3, gk = lane >> 2;  // rows 4gr..4gr+3, keys 4gk..4gk+3 of a unit
  const int qoff = 2 * gr, koff = 4 * gk;
  int deal = 0;  // producer warp that takes the next unit
  for (int k = 0;; ++k) {
    const int q = ws_item(k, cta, G, a.n_items);
    if (q < 0) break;
    const int buf = k & 1;
    const ItemInfo it = ws_decode(q, a);
    bar_sync(BAR_EMPTY0 + buf, WS_NT);  // the consumers are done with this buffer
    u64* sQ = reinterpret_cast<u64*>(smem + L.q) + buf * D * WS_BM;
    for (int u = tidp; u < WS_BM * D / 8; u += WS_NP * 32) {
      const int r = u / (D / 8), c8 = (u % (D / 8)) * 8;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (r < it.rows)
        w = __ldg(reinterpret_cast<const uint4*>(p.Q + ((size_t)it.bh * p.n_q + it.i0 + r) * D + c8));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      const int pos = ws_qpos(r);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v0 = bf16_lo(ws[e]), v1 = bf16_hi(ws[e]);
        sQ[(c8 + 2 * e) * WS_BM + pos] = pack2(v0, v0);
        sQ[(c8 + 2 * e + 1) * WS_BM + pos] = pack2(v1, v1);
      }
    }
    bar_sync(BAR_PROD, WS_NP * 32);
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    float* rows = reinterpret_cast<float*>(smem + L.rows) + (size_t)buf * WS_BM * a.nkp;
    const int U = (it.kv_end + WS_UNIT - 1) / WS_UNIT;
    const int first = (warp - deal + WS_NP) % WS_NP;
    const int mine = first < U ? (U - first + WS_NP - 1) / WS_NP : 0;
    const int total = mine * NSL;
    uint4 kr[2];
    auto load = [&](int pos) {  // slice of stream position pos into registers
      const int j = first + WS_NP * (pos / NSL), sl = pos % NSL;
      const int key = j * WS_UNIT + lane;
      kr[0] = kr[1] = make_uint4(0u, 0u, 0u, 0u);
      if (key < it.kv_end) {
        const uint4* src = reinterpret_cast<const uint4*>(Kh + (size_t)key * D + sl * WS_DS);
        kr[0] = __ldg(src);
        kr[1] = __ldg(src + 1);
      }
    };
    auto store = [&](int b2) {
      float* dst = ksw + b2 * WS_DS * WS_UNIT + lane;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t ws[4] = {kr[h].x, kr[h].y, kr[h].z, kr[h].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dst[(8 * h + 2 * e) * WS_UNIT] = bf16_lo(ws[e]);
          dst[(8 * h + 2 * e + 1) * WS_UNIT] = bf16_hi(ws[e]);
        }
      }
    };
    if (total > 0) {
      load(0);
      store(0);
    }
    __syncwarp();
    u64 acc[4][2];
    for (int pos = 0; pos < total; ++pos) {
      const int j = first + WS_NP * (pos / NSL), sl = pos % NSL;
      if (pos + 1 < total) load(pos + 1);
      if (sl == 0) {
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = 0ull;
      }
      const u64* qs = sQ + sl * WS_DS * WS_BM;
      const float* ks = ksw + (pos & 1) * WS_DS * WS_UNIT;
      if (RND == kRndFast && fast) score_slice_ws<kStepFast>(qs, ks, qoff, koff, acc, negc, pow2s, s);
      else if (RND == kRndNone && fast) score_slice_ws<kStepF32>(qs, ks, qoff, koff, acc, negc, pow2s, s);
      else score_slice_ws<kStepExact>(qs, ks, qoff, koff, acc, negc, pow2s, s);
      if (sl == NSL - 1) {
        const int j0 = j * WS_UNIT + koff;
#pragma unroll
        for (int r4 = 0; r4 < 4; ++r4) {
          const int r = 4 * gr + r4;
          const int nv = r < it.rows ? ws_valid_keys(it.i0 + r, p) : 0;
          const u64 y01 = mul2u(acc[r4][0], scale2), y23 = mul2u(acc[r4][1], scale2);
          float4 y;
          y.x = j0 < nv ? lo_f(y01) : -INFINITY;
          y.y = j0 + 1 < nv ? hi_f(y01) : -INFINITY;
          y.z = j0 + 2 < nv ? lo_f(y23) : -INFINITY;
          y.w = j0 + 3 < nv ? hi_f(y23) : -INFINITY;
          *reinterpret_cast<float4*>(rows + (size_t)r * a.nkp + j0) = y;
        }
      }
      if (pos + 1 < total) store((pos + 1) & 1);
      __syncwarp();
    }
    deal = (deal + U) % WS_NP;
    bar_arrive(BAR_FULL0 + buf, WS_NT);  // scores of this item are in place
  }
}

// FP32 recompute of score (row r, key j) from the Q pairs and K in global memory.
template <int D>
__device__ __forceinline__ float ws_recompute(const u64* __restrict__ sQ, int r, const uint16_t* __restrict__ krow,
                                              float scale, bool fused) {
  const int pos = ws_qpos(r);
  float acc = 0.f;
#pragma unroll
  for (int kk = 0; kk < D; kk += 8) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(krow + kk));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float k0 = bf16_lo(ws[e]), k1 = bf16_hi(ws[e]);
      const float q0 = lo_f(sQ[(kk + 2 * e) * WS_BM + pos]);
      const float q1 = lo_f(sQ[(kk + 2 * e + 1) * WS_BM + pos]);
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

// ---------------------------------------------------------------------------
// Consumers: selection, recompute, softmax, P.V and the output of every item.
// ---------------------------------------------------------------------------
template <int D, int RND>
__device__ __forceinline__ void ws_consumer(const WsArgs& a, unsigned char* smem, const WsSmem& L, int cw,
                                            int lane) {
  constexpr int VK = ws_vkeys<D>();
  constexpr int VS = D + 8;
  constexpr int NH = D / 64;
  constexpr int KQ = WS_NC / NH;
  constexpr int SPW = (VK / 8) / KQ;
  constexpr int TPG = 8 / KQ;
  const Problem& p = a.p;
  const int tidc = cw * 32 + lane;
  const int G = gridDim.x, cta = blockIdx.x;
  const int nwords = (p.n_k + 31) >> 5;
  const uint32_t lanemask_lt = (1u << lane) - 1u;
  const bool strict = p.variant == 0, relaxed = p.variant == 1, given = p.variant == 2;
  const bool refine_ok = isfinite(p.tau) && p.tau >= 0.f;
  const float band = WS_BAND * p.tau;
  int* list = reinterpret_cast<int*>(smem + L.list) + cw * WS_LIST;
  uint16_t* sV = reinterpret_cast<uint16_t*>(smem + L.v);
  float* sO = reinterpret_cast<float*>(smem + L.v);
  long long nsel = 0;
  // the first two buffers start out free
  if (ws_item(0, cta, G, a.n_items) >= 0) bar_arrive(BAR_EMPTY0 + 0, WS_NT);
  if (ws_item(1, cta, G, a.n_items) >= 0) bar_arrive(BAR_EMPTY0 + 1, WS_NT);
  for (int k = 0;; ++k) {
    const int q = ws_item(k, cta, G, a.n_items);
    if (q < 0) break;
    const int buf = k & 1;
    const ItemInfo it = ws_decode(q, a);
    bar_sync(BAR_FULL0 + buf, WS_NT);  // the producers have written this item's scores
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    const uint16_t* Vh = p.V + (size_t)it.bh * p.n_k * D;
    const u64* sQ = reinterpret_cast<const u64*>(smem + L.q) + buf * D * WS_BM;
    float* rows = reinterpret_cast<float*>(smem + L.rows) + (size_t)buf * WS_BM * a.nkp;
    float* st = reinterpret_cast<float*>(smem + L.stats) + buf * WS_BM * 2;
    const int written = ((it.kv_end + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;  // keys the producers wrote
    const int nch_kv = written >> 5;

    // ---- selection and recompute, rows 2cw and 2cw + 1 together ---------------------
    int rr_[2], nv[2];
    size_t grow[2];
    float* row[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      rr_[t] = 2 * cw + t;
      nv[t] = rr_[t] < it.rows ? ws_valid_keys(it.i0 + rr_[t], p) : 0;
      grow[t] = (size_t)it.bh * p.n_q + it.i0 + rr_[t];
      row[t] = rows + (size_t)rr_[t] * a.nkp;
    }
    const int nvmax = max(nv[0], nv[1]);
    int list_n = 0;
    auto flush = [&](int cnt) {
      if (lane < cnt) {
        const int e = list[lane];
        const int t = e >> 16, j = e & 0xFFFF;
        const float y32 = ws_recompute<D>(sQ, 2 * cw + t, Kh + (size_t)j * D, p.scale, fast);
        rows[(size_t)(2 * cw + t) * a.nkp + j] = y32;
      }
      __syncwarp();
      const int rest = list_n - cnt;
      if (lane < rest) list[lane] = list[cnt + lane];
      __syncwarp();
      list_n = rest;
    };
    // A: maximum and first argmax of each row
    float m[2] = {-INFINITY, -INFINITY};
    int am[2] = {0x7FFFFFFF, 0x7FFFFFFF};
    const int nit = (nvmax + 127) >> 7;
    for (int i4 = 0; i4 < nit; ++i4) {
      const int j0 = 128 * i4 + 4 * lane;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (j0 < written) {
          const float4 v = *reinterpret_cast<const float4*>(row[t] + j0);
          if (v.x > m[t]) { m[t] = v.x; am[t] = j0; }
          if (v.y > m[t]) { m[t] = v.y; am[t] = j0 + 1; }
          if (v.z > m[t]) { m[t] = v.z; am[t] = j0 + 2; }
          if (v.w > m[t]) { m[t] = v.w; am[t] = j0 + 3; }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const float mw = warp_max(m[t]);
      am[t] = warp_min_i(m[t] == mw ? am[t] : 0x7FFFFFFF);
      m[t] = mw;
    }
    // B: S_rest in double (strict)
    double srest[2] = {0.0, 0.0};
    if (strict) {
      for (int i4 = 0; i4 < nit; ++i4) {
        const int j0 = 128 * i4 + 4 * lane;
        if (j0 < written) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const float4 v = *reinterpret_cast<const float4*>(row[t] + j0);
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float ex = expf(__fsub_rn(vv[e], m[t]));
              srest[t] += (j0 + e != am[t]) ? (double)ex : 0.0;
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) srest[t] = warp_sum_d(srest[t]);
    }
    double Sd[2];
    float Sf[2], srest_f[2], invS2[2], mrun[2] = {-INFINITY, -INFINITY};
    uint32_t myword[2] = {0u, 0u};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      Sd[t] = 1.0 + srest[t];
      Sf[t] = (float)Sd[t];
      srest_f[t] = (float)srest[t];
      invS2[t] = (float)(1.0 / (Sd[t] * Sd[t]));
    }
    // C: criterion, mask words, compaction of the selected keys
    const int nch = (nvmax + 31) >> 5;
    for (int c = 0; c < nch; ++c) {
      const int j = 32 * c + lane;
      float y[2];
      bool sel[2], near[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        y[t] = row[t][j];
        const bool valid = j < nv[t];
        sel[t] = near[t] = false;
        if (given) {
          sel[t] = valid && ((__ldg(p.mask_in + grow[t] * nwords + c) >> lane) & 1u);
        } else {
          float cr;
          if (relaxed) {
            if ((c & 1) == 0) {
              const float y2 = j + 32 < written ? row[t][j + 32] : -INFINITY;
              mrun[t] = fmaxf(mrun[t], warp_max(fmaxf(y[t], y2)));
            }
            cr = 2.f * fabsf(y[t]) * exp_fast(__fsub_rn(y[t], mrun[t]));
          } else {
            const float e = (j == am[t]) ? 1.f : exp_fast(__fsub_rn(y[t], m[t]));
            const float om = (j == am[t]) ? srest_f[t] : __fsub_rn(Sf[t], e);
            cr = (2.f * fabsf(y[t]) * e) * (om * invS2[t]);
          }
          sel[t] = valid && cr > p.tau;
          near[t] = valid && refine_ok && (fabsf(cr - p.tau) <= band || (p.tau == 0.f && cr < 1e-30f));
        }
      }
      if (__any_sync(0xFFFFFFFFu, near[0] || near[1])) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (near[t]) {
            double cd;
            if (relaxed) {
              cd = 2.0 * exp((double)y[t] - (double)mrun[t]) * fabs((double)y[t]);
            } else {
              const double ed = (j == am[t]) ? 1.0 : exp((double)y[t] - (double)m[t]);
              const double z = ed / Sd[t];
              const double omz = (j == am[t]) ? srest[t] / Sd[t] : (Sd[t] - ed) / Sd[t];
              cd = 2.0 * z * omz * fabs((double)y[t]);
            }
            sel[t] = cd > (double)p.tau;
          }
        }
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (p.ps_out && j < p.n_k && rr_[t] < it.rows) p.ps_out[grow[t] * p.n_k + j] = j < nv[t] ? y[t] : -INFINITY;
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, sel[t]);
        if ((c & 31) == lane) myword[t] = bal;
        if (p.mask_out && rr_[t] < it.rows && ((c & 31) == 31 || c == nch - 1)) {
          const int g0 = c & ~31;
          if (g0 + lane <= c) p.mask_out[grow[t] * nwords + g0 + lane] = myword[t];
        }
        nsel += __popc(bal);
        if (sel[t]) list[list_n + __popc(bal & lanemask_lt)] = (t << 16) | j;
        list_n += __popc(bal);
        __syncwarp();
        if (list_n >= 32) flush(32);
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (rr_[t] >= it.rows) continue;
      if (p.mask_out)
        for (int w = nch + lane; w < nwords; w += 32) p.mask_out[grow[t] * nwords + w] = 0u;
      if (p.ps_out)
        for (int j = 32 * nch + lane; j < p.n_k; j += 32) p.ps_out[grow[t] * p.n_k + j] = -INFINITY;
    }
    if (list_n > 0) flush(list_n);
    __syncwarp();

    // D: softmax numerators of the mixed rows, in place
    float mm[2] = {-INFINITY, -INFINITY};
    for (int i4 = 0; i4 < nit; ++i4) {
      const int j0 = 128 * i4 + 4 * lane;
      if (j0 < written) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const float4 v = *reinterpret_cast<const float4*>(row[t] + j0);
          mm[t] = fmaxf(mm[t], fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
        }
      }
    }
    float l[2] = {0.f, 0.f};
#pragma unroll
    for (int t = 0; t < 2; ++t) mm[t] = warp_max(mm[t]);
    for (int c = 0; c < nch_kv; ++c) {
      const int j = 32 * c + lane;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float yv = row[t][j];
        const float pj = j < nv[t] ? exp_fast(__fsub_rn(yv, mm[t])) : 0.f;
        l[t] += pj;
        if (p.mixed_out && j < p.n_k && rr_[t] < it.rows)
          p.mixed_out[grow[t] * p.n_k + j] = j < nv[t] ? yv : -INFINITY;
        reinterpret_cast<uint32_t*>(row[t])[j] = p_pair(pj);
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (p.mixed_out && rr_[t] < it.rows)
        for (int j = 32 * nch_kv + lane; j < p.n_k; j += 32) p.mixed_out[grow[t] * p.n_k + j] = -INFINITY;
      l[t] = warp_sum(l[t]);
      if (lane == 0) {
        st[2 * rr_[t]] = mm[t];
        st[2 * rr_[t] + 1] = l[t];
        if (p.lse_out && rr_[t] < it.rows) p.lse_out[grow[t]] = nv[t] > 0 ? mm[t] + logf(l[t]) : -INFINITY;
      }
    }
    bar_sync(BAR_CONS, WS_NC * 32);  // every P row of the item is in place

    // ---- O = (P.V) / l on tensor cores ----------------------------------------------
    const int nh = NH == 2 ? (cw & 1) : 0;
    const int kq = NH == 2 ? (cw >> 1) : cw;
    const int mi = lane >> 3;
    float acc[8][4];
#pragma unroll
    for (int tt = 0; tt < 8; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tt][e] = 0.f;
    const int nvc = (it.kv_end + VK - 1) / VK;
    auto load_v = [&](int vc, int b2) {
      uint16_t* dst = sV + b2 * VK * VS;
      for (int u = tidc; u < VK * (D / 8); u += WS_NC * 32) {
        const int key = u / (D / 8), ch = u % (D / 8);
        const int gkey = vc * VK + key;
        uint16_t* dd = dst + key * VS + ch * 8;
        if (gkey < p.n_k) cp_async16(dd, Vh + (size_t)gkey * D + ch * 8);
        else *reinterpret_cast<uint4*>(dd) = make_uint4(0u, 0u, 0u, 0u);
      }
      cp_async_commit();
    };
    if (nvc > 0) load_v(0, 0);
    for (int vc = 0; vc < nvc; ++vc) {
      if (vc + 1 < nvc) {
        load_v(vc + 1, (vc + 1) & 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      bar_sync(BAR_CONS, WS_NC * 32);
      const uint16_t* vb = sV + (vc & 1) * VK * VS;
#pragma unroll
      for (int qq = 0; qq < SPW; ++qq) {
        const int stp = kq + KQ * qq;
        const int kb = vc * VK + 8 * stp;
        if (kb < it.kv_end) {
          uint32_t af[4];
          const int ra = 8 * (mi & 1) + (lane & 7);
          ldmatrix_x4(smem_u32(rows + (size_t)ra * a.nkp + kb + 4 * (mi >> 1)), af[0], af[1], af[2], af[3]);
          const int kl = 8 * stp + 4 * (mi & 1) + ((lane & 7) >> 1);
#pragma unroll
          for (int nb = 0; nb < 4; ++nb) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(smem_u32(vb + kl * VS + nh * 64 + 16 * nb + 8 * (mi >> 1)), b0, b1, b2, b3);
            mma_bf16_16816(acc[2 * nb], af[0], af[1], af[2], af[3], b0, b1);
            mma_bf16_16816(acc[2 * nb + 1], af[0], af[1], af[2], af[3], b2, b3);
          }
        }
      }
      bar_sync(BAR_CONS, WS_NC * 32);
    }
#pragma unroll
    for (int rho = 0; rho < KQ; ++rho) {
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) {
        if ((tt / TPG - kq - rho + 2 * KQ) % KQ == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int rr = (lane >> 2) + 8 * h;
            float2* dst = reinterpret_cast<float2*>(sO + rr * D + nh * 64 + 8 * tt + 2 * (lane & 3));
            const float2 v = make_float2(acc[tt][2 * h], acc[tt][2 * h + 1]);
            if (rho == 0) {
              *dst = v;
            } else {
              const float2 o = *dst;
              *dst = make_float2(o.x + v.x, o.y + v.y);
            }
          }
        }
      }
      bar_sync(BAR_CONS, WS_NC * 32);
    }
    for (int u = tidc; u < WS_BM * D / 2; u += WS_NC * 32) {
      const int rr = u / (D / 2), col = (u % (D / 2)) * 2;
      if (rr >= it.rows) continue;
      const float lv = st[2 * rr + 1];
      const float inv = lv > 0.f ? 1.f / lv : 0.f;
      const float2 o = *reinterpret_cast<const float2*>(sO + rr * D + col);
      const float v0 = o.x * inv, v1 = o.y * inv;
      const size_t off = ((size_t)it.bh * p.n_q + it.i0 + rr) * D + col;
      *reinterpret_cast<uint32_t*>(p.out + off) =
          (uint32_t)f32_to_bf16_rne(v0) | ((uint32_t)f32_to_bf16_rne(v1) << 16);
      if (p.out_f32) *reinterpret_cast<float2*>(p.out_f32 + off) = make_float2(v0, v1);
    }
    bar_sync(BAR_CONS, WS_NC * 32);  // sO (the V area) is read before the next item's V loads
    if (ws_item(k + 2, cta, G, a.n_items) >= 0) bar_arrive(BAR_EMPTY0 + buf, WS_NT);
  }
  if (lane == 0 && nsel && p.nsel_out) atomicAdd(p.nsel_out, (unsigned long long)nsel);
}

template <int D, int RND>
__global__ void __launch_bounds__(WS_NT, 1) ws_kernel(const WsArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const WsSmem L = ws_plan<D>(a.nkp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < WS_NP) ws_producer<D, RND>(a, smem, L, warp, lane);
  else ws_consumer<D, RND>(a, smem, L, warp - WS_NP, lane);
}

template <int D, int RND>
cudaError_t ws_launch_one(const WsArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto k = ws_kernel<D, RND>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, WS_NT, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

int ws_nkp(int n_k) { return ((n_k + 127) / 128) * 128 + 4; }

size_t ws_smem_bytes(int d, int n_k) {
  const int nkp = ws_nkp(n_k);
  return d == 64 ? (size_t)ws_plan<64>(nkp).total : (size_t)ws_plan<128>(nkp).total;
}

bool ws_fits(int d, int n_k, size_t smem_optin) {
  return n_k <= 0xFFFF && ws_smem_bytes(d, n_k) + kStaticSmemReserve <= smem_optin;
}

cudaError_t launch_ws(const Problem& p, const Workspace& ws, char* base, int num_sms, cudaStream_t st) {
  WsArgs a;
  a.p = p;
  a.stats = reinterpret_cast<const int*>(base + ws.stats);
  a.nchunk = ws.nchunk;
  a.nkp = ws_nkp(p.n_k);
  a.n_rb = (p.n_q + WS_BM - 1) / WS_BM;
  a.n_items = a.n_rb * p.B * p.H;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  const size_t smem = ws_smem_bytes(p.d, p.n_k);
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  if (p.d == 64) {
    if (rnd == kRndFast) return ws_launch_one<64, kRndFast>(a, grid, smem, st);
    if (rnd == kRndNone) return ws_launch_one<64, kRndNone>(a, grid, smem, st);
    return ws_launch_one<64, kRndExact>(a, grid, smem, st);
  }
  if (rnd == kRndFast) return ws_launch_one<128, kRndFast>(a, grid, smem, st);
  if (rnd == kRndNone) return ws_launch_one<128, kRndNone>(a, grid, smem, st);
  return ws_launch_one<128, kRndExact>(a, grid, smem, st);
}

}  // namespace lamp
