// LAMP attention, on-chip row kernel: strict, relaxed and given-mask variants for
// rows that fit in shared memory (n_k up to a few thousand keys).
//
// Method ("LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models",
// technical summary, gist.science paper 2601.21623): section "Implementation
// strategy", steps 1-3 (low-precision baseline of the key-query products, look-
// ahead selection from that baseline, FP32 recompute of the selection before
// f); section "Theoretical basis", item 3, softmax bullet (the strict test
// 2 z (1 - z) |y| > tau); section "Experimental results" (PS(mu) accumulation,
// the relaxed relative-threshold test, the random-selection control). The strict
// test needs the whole probability row ("Significance and limitations"), so
// every work item keeps complete score rows resident in shared memory.
//
// One persistent CTA of 256 threads per SM. A work item is (b, h, block of BM
// query rows); items are taken heaviest-causal-first from an atomic counter.
//
// Phase 1, scores. A CTA tile is BM rows x BN keys; warp w owns BN/8 keys of it
// and all BM rows. A lane holds 4 rows x 4 keys as eight packed binary32 pairs
// (two keys of one row per 64-bit register). Q rows are staged once per item as
// duplicated pairs {q, q}; K is staged in slices of 16 head dimensions as
// binary32, double buffered, so the accumulation runs k = 0..d-1 in order. One
// accumulation step of a pair is fma.rn.f32x2 followed by the two-instruction
// PS(mu) rounding (mul.rn.f32x2, fma.rn.f32x2), or the exact integer rounding
// when the head's exponent range leaves the fast rounding's domain.
//
// Phase 2, per row (one warp per row, rows of a warp in turn):
//   A. row maximum m and its first index a;
//   B. S_rest = sum_{j != a} exp(y_j - m), binary32 exp summed in double;
//   C. per key: the criterion in binary32 (strict: z(1 - z) through S_rest;
//      relaxed: exp(y - M_t) with M_t the running maximum over 64-key tiles),
//      re-evaluated in double within a relative band around tau; ballot into the
//      mask word; warp-aggregated compaction of the selected keys. Lists of
//      selected (row, key) pairs of the warp's rows are recomputed as sequential
//      binary32 dot products, one pair per lane, into the row (the mixed row).
//   D. softmax numerators P_j = exp(y_j - m') of the mixed row, m' its maximum,
//      written in place of y_j as two bf16 halves (hi, lo); l = sum P_j is kept
//      per row and out = (P.V) / l.
// Phase 3, P.V on tensor cores (mma.sync m16n8k16, bf16 hi and lo of P against
// bf16 V, fp32 accumulation). Warps split the keys; V chunks are staged by
// cp.async; the per-warp partial outputs are summed in a fixed order.
#include <cfloat>

#include "lamp_device.cuh"
#include "lamp_kernels.h"

namespace lamp {
namespace {

constexpr int NT = kRowsThreads;   // 256
constexpr int NW = NT / kWarp;     // 8 warps
constexpr int DS = 16;             // head dimensions per K slice
constexpr int LIST = 64;           // per-warp recompute list capacity
constexpr float kBand = 8e-6f;     // relative band around tau re-evaluated in double

// Shared-memory plan of one CTA (byte offsets from the dynamic base).
struct Smem {
  int q;       // Q as duplicated pairs, [D][BM] u64 in lane order
  int kv;      // union: K slices [2][DS][BN] f32 | V chunks [2][VK][D + 8] bf16 | output sums [BM][D] f32
  int list;    // per-warp recompute lists, [NW][LIST] int
  int stats;   // per-row softmax maximum and normaliser: [BM][4] floats
  int rows;    // score rows [BM][nkp] f32 (P in place as bf16 hi/lo)
  int total;
};

template <int D>
__host__ __device__ constexpr int v_keys() { return D == 64 ? 128 : 64; }  // keys per V chunk

template <int D, int BM>
__host__ __device__ inline Smem smem_plan(int nkp) {
  constexpr int BN = 4096 / BM;  // CTA key tile: BM = 32 -> 128, 16 -> 256, 8 -> 512
  Smem s{};
  s.q = 0;
  s.kv = s.q + D * BM * 8;
  int kbytes = 2 * DS * BN * 4;
  int vbytes = 2 * v_keys<D>() * (D + 8) * 2;
  int obytes = BM * D * 4;
  int u = kbytes > vbytes ? kbytes : vbytes;
  u = u > obytes ? u : obytes;
  s.list = s.kv + u;
  s.stats = s.list + NW * LIST * 4;
  s.rows = s.stats + BM * 16;
  s.total = s.rows + BM * nkp * 4;
  return s;
}

__device__ __forceinline__ int n_valid_keys(int i, const Problem& p) {
  if (!p.causal) return p.n_k;
  return min(p.n_k, max(0, i + 1 + (p.n_k - p.n_q)));
}


struct RowsArgs {
  Problem p;
  const int* stats;   // per-(b, h) exponent statistics (preparation kernel)
  int nchunk;
  uint32_t* counter;  // work counter, zeroed by the preparation kernel
  int nkp;            // row stride in floats
  int n_items;
  int n_rb;
};

// Position of query row r (0 <= r < BM) in the duplicated-pair Q layout: lane
// group gr reads rows 4gr + 2h and 4gr + 2h + 1 with one 16-byte load at
// h * BM/2 + 2gr, so that the GR groups of a load cover one contiguous span.
template <int BM>
__device__ __forceinline__ int qpos(int r) {
  return ((r >> 1) & 1) * (BM / 2) + (r >> 2) * 2 + (r & 1);
}

// DS accumulation steps of the lane's 4 x 4 score tile from one K slice.
//   qs: this slice's Q pairs, [DS][BM] u64; ks: K slice [DS][BN] f32.
template <int BM, int BN, int MODE>
__device__ __forceinline__ void score_slice(const u64* __restrict__ qs, const float* __restrict__ ks,
                                            int qoff, int koff, u64 (&acc)[4][2], u64 negc, u64 pow2s,
                                            int s) {
#pragma unroll 4
  for (int dd = 0; dd < DS; ++dd) {
    const ulonglong2 qa = *reinterpret_cast<const ulonglong2*>(qs + dd * BM + qoff);
    const ulonglong2 qb = *reinterpret_cast<const ulonglong2*>(qs + dd * BM + BM / 2 + qoff);
    const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(ks + dd * BN + koff);
    const u64 q[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      acc[r][0] = ps_step<MODE>(q[r], kk.x, acc[r][0], negc, pow2s, s);
      acc[r][1] = ps_step<MODE>(q[r], kk.y, acc[r][1], negc, pow2s, s);
    }
  }
}


// FP32 recompute of score (row r, key j): the sequential binary32 sum over
// k = 0..D-1 (one multiply and one add per step; a fused multiply-add when the
// head's products are exact), then the scale.
template <int D, int BM>
__device__ __forceinline__ float recompute_fp32(const u64* __restrict__ sQ, int r,
                                                const uint16_t* __restrict__ krow, float scale,
                                                bool fused) {
  const int pos = qpos<BM>(r);
  float acc = 0.f;
#pragma unroll
  for (int kk = 0; kk < D; kk += 8) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(krow + kk));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float k0 = bf16_lo(ws[e]), k1 = bf16_hi(ws[e]);
      const float q0 = lo_f(sQ[(kk + 2 * e) * BM + pos]);
      const float q1 = lo_f(sQ[(kk + 2 * e + 1) * BM + pos]);
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

template <int D, int BM, int RND>
__global__ void __launch_bounds__(NT, 1) rows_kernel(const RowsArgs a) {
  constexpr int GR = BM / 4;         // row groups of a warp tile
  constexpr int GK = 32 / GR;        // key groups
  constexpr int WK = 4 * GK;         // keys per warp per tile
  constexpr int BN = NW * WK;        // keys per CTA tile
  constexpr int SPT = D / DS;        // K slices per tile
  constexpr int KU = BN / 128;       // K-slice units (8 bf16) per thread
  constexpr int RPW = BM / NW;       // rows per warp in the selection phase
  static_assert(BN == 4096 / BM, "tile plan");

  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int sItem;
  const Problem& p = a.p;
  const int nkp = a.nkp;
  const Smem L = smem_plan<D, BM>(nkp);
  u64* sQ = reinterpret_cast<u64*>(smem + L.q);
  float* sK = reinterpret_cast<float*>(smem + L.kv);
  int* sList = reinterpret_cast<int*>(smem + L.list);
  float* sStat = reinterpret_cast<float*>(smem + L.stats);
  float* sRows = reinterpret_cast<float*>(smem + L.rows);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gr = lane % GR, gk = lane / GR;
  const int BH = p.B * p.H;
  const int nwords = (p.n_k + 31) >> 5;
  const int s = 23 - p.mu;
  const u64 negc = pack2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const u64 pow2s = pack2((float)(1u << s), (float)(1u << s));
  const u64 scale2 = pack2(p.scale, p.scale);
  long long warp_nsel = 0;

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

    // ---- Q rows as duplicated binary32 pairs -----------------------------------
    for (int u = tid; u < BM * D / 8; u += NT) {
      const int r = u / (D / 8), c8 = (u % (D / 8)) * 8;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (r < rows) w = __ldg(reinterpret_cast<const uint4*>(p.Q + ((size_t)bh * p.n_q + i0 + r) * D + c8));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      const int pos = qpos<BM>(r);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v0 = bf16_lo(ws[e]), v1 = bf16_hi(ws[e]);
        sQ[(c8 + 2 * e) * BM + pos] = pack2(v0, v0);
        sQ[(c8 + 2 * e + 1) * BM + pos] = pack2(v1, v1);
      }
    }

    // ---- phase 1: PS(mu) scores ----------------------------------------------------
    const int ntiles = (kv_end + BN - 1) / BN;
    const int nsl = ntiles * SPT;
    uint4 kreg[KU];
    auto load_slice = [&](int g) {
      const int T = g / SPT, sl = g % SPT;
#pragma unroll
      for (int i = 0; i < KU; ++i) {
        const int u = tid + NT * i;
        const int key = u % BN, half = u / BN;
        const int gkey = T * BN + key;
        kreg[i] = make_uint4(0u, 0u, 0u, 0u);
        if (gkey < kv_end)
          kreg[i] = __ldg(reinterpret_cast<const uint4*>(Kh + (size_t)gkey * D + sl * DS + half * 8));
      }
    };
    auto store_slice = [&](int buf) {
      float* dst = sK + buf * DS * BN;
#pragma unroll
      for (int i = 0; i < KU; ++i) {
        const int u = tid + NT * i;
        const int key = u % BN, half = u / BN;
        const uint32_t ws[4] = {kreg[i].x, kreg[i].y, kreg[i].z, kreg[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dst[(half * 8 + 2 * e) * BN + key] = bf16_lo(ws[e]);
          dst[(half * 8 + 2 * e + 1) * BN + key] = bf16_hi(ws[e]);
        }
      }
    };
    if (nsl > 0) {
      load_slice(0);
      store_slice(0);
    }
    __syncthreads();
    {
      const int wbase = warp * WK;
      const int qoff = 2 * gr, koff = wbase + 4 * gk;
      u64 acc[4][2];
      for (int g = 0; g < nsl; ++g) {
        const int T = g / SPT, sl = g % SPT;
        if (g + 1 < nsl) load_slice(g + 1);
        if (sl == 0) {
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = 0ull;
        }
        const bool active = T * BN + wbase < kv_end;
        if (active) {
          const u64* qs = sQ + sl * DS * BM;
          const float* ks = sK + (g & 1) * DS * BN;
          if (RND == kRndFast && fast) score_slice<BM, BN, kStepFast>(qs, ks, qoff, koff, acc, negc, pow2s, s);
          else if (RND == kRndNone && fast) score_slice<BM, BN, kStepF32>(qs, ks, qoff, koff, acc, negc, pow2s, s);
          else score_slice<BM, BN, kStepExact>(qs, ks, qoff, koff, acc, negc, pow2s, s);
        }
        if (sl == SPT - 1) {
          // y_hat = fl32(scale * acc); keys past the row's valid range hold -inf
          const int j0 = T * BN + koff;
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4) {
            const int r = 4 * gr + r4;
            const int nv = r < rows ? n_valid_keys(i0 + r, p) : 0;
            float4 y = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            if (active) {
              const u64 y01 = mul2u(acc[r4][0], scale2), y23 = mul2u(acc[r4][1], scale2);
              if (j0 < nv) y.x = lo_f(y01);
              if (j0 + 1 < nv) y.y = hi_f(y01);
              if (j0 + 2 < nv) y.z = lo_f(y23);
              if (j0 + 3 < nv) y.w = hi_f(y23);
            }
            *reinterpret_cast<float4*>(sRows + (size_t)r * nkp + j0) = y;
          }
        }
        if (g + 1 < nsl) store_slice((g + 1) & 1);
        __syncthreads();
      }
    }

    // ---- phase 2: selection and recompute (A, B, C per row), then P (D) ------------
    {
      const uint32_t lanemask_lt = (1u << lane) - 1u;
      int* list = sList + warp * LIST;
      int list_n = 0;
      const bool strict = p.variant == 0, relaxed = p.variant == 1, given = p.variant == 2;
      const bool refine_ok = isfinite(p.tau) && p.tau >= 0.f;
      const float band = kBand * p.tau;
      const int nch_kv = (kv_end + 31) >> 5;

      // recompute the first cnt listed (row, key) pairs, one per lane
      auto flush = [&](int cnt) {
        if (lane < cnt) {
          const int e = list[lane];
          const int r = warp * RPW + (e >> 16), j = e & 0xFFFF;
          const float y32 = recompute_fp32<D, BM>(sQ, r, Kh + (size_t)j * D, p.scale, fast);
          sRows[(size_t)r * nkp + j] = y32;
        }
        __syncwarp();
        const int rest = list_n - cnt;
        if (lane < rest) list[lane] = list[cnt + lane];
        __syncwarp();
        list_n = rest;
      };

      for (int ri = 0; ri < RPW; ++ri) {
        const int r = warp * RPW + ri;
        if (r >= rows) break;
        const int i = i0 + r;
        const int nv = n_valid_keys(i, p);
        float* row = sRows + (size_t)r * nkp;
        const size_t grow = (size_t)bh * p.n_q + i;
        uint32_t* mrow = p.mask_out ? p.mask_out + grow * nwords : nullptr;
        // A: row maximum and its first index
        float m = -INFINITY;
        int am = 0x7FFFFFFF;
        const int nit = (nv + 127) >> 7;
        for (int it = 0; it < nit; ++it) {
          const int j0 = 128 * it + 4 * lane;
          const float4 v = *reinterpret_cast<const float4*>(row + j0);
          if (v.x > m) { m = v.x; am = j0; }
          if (v.y > m) { m = v.y; am = j0 + 1; }
          if (v.z > m) { m = v.z; am = j0 + 2; }
          if (v.w > m) { m = v.w; am = j0 + 3; }
        }
        {
          const float mw = warp_max(m);
          am = warp_min_i(m == mw ? am : 0x7FFFFFFF);
          m = mw;
        }
        // B: S_rest = sum over j != argmax of exp(y_j - m), in double (strict only)
        double srest = 0.0;
        if (strict) {
          for (int it = 0; it < nit; ++it) {
            const int j0 = 128 * it + 4 * lane;
            const float4 v = *reinterpret_cast<const float4*>(row + j0);
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (j0 + e != am) srest += (double)expf(__fsub_rn(vv[e], m));
          }
          srest = warp_sum_d(srest);
        }
        const double Sd = 1.0 + srest;
        const float Sf = (float)Sd, srest_f = (float)srest;
        const float invS2 = (float)(1.0 / (Sd * Sd));
        // C: criterion, mask, compaction of the selected keys
        float mrun = -INFINITY;
        uint32_t myword = 0u;
        int row_nsel = 0;
        const int nch = (nv + 31) >> 5;
        for (int t = 0; t < nch; ++t) {
          const int j = 32 * t + lane;
          const float y = row[j];
          const bool valid = j < nv;
          bool sel = false, near = false;
          float c = 0.f;
          if (given) {
            sel = valid && ((__ldg(p.mask_in + grow * nwords + t) >> lane) & 1u);
          } else {
            if (relaxed) {
              if ((t & 1) == 0) mrun = fmaxf(mrun, warp_max(fmaxf(y, row[j + 32])));
              c = 2.f * fabsf(y) * exp_fast(__fsub_rn(y, mrun));
            } else {
              const float e = (j == am) ? 1.f : exp_fast(__fsub_rn(y, m));
              const float om = (j == am) ? srest_f : __fsub_rn(Sf, e);
              c = (2.f * fabsf(y) * e) * (om * invS2);
            }
            sel = valid && c > p.tau;
            near = valid && refine_ok && (fabsf(c - p.tau) <= band || (p.tau == 0.f && c < 1e-30f));
          }
          if (__any_sync(0xFFFFFFFFu, near) && near) {
            double cd;
            if (relaxed) {
              cd = 2.0 * exp((double)y - (double)mrun) * fabs((double)y);
            } else {
              const double ed = (j == am) ? 1.0 : exp((double)y - (double)m);
              const double z = ed / Sd;
              const double omz = (j == am) ? srest / Sd : (Sd - ed) / Sd;
              cd = 2.0 * z * omz * fabs((double)y);
            }
            sel = cd > (double)p.tau;
          }
          if (p.ps_out && j < p.n_k) p.ps_out[grow * p.n_k + j] = valid ? y : -INFINITY;
          const uint32_t bal = __ballot_sync(0xFFFFFFFFu, sel);
          if ((t & 31) == lane) myword = bal;
          if (mrow && ((t & 31) == 31 || t == nch - 1)) {
            const int g0 = t & ~31;
            if (g0 + lane <= t) mrow[g0 + lane] = myword;
          }
          row_nsel += __popc(bal);
          if (sel) list[list_n + __popc(bal & lanemask_lt)] = (ri << 16) | j;
          list_n += __popc(bal);
          __syncwarp();
          if (list_n >= 32) flush(32);
        }
        if (mrow)
          for (int w = nch + lane; w < nwords; w += 32) mrow[w] = 0u;
        if (p.ps_out)
          for (int j = 32 * nch + lane; j < p.n_k; j += 32) p.ps_out[grow * p.n_k + j] = -INFINITY;
        warp_nsel += row_nsel;
      }
      if (list_n > 0) flush(list_n);
      __syncwarp();

      // D: softmax numerators P_j = exp(y_j - m') of the mixed row, written in place
      for (int ri = 0; ri < RPW; ++ri) {
        const int r = warp * RPW + ri;
        if (r >= rows) break;
        const int i = i0 + r;
        const int nv = n_valid_keys(i, p);
        float* row = sRows + (size_t)r * nkp;
        const size_t grow = (size_t)bh * p.n_q + i;
        // maximum of the mixed row (entries past the valid keys hold -inf)
        float m = -INFINITY;
        for (int it = 0; it < (nv + 127) >> 7; ++it) {
          const float4 v = *reinterpret_cast<const float4*>(row + 128 * it + 4 * lane);
          m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
        }
        m = warp_max(m);
        float l = 0.f;
        for (int t = 0; t < nch_kv; ++t) {
          const int j = 32 * t + lane;
          const float y = row[j];
          const float pj = j < nv ? exp_fast(__fsub_rn(y, m)) : 0.f;
          l += pj;
          if (p.mixed_out && j < p.n_k) p.mixed_out[grow * p.n_k + j] = j < nv ? y : -INFINITY;
          reinterpret_cast<uint32_t*>(row)[j] = p_pair(pj);
        }
        if (p.mixed_out)
          for (int j = 32 * nch_kv + lane; j < p.n_k; j += 32) p.mixed_out[grow * p.n_k + j] = -INFINITY;
        l = warp_sum(l);
        if (lane == 0) {
          sStat[4 * r] = m;
          sStat[4 * r + 1] = l;
          if (p.lse_out) p.lse_out[grow] = nv > 0 ? m + logf(l) : -INFINITY;
        }
      }
    }
    __syncthreads();

    // ---- phase 3: O = (P.V) / l on tensor cores ------------------------------------
    {
      constexpr int VK = v_keys<D>();
      constexpr int VS = D + 8;
      constexpr int MT = BM >= 16 ? BM / 16 : 1;
      constexpr int NH = D / 64;
      constexpr int KQ = NW / NH;
      constexpr int SPW = (VK / 8) / KQ;  // 8-key steps per warp per V chunk
      constexpr int TPG = 8 / KQ;         // n8 tiles per reduction group
      uint16_t* sV = reinterpret_cast<uint16_t*>(smem + L.kv);
      float* sO = reinterpret_cast<float*>(smem + L.kv);
      const int nh = NH == 2 ? (warp & 1) : 0;
      const int kq = NH == 2 ? (warp >> 1) : warp;
      const int mi = lane >> 3;
      float acc[MT][8][4];
#pragma unroll
      for (int rt = 0; rt < MT; ++rt)
#pragma unroll
        for (int tt = 0; tt < 8; ++tt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[rt][tt][e] = 0.f;
      const int nvc = (kv_end + VK - 1) / VK;
      auto load_v = [&](int vc, int buf) {
        uint16_t* dst = sV + buf * VK * VS;
        for (int u = tid; u < VK * (D / 8); u += NT) {
          const int key = u / (D / 8), ch = u % (D / 8);
          const int gkey = vc * VK + key;
          uint16_t* d = dst + key * VS + ch * 8;
          if (gkey < p.n_k) cp_async16(d, Vh + (size_t)gkey * D + ch * 8);
          else *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
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
        __syncthreads();
        const uint16_t* vb = sV + (vc & 1) * VK * VS;
#pragma unroll
        for (int q = 0; q < SPW; ++q) {
          const int st = kq + KQ * q;
          const int kb = vc * VK + 8 * st;
          if (kb < kv_end) {
            uint32_t af[MT][4];
#pragma unroll
            for (int rt = 0; rt < MT; ++rt) {
              int rr = rt * 16 + 8 * (mi & 1) + (lane & 7);
              if (BM < 16) rr &= BM - 1;
              ldmatrix_x4(smem_u32(sRows + (size_t)rr * nkp + kb + 4 * (mi >> 1)), af[rt][0], af[rt][1],
                          af[rt][2], af[rt][3]);
            }
            const int kl = 8 * st + 4 * (mi & 1) + ((lane & 7) >> 1);
#pragma unroll
            for (int nb = 0; nb < 4; ++nb) {
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4_trans(smem_u32(vb + kl * VS + nh * 64 + 16 * nb + 8 * (mi >> 1)), b0, b1, b2, b3);
#pragma unroll
              for (int rt = 0; rt < MT; ++rt) {
                mma_bf16_16816(acc[rt][2 * nb], af[rt][0], af[rt][1], af[rt][2], af[rt][3], b0, b1);
                mma_bf16_16816(acc[rt][2 * nb + 1], af[rt][0], af[rt][1], af[rt][2], af[rt][3], b2, b3);
              }
            }
          }
        }
        __syncthreads();
      }
      // partial sums of the KQ key groups, added in a fixed order
#pragma unroll
      for (int rho = 0; rho < KQ; ++rho) {
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
          if ((tt / TPG - kq - rho + 2 * KQ) % KQ == 0) {
#pragma unroll
            for (int rt = 0; rt < MT; ++rt) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int rr = rt * 16 + (lane >> 2) + 8 * h;
                if (rr < BM) {
                  float2* dst = reinterpret_cast<float2*>(sO + rr * D + nh * 64 + 8 * tt + 2 * (lane & 3));
                  const float2 v = make_float2(acc[rt][tt][2 * h], acc[rt][tt][2 * h + 1]);
                  if (rho == 0) {
                    *dst = v;
                  } else {
                    const float2 o = *dst;
                    *dst = make_float2(o.x + v.x, o.y + v.y);
                  }
                }
              }
            }
          }
        }
        __syncthreads();
      }
      for (int u = tid; u < BM * D / 2; u += NT) {
        const int rr = u / (D / 2), col = (u % (D / 2)) * 2;
        if (rr >= rows) continue;
        const float l = sStat[4 * rr + 1];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float2 o = *reinterpret_cast<const float2*>(sO + rr * D + col);
        const float v0 = nvc > 0 ? o.x * inv : 0.f, v1 = nvc > 0 ? o.y * inv : 0.f;
        const size_t off = ((size_t)bh * p.n_q + i0 + rr) * D + col;
        *reinterpret_cast<uint32_t*>(p.out + off) =
            (uint32_t)f32_to_bf16_rne(v0) | ((uint32_t)f32_to_bf16_rne(v1) << 16);
        if (p.out_f32) *reinterpret_cast<float2*>(p.out_f32 + off) = make_float2(v0, v1);
      }
    }
    __syncthreads();
  }
  if (lane == 0 && warp_nsel && p.nsel_out) atomicAdd(p.nsel_out, (unsigned long long)warp_nsel);
}

template <int D, int BM, int RND>
cudaError_t launch_one(const RowsArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto k = rows_kernel<D, BM, RND>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, NT, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D, int BM>
cudaError_t launch_bm(const RowsArgs& a, int rnd, int grid, size_t smem, cudaStream_t st) {
  if (rnd == kRndFast) return launch_one<D, BM, kRndFast>(a, grid, smem, st);
  if (rnd == kRndNone) return launch_one<D, BM, kRndNone>(a, grid, smem, st);
  return launch_one<D, BM, kRndExact>(a, grid, smem, st);
}

template <int D>
size_t plan_bytes(int bm, int nkp) {
  if (bm == 32) return (size_t)smem_plan<D, 32>(nkp).total;
  if (bm == 16) return (size_t)smem_plan<D, 16>(nkp).total;
  return (size_t)smem_plan<D, 8>(nkp).total;
}

}  // namespace

int rows_nkp(int bm, int n_k) {
  const int bn = 4096 / bm;
  return ((n_k + bn - 1) / bn) * bn + 4;
}

size_t rows_smem_bytes(int d, int bm, int n_k) {
  const int nkp = rows_nkp(bm, n_k);
  return d == 64 ? plan_bytes<64>(bm, nkp) : plan_bytes<128>(bm, nkp);
}

int rows_pick_bm(int d, int n_k, size_t smem_optin) {
  if (n_k > 0xFFFF) return 0;  // keys are packed in 16 bits in the recompute lists
  for (int bm = 32; bm >= 8; bm /= 2)
    if (rows_smem_bytes(d, bm, n_k) + kStaticSmemReserve <= smem_optin) return bm;
  return 0;
}

cudaError_t launch_rows(const Problem& p, const Workspace& ws, char* base, int num_sms, cudaStream_t st) {
  RowsArgs a;
  a.p = p;
  a.stats = reinterpret_cast<const int*>(base + ws.stats);
  a.nchunk = ws.nchunk;
  a.counter = reinterpret_cast<uint32_t*>(base + ws.counters);
  const int bm = ws.rows_bm;
  a.nkp = rows_nkp(bm, p.n_k);
  a.n_rb = (p.n_q + bm - 1) / bm;
  a.n_items = a.n_rb * p.B * p.H;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  const size_t smem = rows_smem_bytes(p.d, bm, p.n_k);
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  if (p.d == 64) {
    if (bm == 32) return launch_bm<64, 32>(a, rnd, grid, smem, st);
    if (bm == 16) return launch_bm<64, 16>(a, rnd, grid, smem, st);
    return launch_bm<64, 8>(a, rnd, grid, smem, st);
  }
  if (bm == 32) return launch_bm<128, 32>(a, rnd, grid, smem, st);
  if (bm == 16) return launch_bm<128, 16>(a, rnd, grid, smem, st);
  return launch_bm<128, 8>(a, rnd, grid, smem, st);
}

}  // namespace lamp
