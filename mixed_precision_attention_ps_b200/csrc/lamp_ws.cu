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
//     keys are cut into 64-key units dealt round-robin to the producer warps,
//     continuing across items. Each warp stages its own K slices (8 head
//     dimensions x 64 keys, binary32, double buffered) and waits for nothing but
//     a free buffer. A lane holds 8 rows x 4 keys as sixteen packed binary32
//     pairs (two rows of one key per 64-bit register): one accumulation step is
//     fma.rn.f32x2 plus the two-instruction PS(mu) rounding (or the exact
//     integer rounding), and three shared-memory loads feed 16 packed steps.
//   consumers (warps 8-15): for item k, two rows per warp, four keys per lane:
//     row maximum and first argmax, S_rest in double (strict), the criterion
//     with a double re-evaluation near tau, mask words, warp-compacted FP32
//     recompute, softmax numerators of the mixed row written in place as bf16
//     hi/lo pairs; then P.V on tensor cores (mma.sync, V staged by cp.async), the
//     output, and the staging of Q for item k + 2.
//
// Hand-offs use mbarriers: full[b] (256 producer arrivals per item) and empty[b]
// (256 consumer arrivals: the buffer and its Q are ready for the next item).
// Every wait is bounded; a wait that gives up records LAMP_ERR_TIMEOUT in the
// caller's status word (when given) and ends the kernel.
#include <cfloat>

#include "lamp_ws_common.cuh"

namespace lamp {
namespace {

struct WsSmem {
  int bars;   // mbarriers: full[2], empty[2]
  int q;      // Q [2][D][16] f32
  int ks;     // producer K slices [8 warps][2][8][64] f32
  int v;      // consumer V rings [8 warps][WR][8][72] bf16, later the partial outputs [KQ][16][D] f32
  int list;   // consumer mask-word buffers [8][2][32] uint32
  int stats;  // per buffer and row: softmax max, normaliser [2][16][2] f32
  int rows;   // score rows [2][16][nkp] f32
  int total;
};

template <int D>
__host__ __device__ inline WsSmem ws_plan(int nkp) {
  WsSmem s{};
  s.bars = 0;
  s.q = 64;
  s.ks = s.q + 2 * ws_qfloats<D>() * 4;
  s.v = s.ks + WS_NP * 2 * WS_DS * WS_UNIT * 4;
  const int vb = WS_NC * ws_vring<D>() * 8 * WS_VSW * 2;  // per-warp V rings
  const int ob = (WS_NC / (D / 64)) * WS_BM * D * 4;  // per-warp partial outputs
  s.list = s.v + (vb > ob ? vb : ob);
  s.stats = s.list + WS_NC * 2 * SEL_WMAX * 4;
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

// ---------------------------------------------------------------------------
// Producers: PS(mu) scores of every item into the item's row buffer.
// ---------------------------------------------------------------------------
template <int D, int RND>
__device__ __forceinline__ void ws_producer(const WsArgs& a, unsigned char* smem, const WsSmem& L, int warp,
                                            int lane) {
  const Problem& p = a.p;
  const int G = gridDim.x, cta = blockIdx.x;
  const int s = 23 - p.mu;
  const u64 negc = pack2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const u64 pow2s = pack2((float)(1u << s), (float)(1u << s));
  const u64 scale2 = pack2(p.scale, p.scale);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);  // full[0], full[1], empty[0], empty[1]
  float* ksw = reinterpret_cast<float*>(smem + L.ks) + warp * 2 * WS_DS * WS_UNIT;
  int deal = 0;  // producer warp that takes the next unit
  for (int k = 0;; ++k) {
    const int q = ws_item(k, cta, G, a.n_items);
    if (q < 0) break;
    const int buf = k & 1;
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    // one decision per warp: the tile routine synchronises the whole warp
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(bars + 2 + buf, (k >> 1) & 1))) {  // buffer free, Q staged
      ws_timeout(p);
      return;
    }
    const float* sQ = reinterpret_cast<const float*>(smem + L.q) + buf * ws_qfloats<D>();
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    float* rows = reinterpret_cast<float*>(smem + L.rows) + (size_t)buf * WS_BM * a.nkp;
    const int U = (it.kv_end + WS_UNIT - 1) / WS_UNIT;
    ws_produce_tile<D, RND>(p, it, 0, it.kv_end, sQ, rows, a.nkp, ksw, lane, (warp - deal + WS_NP) % WS_NP, fast, Kh,
                            negc, pow2s, scale2, s);
    deal = (deal + U) % WS_NP;
    mbar_arrive(bars + buf);  // this thread's scores of item k are in place
  }
}

// ---------------------------------------------------------------------------
// Consumers: selection, recompute, softmax, P.V and the output of every item.
// ---------------------------------------------------------------------------
template <int D, int RND, int VAR>
__device__ __forceinline__ void ws_consumer(const WsArgs& a, unsigned char* smem, const WsSmem& L, int cw,
                                            int lane) {
  constexpr int NH = D / 64;
  constexpr int KQ = WS_NC / NH;
  constexpr int WR = ws_vring<D>();
  constexpr int NCT = WS_NC * 32;  // consumer threads
  const Problem& p = a.p;
  const int tidc = cw * 32 + lane;
  const int G = gridDim.x, cta = blockIdx.x;
  const int nwords = (p.n_k + 31) >> 5;
  const bool refine_ok = VAR != LAMP_GIVEN_MASK && isfinite(p.tau) && p.tau >= 0.f;
  const float band = WS_BAND * p.tau;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(smem + L.list) + cw * 2 * SEL_WMAX;
  uint16_t* sV = reinterpret_cast<uint16_t*>(smem + L.v);
  float* sO = reinterpret_cast<float*>(smem + L.v);
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  long long nsel = 0;
  // Q of the first two items, then both buffers are released to the producers
  for (int k0 = 0; k0 < 2; ++k0) {
    const int q0 = ws_item(k0, cta, G, a.n_items);
    if (q0 < 0) break;
    ws_stage_q<D>(qbase + k0 * ws_qfloats<D>(), p, ws_decode(q0, p, a.n_rb), tidc, NCT);
    mbar_arrive(bars + 2 + k0);
  }
  for (int k = 0;; ++k) {
    const int q = ws_item(k, cta, G, a.n_items);
    if (q < 0) break;
    const int buf = k & 1;
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    const uint16_t* Vh = p.V + (size_t)it.bh * p.n_k * D;
    // P.V split: warp (kq, nh) takes the 8-key steps kq, kq + KQ, ... of the row and
    // the value columns nh*64 .. nh*64 + 63. It stages exactly those V rows in a
    // ring of WR steps of its own (cp.async, one group per step, empty groups past
    // the end), so the P.V loop needs no group barrier.
    const int nh = NH == 2 ? (cw & 1) : 0;
    const int kq = NH == 2 ? (cw >> 1) : cw;
    const int ns_all = (it.kv_end + 7) >> 3;
    const int nsw = ns_all > kq ? (ns_all - kq + KQ - 1) / KQ : 0;  // this warp's steps
    uint16_t* vring = sV + cw * WR * 8 * WS_VSW;
    auto load_step = [&](int i) {  // step i of this warp into ring slot i % WR
      if (i < nsw) {
        const int key0 = 8 * (kq + KQ * i);
        uint16_t* dst = vring + (i % WR) * 8 * WS_VSW;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = lane + 32 * h, key = c >> 3, ch = c & 7;
          uint16_t* dd = dst + key * WS_VSW + ch * 8;
          if (key0 + key < p.n_k) cp_async16(dd, Vh + (size_t)(key0 + key) * D + nh * 64 + ch * 8);
          else *reinterpret_cast<uint4*>(dd) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      cp_async_commit();
    };
    for (int i = 0; i < WR - 1; ++i) load_step(i);  // V does not depend on the scores

    const bool ok = mbar_wait(bars + buf, (k >> 1) & 1);
    if (named_or(BAR_CONS, NCT, !ok)) {
      ws_timeout(p);
      cp_async_wait<0>();
      return;
    }
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    float* sQ = qbase + buf * ws_qfloats<D>();
    float* rows = reinterpret_cast<float*>(smem + L.rows) + (size_t)buf * WS_BM * a.nkp;
    float* st = reinterpret_cast<float*>(smem + L.stats) + buf * WS_BM * 2;
    const int written = ((it.kv_end + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;  // keys the producers wrote

    // ---- selection and recompute, rows 2cw and 2cw + 1 ------------------------------
    // Keys past a row's valid range hold -inf: their criterion is NaN, which no
    // comparison selects, so the hot loops need no validity test.
    int rr_[2], nv[2];
    size_t grow[2];
    float* row[2];
    SelRows S;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      rr_[t] = 2 * cw + t;
      nv[t] = rr_[t] < it.rows ? ws_valid_keys(it.i0 + rr_[t], p) : 0;
      grow[t] = (size_t)it.bh * p.n_q + it.i0 + rr_[t];
      row[t] = rows + (size_t)rr_[t] * a.nkp;
      S.row[t] = row[t];
      S.nv[t] = nv[t];
      S.word0[t] = grow[t] * nwords;
      S.live[t] = rr_[t] < it.rows;
      S.mx[t] = -INFINITY;
      S.mrun[t] = -INFINITY;
    }
    const int nvmax = max(nv[0], nv[1]);
    const int nit = (nvmax + 127) >> 7;
    if (p.ps_out) {  // dump of the low-precision scores (before any recompute)
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (rr_[t] < it.rows)
          for (int j = lane; j < p.n_k; j += 32) p.ps_out[grow[t] * p.n_k + j] = j < written ? row[t][j] : -INFINITY;
    }
    if (VAR == LAMP_STRICT) {
      // A: maximum and first argmax of each row
      float m[2] = {-INFINITY, -INFINITY};
      int am[2] = {0x7FFFFFFF, 0x7FFFFFFF};
      for (int i4 = 0; i4 < nit; ++i4) {
        const int j0 = 128 * i4 + 4 * lane;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const float4 v = lds4_or_ninf(row[t] + j0, j0 < written);
          if (v.x > m[t]) { m[t] = v.x; am[t] = j0; }
          if (v.y > m[t]) { m[t] = v.y; am[t] = j0 + 1; }
          if (v.z > m[t]) { m[t] = v.z; am[t] = j0 + 2; }
          if (v.w > m[t]) { m[t] = v.w; am[t] = j0 + 3; }
        }
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float mw = warp_max_redux(m[t]);
        am[t] = __reduce_min_sync(0xFFFFFFFFu, m[t] == mw ? am[t] : 0x7FFFFFFF);
        m[t] = mw;
      }
      // B: S_rest = sum_{j != argmax} exp(y_j - m) in double, two chains per row
      double sa[2] = {0.0, 0.0}, sb[2] = {0.0, 0.0};
      for (int i4 = 0; i4 < nit; ++i4) {
        const int j0 = 128 * i4 + 4 * lane;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          float4 v = lds4_or_ninf(row[t] + j0, j0 < written);
          if (j0 == (am[t] & ~3)) {  // the argmax itself is not part of S_rest
            const int e = am[t] & 3;
            if (e == 0) v.x = -INFINITY;
            else if (e == 1) v.y = -INFINITY;
            else if (e == 2) v.z = -INFINITY;
            else v.w = -INFINITY;
          }
          // exp(y - m) as 2^(y log2 e - m log2 e) on the special-function unit
          // (relative error about 2^-22, the selection pass's form): S_rest then
          // carries a few 1e-7 relative error, inside the criterion's double band
          const float ml = m[t] * kLog2e;
          float e0, e1, e2, e3;
          asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(fmaf(v.x, kLog2e, -ml)));
          asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(fmaf(v.y, kLog2e, -ml)));
          asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e2) : "f"(fmaf(v.z, kLog2e, -ml)));
          asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e3) : "f"(fmaf(v.w, kLog2e, -ml)));
          sa[t] += (double)e0 + (double)e1;
          sb[t] += (double)e2 + (double)e3;
        }
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const double srest = warp_sum_d(sa[t] + sb[t]);
        S.m[t] = m[t];
        S.am[t] = am[t];
        S.srest[t] = srest;
        S.Sd[t] = 1.0 + srest;
        S.Sf[t] = (float)S.Sd[t];
        S.srest_f[t] = (float)srest;
        S.c2[t] = (float)(2.0 / (S.Sd[t] * S.Sd[t]));
        S.mL[t] = m[t] * kLog2e;
      }
    }
    // C: criterion, mask words, compaction and recompute of the selected keys
    const float tlo = refine_ok ? p.tau - band : INFINITY;
    const float thi = refine_ok ? (p.tau == 0.f ? 1e-30f : p.tau + band) : -INFINITY;
    for (int i4 = 0; i4 < nit; ++i4) sel_step<VAR>(p, S, 128 * i4, written, nwords, tlo, thi, lane, wbuf, nsel);
    sel_finish(p, S, wbuf, 4 * nit, nwords, lane, [&](int t, int j) {
      const float v = ws_recompute<D>(sQ, 2 * cw + t, Kh + (size_t)j * D, p.scale, fast);
      rows[(size_t)(2 * cw + t) * a.nkp + j] = v;
      if (t == 0) S.mx[0] = fmaxf(S.mx[0], v);
      else S.mx[1] = fmaxf(S.mx[1], v);
    });
    __syncwarp();
    if (p.mixed_out) {  // dump of the mixed scores
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (rr_[t] < it.rows)
          for (int j = lane; j < p.n_k; j += 32)
            p.mixed_out[grow[t] * p.n_k + j] = j < written ? row[t][j] : -INFINITY;
    }

    // D: softmax numerators of the mixed rows, in place; the maximum m' of each
    // mixed row was tracked through the selection and the recompute
    const int nitw = (written + 127) >> 7;
    float mm[2], mL[2], l[2] = {0.f, 0.f};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      mm[t] = warp_max_redux(S.mx[t]);
      mL[t] = mm[t] == -INFINITY ? 0.f : mm[t] * kLog2e;
    }
    for (int i4 = 0; i4 < nitw; ++i4) {
      const int j0 = 128 * i4 + 4 * lane;
      if (j0 >= written) continue;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float4 v = *reinterpret_cast<const float4*>(row[t] + j0);
        const float vv[4] = {v.x, v.y, v.z, v.w};
        uint32_t pw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float pj;  // exp(y - m'), 0 for -inf
          asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(pj) : "f"(fmaf(vv[e], kLog2e, -mL[t])));
          l[t] += pj;
          pw[e] = p_pair_cvt(pj);
        }
        *reinterpret_cast<uint4*>(row[t] + j0) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      l[t] = warp_sum(l[t]);
      if (lane == 0) {
        st[2 * rr_[t]] = mm[t];
        st[2 * rr_[t] + 1] = l[t];
        if (p.lse_out && rr_[t] < it.rows) p.lse_out[grow[t]] = nv[t] > 0 ? mm[t] + logf(l[t]) : -INFINITY;
      }
    }
    named_sync(BAR_CONS, NCT);  // every P row of the item is in place

    // ---- O = (P.V) / l on tensor cores ----------------------------------------------
    const int mi = lane >> 3;
    float acc[8][4];
#pragma unroll
    for (int tt = 0; tt < 8; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tt][e] = 0.f;
    const int ra = 8 * (mi & 1) + (lane & 7);
    const int kl = 4 * (mi & 1) + ((lane & 7) >> 1);  // each V row serves the hi and the lo half of P
    for (int i = 0; i < nsw; ++i) {
      cp_async_wait<WR - 2>();  // step i has landed (this lane's copies)
      __syncwarp();             // ... and every lane's; step i - 1's slot is free
      load_step(i + WR - 1);
      const int kb = 8 * (kq + KQ * i);
      const uint16_t* vb = vring + (i % WR) * 8 * WS_VSW;
      uint32_t af[4];
      ldmatrix_x4(smem_u32(rows + (size_t)ra * a.nkp + kb + 4 * (mi >> 1)), af[0], af[1], af[2], af[3]);
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(smem_u32(vb + kl * WS_VSW + 16 * nb + 8 * (mi >> 1)), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * nb], af[0], af[1], af[2], af[3], b0, b1);
        mma_bf16_16816(acc[2 * nb + 1], af[0], af[1], af[2], af[3], b2, b3);
      }
    }
    cp_async_wait<0>();
    named_sync(BAR_CONS, NCT);  // every warp is done with the V stages (the partial sums reuse them)
    // each warp's partial sums go to a slot of their own; then one pass adds the KQ
    // slots of every output in a fixed order (deterministic) and scales by 1 / l
#pragma unroll
    for (int tt = 0; tt < 8; ++tt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rr = (lane >> 2) + 8 * h;
        *reinterpret_cast<float2*>(sO + ((size_t)kq * WS_BM + rr) * D + nh * 64 + 8 * tt + 2 * (lane & 3)) =
            make_float2(acc[tt][2 * h], acc[tt][2 * h + 1]);
      }
    named_sync(BAR_CONS, NCT);
    for (int u = tidc; u < WS_BM * D / 2; u += NCT) {
      const int rr = u / (D / 2), col = (u % (D / 2)) * 2;
      if (rr >= it.rows) continue;
      float2 o = *reinterpret_cast<const float2*>(sO + rr * D + col);
#pragma unroll
      for (int g = 1; g < KQ; ++g) {
        const float2 v = *reinterpret_cast<const float2*>(sO + ((size_t)g * WS_BM + rr) * D + col);
        o.x += v.x;
        o.y += v.y;
      }
      const float lv = st[2 * rr + 1];
      const float inv = lv > 0.f ? 1.f / lv : 0.f;
      const float v0 = o.x * inv, v1 = o.y * inv;
      const size_t off = ((size_t)it.bh * p.n_q + it.i0 + rr) * D + col;
      *reinterpret_cast<uint32_t*>(p.out + off) =
          (uint32_t)f32_to_bf16_rne(v0) | ((uint32_t)f32_to_bf16_rne(v1) << 16);
      if (p.out_f32) *reinterpret_cast<float2*>(p.out_f32 + off) = make_float2(v0, v1);
    }
    named_sync(BAR_CONS, NCT);  // the output sums (V area) and this item's Q are no longer read
    const int q2 = ws_item(k + 2, cta, G, a.n_items);
    if (q2 >= 0) ws_stage_q<D>(sQ, p, ws_decode(q2, p, a.n_rb), tidc, NCT);
    mbar_arrive(bars + 2 + buf);  // buffer free (and Q of item k + 2 staged)
  }
  if (lane == 0 && nsel && p.nsel_out) atomicAdd(p.nsel_out, (unsigned long long)nsel);
}

template <int D, int RND, int VAR>
__global__ void __launch_bounds__(WS_NT, 1) ws_kernel(const WsArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const WsSmem L = ws_plan<D>(a.nkp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
    mbar_init(bars + 0, WS_NP * 32);  // full[0]
    mbar_init(bars + 1, WS_NP * 32);  // full[1]
    mbar_init(bars + 2, WS_NC * 32);  // empty[0]
    mbar_init(bars + 3, WS_NC * 32);  // empty[1]
    mbar_fence_init();
  }
  __syncthreads();
  if (warp < WS_NP) ws_producer<D, RND>(a, smem, L, warp, lane);
  else ws_consumer<D, RND, VAR>(a, smem, L, warp - WS_NP, lane);
}

template <int D, int RND, int VAR>
cudaError_t ws_launch_one(const WsArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto k = ws_kernel<D, RND, VAR>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, WS_NT, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D, int RND>
cudaError_t ws_launch_var(const WsArgs& a, int grid, size_t smem, cudaStream_t st) {
  if (a.p.variant == LAMP_RELAXED) return ws_launch_one<D, RND, LAMP_RELAXED>(a, grid, smem, st);
  if (a.p.variant == LAMP_GIVEN_MASK) return ws_launch_one<D, RND, LAMP_GIVEN_MASK>(a, grid, smem, st);
  return ws_launch_one<D, RND, LAMP_STRICT>(a, grid, smem, st);
}

}  // namespace

int ws_nkp(int n_k) { return ((n_k + 127) / 128) * 128 + 4; }

size_t ws_smem_bytes(int d, int n_k) {
  const int nkp = ws_nkp(n_k);
  return d == 64 ? (size_t)ws_plan<64>(nkp).total : (size_t)ws_plan<128>(nkp).total;
}

bool ws_fits(int d, int n_k, size_t smem_optin) {
  return n_k <= 32 * SEL_WMAX && ws_smem_bytes(d, n_k) + kStaticSmemReserve <= smem_optin;
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
    if (rnd == kRndFast) return ws_launch_var<64, kRndFast>(a, grid, smem, st);
    if (rnd == kRndNone) return ws_launch_var<64, kRndNone>(a, grid, smem, st);
    return ws_launch_var<64, kRndExact>(a, grid, smem, st);
  }
  if (rnd == kRndFast) return ws_launch_var<128, kRndFast>(a, grid, smem, st);
  if (rnd == kRndNone) return ws_launch_var<128, kRndNone>(a, grid, smem, st);
  return ws_launch_var<128, kRndExact>(a, grid, smem, st);
}

}  // namespace lamp
