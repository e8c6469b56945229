// LAMP attention, streamed one-pass kernel for the relaxed and given-mask
// variants at any row length (the 16K-token shape): scores are produced and
// consumed in tiles of 512 keys with an online softmax, so no complete row is
// ever stored.
//
// Method ("LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models",
// technical summary, gist.science paper 2601.21623), section "Experimental
// results": the relaxed relative-threshold test needs no normalising constant,
// which keeps the softmax one-pass (FlashAttention style); the test here is
// c_j = 2 exp(y_j - M_t) |y_j| > tau with M_t the running maximum of the
// low-precision scores over 64-key tiles counted from key 0. Section
// "Implementation strategy", steps 1-3: low-precision baseline, selection from
// it, FP32 recompute of the selection before the softmax.
//
// Same organisation as the whole-row warp-specialised kernel: one persistent CTA
// of 512 threads per SM, items (b, h, 16 query rows) in a snake order, producer
// warps 0-7 fill tile buffers (64-key units dealt round-robin, PS(mu) steps as
// packed binary32 pairs), consumer warps 8-15 take each tile: the relaxed
// criterion (double re-evaluation near tau), mask words, warp-compacted FP32
// recompute from K in global memory, then the online softmax (running maximum m
// and normaliser l per row; the per-warp partial outputs are rescaled by
// exp(m_old - m_new) before each tile's P.V on tensor cores). After an item's
// last tile the partial outputs are added in a fixed order and divided by l.
// Hand-offs per tile use mbarriers (full[b], empty[b]); every wait is bounded.
#include <cfloat>

#include "lamp_ws_common.cuh"

namespace lamp {
namespace {

constexpr int ST_T = 512;   // keys per streamed tile
constexpr int ST_TS = ST_T + 4;  // tile row stride (floats): 16-byte steps across banks


struct StSmem {
  int bars;   // mbarriers: full[2], empty[2]
  int q;      // Q [2][D][16] f32, by item parity
  int ks;     // producer K slices [8 warps][2][8][64] f32
  int v;      // consumer V rings [8 warps][WR][8][72] bf16, later the partial outputs [KQ][16][D] f32
  int list;   // consumer mask-word buffers [8][2][32] uint32
  int rstat;  // per row: m, l, alpha, spare [16][4] f32
  int tiles;  // score tiles [2][16][ST_TS] f32
  int total;
};

template <int D>
__host__ __device__ inline StSmem st_plan() {
  StSmem s{};
  s.bars = 0;
  s.q = 64;
  s.ks = s.q + 2 * ws_qfloats<D>() * 4;
  s.v = s.ks + WS_NP * 2 * WS_DS * WS_UNIT * 4;
  const int vb = WS_NC * ws_vring<D>() * 8 * WS_VSW * 2;  // per-warp V rings
  const int ob = (WS_NC / (D / 64)) * WS_BM * D * 4;
  s.list = s.v + (vb > ob ? vb : ob);
  s.rstat = s.list + WS_NC * 2 * SEL_WMAX * 4;
  s.tiles = s.rstat + WS_BM * 4 * 4;
  s.total = s.tiles + 2 * WS_BM * ST_TS * 4;
  return s;
}

// Strict rows too long for whole-row buffers run in two passes of this kernel
// (template parameter PH):
//   PH 0: one pass (relaxed, given mask);
//   PH 1: strict statistics: the producers compute the scores; the consumers store
//         every tile to an HBM score slab and keep, per row, the maximum m, its
//         first key am and S_rest = sum over the other keys of exp(y - m) online
//         across tiles (tile maximum and sum, merged in double);
//   PH 2: strict selection: the producers refill the tile buffers from the slab;
//         the consumers run the strict test with the row statistics of pass 1,
//         then recompute, online softmax and P.V as in PH 0.
struct RowStat {
  float m;      // maximum of the row's low-precision scores (-inf if none valid)
  int am;       // its first key
  double srest; // sum over the other keys of exp(y - m)
};

struct StArgs {
  Problem p;
  const int* stats;  // per-(b, h) exponent statistics
  int nchunk;
  int n_items;
  int n_rb;
  float* slab;       // strict: low-precision scores [B*H][n_q][ld]
  size_t ld;         // slab row stride (keys rounded up to whole tiles)
  RowStat* rows;     // strict: [B*H][n_q]
};

__device__ __forceinline__ int st_ntiles(int kv_end) { return kv_end > 0 ? (kv_end + ST_T - 1) / ST_T : 1; }

// ---------------------------------------------------------------------------
// Producers: every tile of every item, in the order the consumers take them.
// ---------------------------------------------------------------------------
template <int D, int RND, int PH>
__device__ __forceinline__ void st_producer(const StArgs& a, unsigned char* smem, const StSmem& L, int warp,
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
  int k = 0;     // tile counter: buffer k & 1, phase k >> 1
  for (int ii = 0;; ++ii) {
    const int q = ws_item(ii, cta, G, a.n_items);
    if (q < 0) break;
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    const float* sQ = reinterpret_cast<const float*>(smem + L.q) + (ii & 1) * ws_qfloats<D>();
    const int nt = st_ntiles(it.kv_end);
    for (int t = 0; t < nt; ++t, ++k) {
      const int buf = k & 1;
      const int t0 = t * ST_T;
      const int tlen = max(0, min(ST_T, it.kv_end - t0));
      // one decision per warp: the tile routine synchronises the whole warp
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bars + 2 + buf, (k >> 1) & 1))) {  // tile buffer free (and the item's Q staged)
        ws_timeout(p);
        return;
      }
      float* tile = reinterpret_cast<float*>(smem + L.tiles) + (size_t)buf * WS_BM * ST_TS;
      if (PH == 2) {
        // the tile's scores from the slab: rows of the item by cp.async, keys of the
        // tile that the scores pass wrote; rows past the item hold -inf
        const int written = ((tlen + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;
        const int per_row = written / 4;  // 16-byte pieces
        for (int u = warp * 32 + lane; u < WS_BM * per_row; u += WS_NP * 32) {
          const int r = u / per_row, c4 = u % per_row;
          float* dst = tile + (size_t)r * ST_TS + 4 * c4;
          if (r < it.rows)
            cp_async16(dst, a.slab + ((size_t)it.bh * p.n_q + it.i0 + r) * a.ld + t0 + 4 * c4);
          else
            *reinterpret_cast<float4*>(dst) = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
        cp_async_commit();
        cp_async_wait<0>();
      } else {
        ws_produce_tile<D, RND>(p, it, t0, tlen, sQ, tile, ST_TS, ksw, lane, (warp - deal + WS_NP) % WS_NP, fast,
                                Kh, negc, pow2s, scale2, s);
        deal = (deal + (tlen + WS_UNIT - 1) / WS_UNIT) % WS_NP;
      }
      mbar_arrive(bars + buf);  // this thread's scores of the tile are in place
    }
  }
}

// ---------------------------------------------------------------------------
// Consumers: selection, recompute, online softmax and P.V, tile by tile.
// ---------------------------------------------------------------------------
template <int D, int RND, int VAR, int PH>
__device__ __forceinline__ void st_consumer(const StArgs& a, unsigned char* smem, const StSmem& L, int cw,
                                            int lane) {
  constexpr int NH = D / 64;
  constexpr int KQ = WS_NC / NH;
  constexpr int WR = ws_vring<D>();
  constexpr int NCT = WS_NC * 32;
  const Problem& p = a.p;
  const int tidc = cw * 32 + lane;
  const int G = gridDim.x, cta = blockIdx.x;
  const int nwords = (p.n_k + 31) >> 5;
  const bool refine_ok = VAR != LAMP_GIVEN_MASK && isfinite(p.tau) && p.tau >= 0.f;
  const float band = WS_BAND * p.tau;
  const float tlo = refine_ok ? p.tau - band : INFINITY;
  const float thi = refine_ok ? (p.tau == 0.f ? 1e-30f : p.tau + band) : -INFINITY;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(smem + L.list) + cw * 2 * SEL_WMAX;
  uint16_t* sV = reinterpret_cast<uint16_t*>(smem + L.v);
  float* sO = reinterpret_cast<float*>(smem + L.v);
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  float* rst = reinterpret_cast<float*>(smem + L.rstat);
  const int nh = NH == 2 ? (cw & 1) : 0;
  const int kq = NH == 2 ? (cw >> 1) : cw;
  const int mi = lane >> 3;
  uint16_t* vring = sV + cw * WR * 8 * WS_VSW;
  long long nsel = 0;
  // Q of the first two items; both tile buffers start out free
  for (int k0 = 0; k0 < 2; ++k0) {
    const int q0 = ws_item(k0, cta, G, a.n_items);
    if (q0 < 0) break;
    ws_stage_q<D>(qbase + k0 * ws_qfloats<D>(), p, ws_decode(q0, p, a.n_rb), tidc, NCT);
  }
  mbar_arrive(bars + 2);
  mbar_arrive(bars + 3);
  int k = 0;
  for (int ii = 0;; ++ii) {
    const int q = ws_item(ii, cta, G, a.n_items);
    if (q < 0) break;
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    const uint16_t* Vh = p.V + (size_t)it.bh * p.n_k * D;
    float* sQ = qbase + (ii & 1) * ws_qfloats<D>();
    const int nt = st_ntiles(it.kv_end);
    int rr_[2], nv[2];
    size_t grow[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      rr_[t] = 2 * cw + t;
      nv[t] = rr_[t] < it.rows ? ws_valid_keys(it.i0 + rr_[t], p) : 0;
      grow[t] = (size_t)it.bh * p.n_q + it.i0 + rr_[t];
    }
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    SelRows S;
    int am_abs[2] = {0x7FFFFFFF, 0x7FFFFFFF};  // strict: first key of each row's maximum
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      S.live[tt] = rr_[tt] < it.rows;
      S.mrun[tt] = -INFINITY;
      if (VAR == LAMP_STRICT) {  // the row statistics of the scores pass
        RowStat rs;
        rs.m = -INFINITY;
        rs.am = 0x7FFFFFFF;
        rs.srest = 0.0;
        if (rr_[tt] < it.rows) rs = a.rows[grow[tt]];
        am_abs[tt] = rs.am;
        S.m[tt] = rs.m;
        S.srest[tt] = rs.srest;
        S.Sd[tt] = 1.0 + rs.srest;
        S.Sf[tt] = (float)S.Sd[tt];
        S.srest_f[tt] = (float)rs.srest;
        S.c2[tt] = (float)(2.0 / (S.Sd[tt] * S.Sd[tt]));
        S.mL[tt] = rs.m * kLog2e;
      }
    }
    float acc[8][4];
#pragma unroll
    for (int tt = 0; tt < 8; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tt][e] = 0.f;

    for (int t = 0; t < nt; ++t, ++k) {
      const int buf = k & 1;
      const int t0 = t * ST_T;
      const int tlen = max(0, min(ST_T, it.kv_end - t0));
      const int written = ((tlen + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;  // keys the producers wrote
      float* tile = reinterpret_cast<float*>(smem + L.tiles) + (size_t)buf * WS_BM * ST_TS;
      float* row[2] = {tile + (size_t)rr_[0] * ST_TS, tile + (size_t)rr_[1] * ST_TS};
      // P.V split as in the whole-row kernel: warp (kq, nh) takes the tile's 8-key
      // steps kq, kq + KQ, ... and columns nh*64 .. nh*64 + 63, staged in its own ring
      const int ns_all = (tlen + 7) >> 3;
      const int nsw = ns_all > kq ? (ns_all - kq + KQ - 1) / KQ : 0;
      auto load_step = [&](int i) {  // step i of this warp into ring slot i % WR
        if (i < nsw) {
          const int key0 = t0 + 8 * (kq + KQ * i);
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
      int nvr[2];
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) nvr[tt] = max(0, min(tlen, nv[tt] - t0));
      const int nit = (max(nvr[0], nvr[1]) + 127) >> 7;
      if (p.ps_out) {  // dump of the low-precision scores of this tile
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
          if (rr_[tt] < it.rows)
            for (int j = lane; j < ST_T && t0 + j < p.n_k; j += 32)
              p.ps_out[grow[tt] * p.n_k + t0 + j] = j < written ? row[tt][j] : -INFINITY;
      }
      // criterion, mask words, compaction and recompute of the selected keys
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        S.row[tt] = row[tt];
        S.nv[tt] = nvr[tt];
        S.word0[tt] = grow[tt] * nwords + (t0 >> 5);
        S.mx[tt] = -INFINITY;
        if (VAR == LAMP_STRICT) S.am[tt] = am_abs[tt] == 0x7FFFFFFF ? 0x7FFFFFFF : am_abs[tt] - t0;
      }
      for (int i4 = 0; i4 < nit; ++i4)
        sel_step<VAR>(p, S, 128 * i4, written, nwords - (t0 >> 5), tlo, thi, lane, wbuf, nsel);
      sel_finish(p, S, wbuf, 4 * nit, min(ST_T / 32, nwords - (t0 >> 5)), lane, [&](int tt, int j) {
        const float v = ws_recompute<D>(sQ, 2 * cw + tt, Kh + (size_t)(t0 + j) * D, p.scale, fast);
        tile[(size_t)(2 * cw + tt) * ST_TS + j] = v;
        if (tt == 0) S.mx[0] = fmaxf(S.mx[0], v);
        else S.mx[1] = fmaxf(S.mx[1], v);
      });
      __syncwarp();
      if (p.mixed_out) {  // dump of the mixed scores of this tile
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
          if (rr_[tt] < it.rows)
            for (int j = lane; j < ST_T && t0 + j < p.n_k; j += 32)
              p.mixed_out[grow[tt] * p.n_k + t0 + j] = j < written ? row[tt][j] : -INFINITY;
      }
      // online softmax: new maximum, rescale factor, numerators of this tile in place
      const int nitw = (written + 127) >> 7;
      float lt[2] = {0.f, 0.f}, mL[2], alpha[2];
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const float mn = fmaxf(m[tt], warp_max_redux(S.mx[tt]));
        alpha[tt] = mn == -INFINITY ? 1.f : exp_fast(__fsub_rn(m[tt], mn));  // exp(-inf) = 0 on the first tile
        mL[tt] = mn == -INFINITY ? 0.f : mn * kLog2e;
        m[tt] = mn;
      }
      for (int i4 = 0; i4 < nitw; ++i4) {
        const int j0 = 128 * i4 + 4 * lane;
        if (j0 >= written) continue;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          const float4 v = *reinterpret_cast<const float4*>(row[tt] + j0);
          const float vv[4] = {v.x, v.y, v.z, v.w};
          uint32_t pw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float pj;  // exp(y - m), 0 for -inf
            asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(pj) : "f"(fmaf(vv[e], kLog2e, -mL[tt])));
            lt[tt] += pj;
            pw[e] = p_pair_cvt(pj);
          }
          *reinterpret_cast<uint4*>(row[tt] + j0) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        }
      }
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        l[tt] = l[tt] * alpha[tt] + warp_sum(lt[tt]);
        if (lane == 0) {
          rst[4 * rr_[tt]] = m[tt];
          rst[4 * rr_[tt] + 1] = l[tt];
          rst[4 * rr_[tt] + 2] = alpha[tt];
        }
      }
      named_sync(BAR_CONS, NCT);  // P of the tile and every row's rescale factor are in place

      // rescale the partial outputs, then add P.V of this tile
      {
        const float a0 = rst[4 * (lane >> 2) + 2], a1 = rst[4 * ((lane >> 2) + 8) + 2];
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
          acc[tt][0] *= a0;
          acc[tt][1] *= a0;
          acc[tt][2] *= a1;
          acc[tt][3] *= a1;
        }
      }
      const int ra = 8 * (mi & 1) + (lane & 7);
      const int kl = 4 * (mi & 1) + ((lane & 7) >> 1);  // each V row serves the hi and the lo half of P
      for (int i = 0; i < nsw; ++i) {
        cp_async_wait<WR - 2>();  // step i has landed (this lane's copies)
        __syncwarp();             // ... and every lane's; step i - 1's slot is free
        load_step(i + WR - 1);
        const int kb = 8 * (kq + KQ * i);  // relative to the tile
        const uint16_t* vb = vring + (i % WR) * 8 * WS_VSW;
        uint32_t af[4];
        ldmatrix_x4(smem_u32(tile + (size_t)ra * ST_TS + kb + 4 * (mi >> 1)), af[0], af[1], af[2], af[3]);
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(smem_u32(vb + kl * WS_VSW + 16 * nb + 8 * (mi >> 1)), b0, b1, b2, b3);
          mma_bf16_16816(acc[2 * nb], af[0], af[1], af[2], af[3], b0, b1);
          mma_bf16_16816(acc[2 * nb + 1], af[0], af[1], af[2], af[3], b2, b3);
        }
      }
      cp_async_wait<0>();
      named_sync(BAR_CONS, NCT);  // V stages and rescale factors are no longer read

      if (t == nt - 1) {  // end of the item: add the partial outputs, divide by l
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
          const float lv = rst[4 * rr + 1];
          const float inv = lv > 0.f ? 1.f / lv : 0.f;
          const float v0 = o.x * inv, v1 = o.y * inv;
          const size_t off = ((size_t)it.bh * p.n_q + it.i0 + rr) * D + col;
          *reinterpret_cast<uint32_t*>(p.out + off) =
              (uint32_t)f32_to_bf16_rne(v0) | ((uint32_t)f32_to_bf16_rne(v1) << 16);
          if (p.out_f32) *reinterpret_cast<float2*>(p.out_f32 + off) = make_float2(v0, v1);
        }
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          if (rr_[tt] >= it.rows) continue;
          if (lane == 0 && p.lse_out) p.lse_out[grow[tt]] = nv[tt] > 0 ? m[tt] + logf(l[tt]) : -INFINITY;
          const int done = nt * ST_T;  // keys covered by the item's tiles
          if (p.mask_out)
            for (int w = (done >> 5) + lane; w < nwords; w += 32) p.mask_out[grow[tt] * nwords + w] = 0u;
          if (p.ps_out)
            for (int j = done + lane; j < p.n_k; j += 32) p.ps_out[grow[tt] * p.n_k + j] = -INFINITY;
          if (p.mixed_out)
            for (int j = done + lane; j < p.n_k; j += 32) p.mixed_out[grow[tt] * p.n_k + j] = -INFINITY;
        }
        named_sync(BAR_CONS, NCT);  // the output sums (V area) and this item's Q are no longer read
        const int q2 = ws_item(ii + 2, cta, G, a.n_items);
        if (q2 >= 0) ws_stage_q<D>(sQ, p, ws_decode(q2, p, a.n_rb), tidc, NCT);
      }
      mbar_arrive(bars + 2 + buf);  // tile buffer free (and, after an item's last tile, Q of item + 2 staged)
    }
  }
  if (lane == 0 && nsel && p.nsel_out) atomicAdd(p.nsel_out, (unsigned long long)nsel);
}

// Pass 1 of the strict rows: every tile stored to the slab, and per row the
// maximum, its first key and S_rest kept online across the tiles. A tile's
// maximum and first key come from warp reductions and its sum of exp(y - tile
// maximum) over the other keys from binary32 exp terms (ex2.approx) summed in double; the
// merge is exact in double: a larger tile maximum rescales the running sum by
// exp(m_old - m_new) with the old maximum joining it as a term 1, a smaller or
// equal one adds (tile sum + 1) exp(m_tile - m).
template <int D>
__device__ __forceinline__ void st_consumer_stats(const StArgs& a, unsigned char* smem, const StSmem& L, int cw,
                                                  int lane) {
  constexpr int NCT = WS_NC * 32;
  const Problem& p = a.p;
  const int tidc = cw * 32 + lane;
  const int G = gridDim.x, cta = blockIdx.x;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  for (int k0 = 0; k0 < 2; ++k0) {
    const int q0 = ws_item(k0, cta, G, a.n_items);
    if (q0 < 0) break;
    ws_stage_q<D>(qbase + k0 * ws_qfloats<D>(), p, ws_decode(q0, p, a.n_rb), tidc, NCT);
  }
  mbar_arrive(bars + 2);
  mbar_arrive(bars + 3);
  int k = 0;
  for (int ii = 0;; ++ii) {
    const int q = ws_item(ii, cta, G, a.n_items);
    if (q < 0) break;
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    float* sQ = qbase + (ii & 1) * ws_qfloats<D>();
    const int nt = st_ntiles(it.kv_end);
    int rr_[2];
    size_t grow[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      rr_[t] = 2 * cw + t;
      grow[t] = (size_t)it.bh * p.n_q + it.i0 + rr_[t];
    }
    float M[2] = {-INFINITY, -INFINITY};
    int AM[2] = {0x7FFFFFFF, 0x7FFFFFFF};
    double Sacc[2] = {0.0, 0.0};
    for (int t = 0; t < nt; ++t, ++k) {
      const int buf = k & 1;
      const int t0 = t * ST_T;
      const int tlen = max(0, min(ST_T, it.kv_end - t0));
      const int written = ((tlen + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;
      const float* tile = reinterpret_cast<const float*>(smem + L.tiles) + (size_t)buf * WS_BM * ST_TS;
      const bool ok = mbar_wait(bars + buf, (k >> 1) & 1);
      if (named_or(BAR_CONS, NCT, !ok)) {
        ws_timeout(p);
        return;
      }
      const int nit = (written + 127) >> 7;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const float* row = tile + (size_t)rr_[tt] * ST_TS;
        if (rr_[tt] < it.rows) {
          float* dst = a.slab + grow[tt] * a.ld + t0;
          for (int j0 = 4 * lane; j0 < written; j0 += 128)
            *reinterpret_cast<float4*>(dst + j0) = *reinterpret_cast<const float4*>(row + j0);
        }
        float lm = -INFINITY;
        int li = 0x7FFFFFFF;
        for (int i4 = 0; i4 < nit; ++i4) {
          const int j0 = 128 * i4 + 4 * lane;
          const float4 v = lds4_or_ninf(row + j0, j0 < written);
          if (v.x > lm) { lm = v.x; li = j0; }
          if (v.y > lm) { lm = v.y; li = j0 + 1; }
          if (v.z > lm) { lm = v.z; li = j0 + 2; }
          if (v.w > lm) { lm = v.w; li = j0 + 3; }
        }
        const float mt = warp_max_redux(lm);
        if (mt > -INFINITY) {  // warp-uniform
          const int at = t0 + __reduce_min_sync(0xFFFFFFFFu, lm == mt ? li : 0x7FFFFFFF);
          double sl = 0.0;
          const float ml = mt * kLog2e;  // exp(y - mt) on the special-function unit, as in the selection
          for (int i4 = 0; i4 < nit; ++i4) {
            const int j0 = 128 * i4 + 4 * lane;
            const float4 v = lds4_or_ninf(row + j0, j0 < written);
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float ex;
              asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ex) : "f"(fmaf(vv[e], kLog2e, -ml)));
              if (t0 + j0 + e != at) sl += (double)ex;
            }
          }
          const double st = warp_sum_d(sl);
          if (mt > M[tt]) {
            Sacc[tt] = M[tt] > -INFINITY ? (Sacc[tt] + 1.0) * exp((double)M[tt] - (double)mt) + st : st;
            M[tt] = mt;
            AM[tt] = at;
          } else {
            Sacc[tt] += (st + 1.0) * exp((double)mt - (double)M[tt]);
          }
        }
      }
      if (t == nt - 1) {  // end of the item: the row statistics, then Q of item + 2
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
          if (lane == 0 && rr_[tt] < it.rows) {
            RowStat rs;
            rs.m = M[tt];
            rs.am = AM[tt];
            rs.srest = Sacc[tt];
            a.rows[grow[tt]] = rs;
          }
        const int q2 = ws_item(ii + 2, cta, G, a.n_items);
        if (q2 >= 0) ws_stage_q<D>(sQ, p, ws_decode(q2, p, a.n_rb), tidc, NCT);
      }
      mbar_arrive(bars + 2 + buf);  // tile buffer free (and, after an item's last tile, Q of item + 2 staged)
    }
  }
}

template <int D, int RND, int VAR, int PH>
__global__ void __launch_bounds__(WS_NP * 32 + WS_NC * 32, 1) st_kernel(const StArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const StSmem L = st_plan<D>();
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
  if (warp < WS_NP) st_producer<D, RND, PH>(a, smem, L, warp, lane);
  else if (PH == 1) st_consumer_stats<D>(a, smem, L, warp - WS_NP, lane);
  else st_consumer<D, RND, VAR, PH>(a, smem, L, warp - WS_NP, lane);
}

template <int D, int RND, int VAR, int PH>
cudaError_t st_launch_one(const StArgs& a, int grid, cudaStream_t st) {
  auto k = st_kernel<D, RND, VAR, PH>;
  const size_t smem = (size_t)st_plan<D>().total;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, WS_NP * 32 + WS_NC * 32, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D, int RND>
cudaError_t st_launch_var(const StArgs& a, int grid, cudaStream_t st) {
  if (a.p.variant == LAMP_GIVEN_MASK) return st_launch_one<D, RND, LAMP_GIVEN_MASK, 0>(a, grid, st);
  if (a.p.variant == LAMP_RELAXED) return st_launch_one<D, RND, LAMP_RELAXED, 0>(a, grid, st);
  // strict: the scores-and-statistics pass, then the selection pass
  cudaError_t e = st_launch_one<D, RND, LAMP_STRICT, 1>(a, grid, st);
  if (e != cudaSuccess) return e;
  return st_launch_one<D, RND, LAMP_STRICT, 2>(a, grid, st);
}

}  // namespace

size_t stream_slab_ld(int n_k) { return (size_t)((n_k + ST_T - 1) / ST_T) * ST_T; }

size_t stream_smem_bytes(int d) { return d == 64 ? (size_t)st_plan<64>().total : (size_t)st_plan<128>().total; }

cudaError_t launch_stream(const Problem& p, const Workspace& ws, char* base, int num_sms, cudaStream_t st) {
  StArgs a;
  a.p = p;
  a.stats = reinterpret_cast<const int*>(base + ws.stats);
  a.nchunk = ws.nchunk;
  a.n_rb = (p.n_q + WS_BM - 1) / WS_BM;
  a.n_items = a.n_rb * p.B * p.H;
  a.slab = reinterpret_cast<float*>(base + ws.st_slab);
  a.ld = stream_slab_ld(p.n_k);
  a.rows = reinterpret_cast<RowStat*>(base + ws.st_rows);
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  if (p.d == 64) {
    if (rnd == kRndFast) return st_launch_var<64, kRndFast>(a, grid, st);
    if (rnd == kRndNone) return st_launch_var<64, kRndNone>(a, grid, st);
    return st_launch_var<64, kRndExact>(a, grid, st);
  }
  if (rnd == kRndFast) return st_launch_var<128, kRndFast>(a, grid, st);
  if (rnd == kRndNone) return st_launch_var<128, kRndNone>(a, grid, st);
  return st_launch_var<128, kRndExact>(a, grid, st);
}

}  // namespace lamp
