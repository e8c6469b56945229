// LAMP attention, streamed kernel for rows longer than the whole-row kernel
// takes: the relaxed and given-mask variants in one pass at any row length (the
// 16K-token shape), strict rows in two passes over an HBM score slab. Scores are
// produced and consumed in tiles of 512 keys with an online softmax, so no
// complete row is ever held on chip.
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
// Same organisation as the whole-row kernel (lamp_ws.cu): one persistent CTA of
// 640 threads per SM, items (b, h, 16 query rows) handed out at run time from a
// global counter, two tile buffers in the block layout of lamp_ws_common.cuh.
//   producers (warps 0-7): 64-key units dealt round-robin, PS(mu) steps as packed
//     binary32 pairs, K slices staged through registers as binary32.
//   consumers (warps 8-15): per tile the criterion (double re-evaluation near
//     tau), mask words, warp-compacted FP32 recompute, then the online softmax
//     (running maximum m and normaliser l per row, rescale factor
//     alpha = exp(m_old - m_new)) with the numerators written in place as the
//     bf16 hi/lo operand of P.V.
//   tensor-core warpgroup (warps 16-19): one thread streams V tiles of 64 keys by
//     TMA (128-byte swizzle) into a ring that runs ahead across tiles and items,
//     and issues 4 tcgen05.mma per V tile into one of two TMEM accumulators; the
//     four warps then fold each tile into a register accumulator,
//     O = alpha O + P.V (a thread holds one head dimension of the item's 16
//     rows), and after an item's last tile store O / l.
// Every wait is bounded; a wait that gives up records LAMP_ERR_TIMEOUT in the
// caller's status word (when given) and ends the kernel after the copies and
// tensor-core work in flight have drained and the tensor memory is released.
#include <cfloat>

#include "lamp_ws_common.cuh"

namespace lamp {
namespace {

constexpr int ST_T = 512;  // keys per streamed tile

template <int D>
__host__ __device__ constexpr int st_vslots() { return D == 64 ? 8 : 5; }  // V tiles in the ring
template <int D>
__host__ __device__ constexpr int st_vtile_bytes() { return WS_VKEYS * D * 2; }

// mbarrier indices
constexpr int SB_FULL = 0, SB_PREADY = 2, SB_EMPTY = 4, SB_TFREE = 6, SB_VFULL = 8;
template <int D>
__host__ __device__ constexpr int sb_vempty() { return SB_VFULL + st_vslots<D>(); }
template <int D>
__host__ __device__ constexpr int sb_drain() { return SB_VFULL + 2 * st_vslots<D>(); }
template <int D>
__host__ __device__ constexpr int sb_count() { return sb_drain<D>() + 1; }
constexpr int BAR_PROD = 2;  // named barrier of the producer group
constexpr int BAR_EPI = 3;   // named barrier of the tensor-core warpgroup (output epilogue)

struct StSmem {  // byte offsets from a 1024-byte aligned base
  int tiles;  // score tiles [2][sw_bytes(512)] (block layout)
  int v;      // V ring [S][D / 64][64 keys][64 dims] bf16 (128-byte swizzle)
  int ks;     // producer K slices [8 warps][2][8][64] f32
  int q;      // Q [2][D][16] f32, by item parity
  int list;   // consumer mask-word buffers [8][2][32] uint32
  int rstat;  // per tile parity and row: m, l, alpha, spare [2][16][4] f32
  int otile;  // output tile of an item [16][D] bf16 (epilogue)
  int bars;   // mbarriers
  int sched;  // item ring [8] and published count (lamp_ws_common.cuh)
  int tmem;   // TMEM base address
  int total;
};

template <int D>
__host__ __device__ inline StSmem st_plan() {
  StSmem s{};
  s.tiles = 0;
  s.v = 2 * sw_bytes(ST_T);
  s.ks = s.v + st_vslots<D>() * st_vtile_bytes<D>();
  s.q = s.ks + WS_NP * 2 * WS_DS * WS_UNIT * 4;
  s.list = s.q + 2 * ws_qfloats<D>() * 4;
  s.rstat = s.list + WS_NC * 2 * SEL_WMAX * 4;
  s.otile = s.rstat + 2 * WS_BM * 4 * 4;
  s.bars = s.otile + WS_BM * D * 2;
  s.sched = s.bars + sb_count<D>() * 8;
  s.tmem = s.sched + 16 * 4;
  s.total = s.tmem + 16;
  return s;
}

// Strict rows too long for whole-row buffers run in two passes of this kernel
// (template parameter PH):
//   PH 0: one pass (relaxed, given mask);
//   PH 1: strict statistics: the producers compute the scores; the consumers store
//         every tile to an HBM score slab and keep, per row, the maximum m, its
//         first key am and S_rest = sum over the other keys of exp(y - m) online
//         across tiles (tile maximum and sum, merged in double); no P.V;
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
  const int* stats;   // per-(b, h) exponent statistics
  unsigned* counter;  // next item to hand out (zeroed by the preparation kernel; one per pass)
  int nchunk;
  int n_items;
  int n_rb;
  float* slab;       // strict: low-precision scores [B*H][n_q][ld]
  size_t ld;         // slab row stride (keys rounded up to whole tiles)
  RowStat* rows;     // strict: [B*H][n_q]
};

__device__ __forceinline__ int st_ntiles(int kv_end) { return kv_end > 0 ? (kv_end + ST_T - 1) / ST_T : 1; }

// The consumers' item ii (-1: none left, -2: the wait for it gave up, agreed by
// every consumer thread). Items 0 and 1 come from the producers; at each item
// thread 0 claims item ii + 2, which the consumers' next barrier (the first
// tile's hand-off) makes visible to all of them.
__device__ __forceinline__ int st_next_item(const StArgs& a, ItemRing sched, int ii, int tidc) {
  int q;
  if (ii < 2) {
    q = wait_published(sched, ii);
    if (named_or(BAR_CONS, WS_NC * 32, q == -2)) return -2;
  } else {
    q = sched.get(ii);
  }
  if (q >= 0 && tidc == 0) publish_item(sched, ii + 2, claim_item(a.counter, a.n_items));
  return q;
}

// ---------------------------------------------------------------------------
// Producers: every tile of every item, in the order the consumers take them.
// ---------------------------------------------------------------------------
template <int D, int RND, int PH>
__device__ __forceinline__ void st_producer(const StArgs& a, unsigned char* smem, const StSmem& L, int warp,
                                            int lane) {
  const Problem& p = a.p;
  const int s = 23 - p.mu;
  const u64 negc = pack2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const u64 pow2s = pack2((float)(1u << s), (float)(1u << s));
  const u64 scale2 = pack2(p.scale, p.scale);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  float* ksw = reinterpret_cast<float*>(smem + L.ks) + warp * 2 * WS_DS * WS_UNIT;
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  const ItemRing sched{smem_u32(smem + L.sched)};
  // claim the first two items and stage their Q (the consumers do the later ones)
  if (warp == 0 && lane == 0) {
    const int q0 = claim_item(a.counter, a.n_items);
    sched.put(0, q0);
    publish_item(sched, 1, q0 < 0 ? -1 : claim_item(a.counter, a.n_items));
  }
  named_sync(BAR_PROD, WS_NP * 32);
  for (int k0 = 0; k0 < 2; ++k0) {
    const int q0 = sched.get(k0);
    if (q0 < 0) break;
    ws_stage_q<D>(qbase + k0 * ws_qfloats<D>(), p, ws_decode(q0, p, a.n_rb), warp * 32 + lane, WS_NP * 32);
  }
  named_sync(BAR_PROD, WS_NP * 32);
  int deal = 0;  // producer warp that takes the next unit
  int k = 0;     // tile counter: buffer k & 1, phase k >> 1
  for (int ii = 0;; ++ii) {
    // the consumers' hand-off of tile k - 2, which follows their claim of item ii
    // (made when they began item ii - 2, whose first tile is k - 2 or earlier);
    // one decision per warp: the tile routine synchronises the warp
    if (k >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait(bars + SB_PREADY + (k & 1), ((k - 2) >> 1) & 1))) {
      ws_timeout(p);
      return;
    }
    const int q = sched.get(ii);
    if (q < 0) break;
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    const float* sQ = qbase + (ii & 1) * ws_qfloats<D>();
    const int nt = st_ntiles(it.kv_end);
    for (int t = 0; t < nt; ++t, ++k) {
      const int buf = k & 1;
      const int t0 = t * ST_T;
      const int tlen = max(0, min(ST_T, it.kv_end - t0));
      const uint32_t ph = ((k - 2) >> 1) & 1;
      // the consumers' hand-off of tile k - 2 (waited above for an item's first
      // tile, whose Q it also brings)
      if (t > 0 && k >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait(bars + SB_PREADY + buf, ph))) {
        ws_timeout(p);
        return;
      }
      float* tile = reinterpret_cast<float*>(smem + L.tiles + buf * sw_bytes(ST_T));
      if (PH == 2) {
        // the tile buffer is free once tile k - 2's P.V has completed and been read
        if (k >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait(bars + SB_TFREE + buf, ph))) {
          ws_timeout(p);
          return;
        }
        // the tile's scores from the slab: rows of the item by cp.async, keys of the
        // tile that the scores pass wrote; rows past the item hold -inf
        const int written = ((tlen + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;
        const int per_row = written / 4;  // 16-byte pieces
        for (int u = warp * 32 + lane; u < WS_BM * per_row; u += WS_NP * 32) {
          const int r = u / per_row, c4 = u % per_row;
          float* dst = tile + sw_off(r, 4 * c4);
          if (r < it.rows)
            cp_async16(dst, a.slab + ((size_t)it.bh * p.n_q + it.i0 + r) * a.ld + t0 + 4 * c4);
          else
            *reinterpret_cast<float4*>(dst) = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
        cp_async_commit();
        cp_async_wait<0>();
      } else {
        // the tile buffer is free once tile k - 2's P.V has completed and been read
        // (tfree): the tile routine waits for that only before its first store
        if (!ws_produce_tile<D, RND, WS_DS>(p, it, t0, tlen, sQ, tile, ksw, lane, (warp - deal + WS_NP) % WS_NP, fast, Kh,
                                     negc, pow2s, scale2, s, k >= 2 ? bars + SB_TFREE + buf : nullptr, ph)) {
          ws_timeout(p);
          return;
        }
        deal = (deal + (tlen + WS_UNIT - 1) / WS_UNIT) % WS_NP;
      }
      mbar_arrive(bars + SB_FULL + buf);  // this thread's scores of the tile are in place
    }
  }
}

// ---------------------------------------------------------------------------
// Consumers: selection, recompute and the online softmax, tile by tile.
// ---------------------------------------------------------------------------
template <int D, int RND, int VAR, int PH>
__device__ __forceinline__ void st_consumer(const StArgs& a, unsigned char* smem, const StSmem& L, int cw, int lane) {
  constexpr int NCT = WS_NC * 32;
  const Problem& p = a.p;
  const int tidc = cw * 32 + lane;
  const int nwords = (p.n_k + 31) >> 5;
  const bool refine_ok = VAR != LAMP_GIVEN_MASK && isfinite(p.tau) && p.tau >= 0.f;
  const float band = WS_BAND * p.tau;
  const float tlo = refine_ok ? p.tau - band : INFINITY;
  const float thi = refine_ok ? (p.tau == 0.f ? 1e-30f : p.tau + band) : -INFINITY;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(smem + L.list) + cw * 2 * SEL_WMAX;
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  float* rst = reinterpret_cast<float*>(smem + L.rstat);
  const ItemRing sched{smem_u32(smem + L.sched)};
  long long nsel = 0;
  int k = 0;
  for (int ii = 0;; ++ii) {
    const int q = st_next_item(a, sched, ii, tidc);
    if (q == -2) {
      ws_timeout(p);
      return;
    }
    if (q < 0) break;
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    const bool fast = (RND != kRndExact) && head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk,
                                                          p.emax_sum_limit);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
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
      S.rr[tt] = rr_[tt];
      S.off[tt] = sw_off(rr_[tt], lane);
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
    // keys 128 i4 + 4 lane .. + 3 of row rr_[t]: scores at ob[t] + 2048 i4, P_hi at pbo[t] + 2048 i4
    const int ob[2] = {sw_off(rr_[0], 4 * lane), sw_off(rr_[1], 4 * lane)};
    const int pbo[2] = {p_off(rr_[0], 4 * lane), p_off(rr_[1], 4 * lane)};

    for (int t = 0; t < nt; ++t, ++k) {
      const int buf = k & 1;
      const int t0 = t * ST_T;
      const int tlen = max(0, min(ST_T, it.kv_end - t0));
      const int written = ((tlen + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;  // keys the producers wrote
      float* tile = reinterpret_cast<float*>(smem + L.tiles + buf * sw_bytes(ST_T));
      const bool ok = mbar_wait(bars + SB_FULL + buf, (k >> 1) & 1);
      if (named_or(BAR_CONS, NCT, !ok)) {
        ws_timeout(p);
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
              p.ps_out[grow[tt] * p.n_k + t0 + j] = j < written ? tile[sw_off(rr_[tt], j)] : -INFINITY;
      }
      // criterion, mask words, compaction and recompute of the selected keys
      S.base = tile;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        S.nv[tt] = nvr[tt];
        S.word0[tt] = grow[tt] * nwords + (t0 >> 5);
        S.mx[tt] = -INFINITY;
        if (VAR == LAMP_STRICT) S.am[tt] = am_abs[tt] == 0x7FFFFFFF ? 0x7FFFFFFF : am_abs[tt] - t0;
      }
      for (int i4 = 0; i4 < nit; ++i4)
        sel_step<VAR>(p, S, 128 * i4, written, nwords - (t0 >> 5), tlo, thi, lane, wbuf, nsel);
      sel_finish(p, S, wbuf, 4 * nit, min(ST_T / 32, nwords - (t0 >> 5)), lane, [&](int tt, int j) {
        const float v = ws_recompute<D>(sQ, 2 * cw + tt, Kh + (size_t)(t0 + j) * D, p.scale, fast);
        tile[sw_off(2 * cw + tt, j)] = v;
        if (tt == 0) S.mx[0] = fmaxf(S.mx[0], v);
        else S.mx[1] = fmaxf(S.mx[1], v);
      });
      __syncwarp();
      if (p.mixed_out) {  // dump of the mixed scores of this tile
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
          if (rr_[tt] < it.rows)
            for (int j = lane; j < ST_T && t0 + j < p.n_k; j += 32)
              p.mixed_out[grow[tt] * p.n_k + t0 + j] = j < written ? tile[sw_off(rr_[tt], j)] : -INFINITY;
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
        const bool act = j0 < written;
        float4 v[2];
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) v[tt] = act ? *reinterpret_cast<const float4*>(tile + ob[tt] + 2048 * i4)
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        __syncwarp();  // the 128 keys of both rows are read before any lane overwrites them
        if (act) {
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            const float vv[4] = {v[tt].x, v[tt].y, v[tt].z, v[tt].w};
            uint32_t pw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float pj;  // exp(y - m), 0 for -inf
              asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(pj) : "f"(fmaf(vv[e], kLog2e, -mL[tt])));
              lt[tt] += pj;
              pw[e] = p_pair_cvt(pj);  // low half bf16(P), high half bf16(P - bf16(P))
            }
            float* dst = tile + pbo[tt] + 2048 * i4;
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(__byte_perm(pw[0], pw[1], 0x5410), __byte_perm(pw[2], pw[3], 0x5410));
            *reinterpret_cast<uint2*>(dst + 512) =
                make_uint2(__byte_perm(pw[0], pw[1], 0x7632), __byte_perm(pw[2], pw[3], 0x7632));
          }
        }
      }
      float* rs = rst + buf * WS_BM * 4;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        l[tt] = l[tt] * alpha[tt] + warp_sum(lt[tt]);
        if (lane == 0) {
          rs[4 * rr_[tt]] = m[tt];
          rs[4 * rr_[tt] + 1] = l[tt];
          rs[4 * rr_[tt] + 2] = alpha[tt];
        }
      }
      fence_async_smem();  // P (generic-proxy stores) becomes visible to the tensor core
      named_sync(BAR_CONS, NCT);  // P and every row's m, l, alpha of the tile are in place
      if (t == nt - 1) {   // Q of the item is no longer read: stage item + 2's
        const int q2 = sched.get(ii + 2);
        if (q2 >= 0) ws_stage_q<D>(sQ, p, ws_decode(q2, p, a.n_rb), tidc, NCT);
      }
      mbar_arrive(bars + SB_PREADY + buf);  // P of the tile in place (and at an item's end, Q of item + 2)

      if (t == nt - 1) {  // end of the item: lse, and the parts of the dumps past its tiles
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
      }
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  const ItemRing sched{smem_u32(smem + L.sched)};
  int k = 0;
  for (int ii = 0;; ++ii) {
    const int q = st_next_item(a, sched, ii, tidc);
    if (q == -2) {
      ws_timeout(p);
      return;
    }
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
      const float* tile = reinterpret_cast<const float*>(smem + L.tiles + buf * sw_bytes(ST_T));
      const bool ok = mbar_wait(bars + SB_FULL + buf, (k >> 1) & 1);
      if (named_or(BAR_CONS, NCT, !ok)) {
        ws_timeout(p);
        return;
      }
      const int nit = (written + 127) >> 7;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int ob = sw_off(rr_[tt], 4 * lane);  // key 128 i4 + 4 lane at ob + 2048 i4
        if (rr_[tt] < it.rows) {
          float* dst = a.slab + grow[tt] * a.ld + t0;
          for (int i4 = 0; 128 * i4 + 4 * lane < written; ++i4)
            *reinterpret_cast<float4*>(dst + 128 * i4 + 4 * lane) =
                *reinterpret_cast<const float4*>(tile + ob + 2048 * i4);
        }
        float lm = -INFINITY;
        int li = 0x7FFFFFFF;
        for (int i4 = 0; i4 < nit; ++i4) {
          const int j0 = 128 * i4 + 4 * lane;
          const float4 v = lds4_or_ninf(tile + ob + 2048 * i4, j0 < written);
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
            const float4 v = lds4_or_ninf(tile + ob + 2048 * i4, j0 < written);
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
        // this pass reads no Q, and the producers are done with the item's
        const int q2 = sched.get(ii + 2);
        if (q2 >= 0) ws_stage_q<D>(sQ, p, ws_decode(q2, p, a.n_rb), tidc, NCT);
      }
      mbar_arrive(bars + SB_PREADY + buf);  // tile buffer read (and, after an item's last tile, Q of item + 2 staged)
    }
  }
}

// ---------------------------------------------------------------------------
// Tensor-core warpgroup (warps 16-19, ew = warp - 16). Per score tile, lane 0 of
// warp 16 streams the V tiles by TMA and issues the tile's P.V by tcgen05.mma
// (in the statistics pass it only hands the buffer on); then the four warps
// (TMEM lane quarter ew: head dimensions 32 ew + lane, or 16 ew + lane in lanes
// 0-15 for the M = 64 shape of d = 64) fold the tile into their register
// accumulator, O = (alpha O + P_hi.V) + P_lo.V with alpha = exp(m_old - m_new)
// of each row, release the buffer (tfree), and after an item's last tile store
// O / l as bf16 through a shared-memory tile with 16-byte stores.
// ---------------------------------------------------------------------------
template <int D, int PH>
__device__ __forceinline__ void st_tensor_warpgroup(const StArgs& a, const CUtensorMap* tmV, unsigned char* smem,
                                                    const StSmem& L, uint32_t tbase, int ew, int lane) {
  constexpr int S = st_vslots<D>();
  constexpr uint32_t TB = st_vtile_bytes<D>();
  const Problem& p = a.p;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  unsigned char* vring = smem + L.v;
  const uint32_t vbase = smem_u32(vring), tiles = smem_u32(smem + L.tiles);
  const ItemRing sched{smem_u32(smem + L.sched)};
  const uint32_t idesc = umma_idesc_bf16(D, 32);
  const float* rst = reinterpret_cast<const float*>(smem + L.rstat);
  uint16_t* otile = reinterpret_cast<uint16_t*>(smem + L.otile);
  const bool issuer = ew == 0 && lane == 0;
  bool ok = true;
  // V tiles form one sequence over the CTA's score tiles: V tile vt of score tile
  // (item il, tile tl) is number gl
  int il = 0, tl = 0, ntl = -1, bhl = 0, kvl = 0, vt = 0, nvl = -1;
  int gl = 0, gm = 0;  // next V tile to load, next V tile to multiply
  auto next_v = [&]() -> bool {  // false: no further V tile known yet (or none left)
    for (;;) {
      if (ntl < 0) {  // enter item il
        if (sched.count() <= il) return false;  // item il is not claimed yet
        __threadfence_block();
        const int q = sched.get(il);
        if (q < 0) return false;
        const ItemInfo it = ws_decode(q, p, a.n_rb);
        ntl = st_ntiles(it.kv_end);
        bhl = it.bh;
        kvl = it.kv_end;
        tl = 0;
        nvl = -1;
      }
      if (tl < ntl) {
        if (nvl < 0) {  // enter score tile tl
          const int tlen = max(0, min(ST_T, kvl - tl * ST_T));
          nvl = (tlen + WS_VKEYS - 1) / WS_VKEYS;
          vt = 0;
        }
        if (vt < nvl) return true;
        ++tl;
        nvl = -1;
        continue;
      }
      ++il;
      ntl = -1;
    }
  };
  auto load_upto = [&](int limit) {  // start the loads of V tiles gl .. limit - 1
    while (ok && gl < limit && next_v()) {
      const int slot = gl % S;
      if (gl >= S && !mbar_wait(bars + sb_vempty<D>() + slot, ((gl / S) - 1) & 1)) {
        ok = false;
        break;
      }
      mbar_expect_tx(bars + SB_VFULL + slot, TB);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(vring + slot * TB + h * 8192, tmV, 64 * h, tl * ST_T + WS_VKEYS * vt, bhl,
                    bars + SB_VFULL + slot);
      ++vt;
      ++gl;
    }
  };
  // P.V of score tile k (the issuing thread only)
  auto mma_tile = [&](int k, int tlen) {
    const int buf = k & 1;
    const int T = (tlen + WS_VKEYS - 1) / WS_VKEYS;
    if (PH != 1) load_upto(gm + S);
    if (!ok || !mbar_wait(bars + SB_PREADY + buf, (k >> 1) & 1)) {
      ok = false;
      return;
    }
    if (PH == 1) {  // the statistics pass reads the tile on the CUDA cores only
      mbar_arrive(bars + SB_EMPTY + buf);
      return;
    }
    tc_fence_after();
    const uint32_t dcol = tbase + 32 * buf;
    const uint32_t pb = tiles + buf * sw_bytes(ST_T);
    for (int v = 0; v < T; ++v, ++gm) {
      load_upto(gm + S - 1);  // keep the ring full (waits for the MMAs two V tiles back)
      const int slot = gm % S;
      if (!ok || !mbar_wait(bars + SB_VFULL + slot, (gm / S) & 1)) {
        ok = false;
        return;
      }
      tc_fence_after();
      const uint32_t va = vbase + slot * TB, pa = pb + v * 4096;
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) {  // 16 keys per MMA
        const uint64_t ad = umma_desc_sw128(va + s4 * 2048, D == 128 ? 8192u : 0u, 1024);
        const uint64_t bd = umma_desc_sw128(pa + s4 * 32, 16, 1024);
        umma_bf16(dcol, ad, bd, idesc, (v | s4) != 0);
      }
      umma_commit(bars + sb_vempty<D>() + slot);
    }
    umma_commit(bars + SB_EMPTY + buf);  // the tile's P.V is complete
  };
  const int dim = D == 128 ? 32 * ew + lane : 16 * ew + lane;
  const bool dim_ok = D == 128 || lane < 16;
  bool good = true;
  int k = 0;
  for (int ii = 0; good; ++ii) {
    const int q = wait_published(sched, ii);
    if (q == -1) break;
    if (q < 0) {  // the wait gave up (agreed: every thread polls the same count)
      good = false;
      break;
    }
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    const int nt = st_ntiles(it.kv_end);
    float o[WS_BM];  // this thread's head dimension of the item's 16 rows
#pragma unroll
    for (int r = 0; r < WS_BM; ++r) o[r] = 0.f;
    for (int t = 0; t < nt; ++t, ++k) {
      const int buf = k & 1;
      if (issuer && ok) mma_tile(k, max(0, min(ST_T, it.kv_end - t * ST_T)));
      __syncwarp();
      // a failed issue leaves the tile incomplete: the bounded wait below then
      // gives up, and all four warps agree on it
      const bool done = mbar_wait(bars + SB_EMPTY + buf, (k >> 1) & 1);
      if (named_or(BAR_EPI, 128, !done)) {
        good = false;
        break;
      }
      if (PH != 1) {
        tc_fence_after();
        const float* rs = rst + buf * WS_BM * 4;
        const uint32_t ta = tbase + 32 * buf + ((uint32_t)(32 * ew) << 16);
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // rows 8h .. 8h + 7: O = alpha O + P_hi.V, then + P_lo.V
          float v[8];
          tmem_ld8(ta + 8 * h, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) o[8 * h + j] = fmaf(o[8 * h + j], rs[4 * (8 * h + j) + 2], v[j]);
          tmem_ld8(ta + 16 + 8 * h, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) o[8 * h + j] = __fadd_rn(o[8 * h + j], v[j]);
        }
        if (t == nt - 1) {
#pragma unroll
          for (int r = 0; r < WS_BM; ++r) {
            const float lv = rs[4 * r + 1];
            o[r] = lv > 0.f ? o[r] * (1.f / lv) : 0.f;
          }
        }
        tc_fence_before();
      }
      mbar_arrive(bars + SB_TFREE + buf);  // accumulator, row statistics and tile buffer are free
      if (PH != 1 && t == nt - 1) {       // the item's output
        if (dim_ok) {
#pragma unroll
          for (int r = 0; r < WS_BM; ++r) {
            otile[r * D + dim] = f32_to_bf16_rne(o[r]);
            if (p.out_f32 && r < it.rows) p.out_f32[((size_t)it.bh * p.n_q + it.i0 + r) * D + dim] = o[r];
          }
        }
        named_sync(BAR_EPI, 128);
        for (int c = ew * 32 + lane; c < WS_BM * D / 8; c += 128) {
          const int r = c / (D / 8), c8 = (c % (D / 8)) * 8;
          if (r < it.rows)
            *reinterpret_cast<uint4*>(p.out + ((size_t)it.bh * p.n_q + it.i0 + r) * D + c8) =
                *reinterpret_cast<const uint4*>(otile + r * D + c8);
        }
        named_sync(BAR_EPI, 128);  // the tile may be refilled
      }
    }
  }
  if (issuer) {
    // drain: every MMA issued and every V load in flight completes before the
    // tensor memory is released and the CTA exits
    umma_commit(bars + sb_drain<D>());
    bool drained = mbar_wait(bars + sb_drain<D>(), 0);
    for (int g = gm; g < gl; ++g) drained = mbar_wait(bars + SB_VFULL + g % S, (g / S) & 1) && drained;
    if (!ok || !drained) good = false;
  }
  if (!good && lane == 0) ws_timeout(p);
}

template <int D, int RND, int VAR, int PH>
__global__ void __launch_bounds__(WS_NT, 1) st_kernel(const StArgs a, const __grid_constant__ CUtensorMap tmV) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + smem_align1k_pad(smem_raw);
  const StSmem L = st_plan<D>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L.tmem);
  if (threadIdx.x == 0) {
    mbar_init(bars + SB_FULL + 0, WS_NP * 32);
    mbar_init(bars + SB_FULL + 1, WS_NP * 32);
    mbar_init(bars + SB_PREADY + 0, WS_NC * 32);
    mbar_init(bars + SB_PREADY + 1, WS_NC * 32);
    mbar_init(bars + SB_EMPTY + 0, 1);
    mbar_init(bars + SB_EMPTY + 1, 1);
    mbar_init(bars + SB_TFREE + 0, 128);
    mbar_init(bars + SB_TFREE + 1, 128);
    for (int i = 0; i < st_vslots<D>(); ++i) {
      mbar_init(bars + SB_VFULL + i, 1);
      mbar_init(bars + sb_vempty<D>() + i, 1);
    }
    mbar_init(bars + sb_drain<D>(), 1);
    mbar_fence_init();
    ItemRing{smem_u32(smem + L.sched)}.set_count(0);  // no item published yet
  }
  if (warp == WS_MW) tmem_alloc(tslot, WS_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  if (warp < WS_NP) {
    regs_inc<kWsProdRegs>();
    st_producer<D, RND, PH>(a, smem, L, warp, lane);
  } else if (warp < WS_MW) {
    regs_inc<kWsConsRegs>();
    if (PH == 1) st_consumer_stats<D>(a, smem, L, warp - WS_NP, lane);
    else st_consumer<D, RND, VAR, PH>(a, smem, L, warp - WS_NP, lane);
  } else {
    regs_dec<kWsMmaRegs>();
    st_tensor_warpgroup<D, PH>(a, &tmV, smem, L, tbase, warp - WS_MW, lane);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WS_MW) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, WS_TMEM_COLS);
  }
}

template <int D, int RND, int VAR, int PH>
cudaError_t st_launch_one(const StArgs& a, const CUtensorMap& tmV, int grid, cudaStream_t st) {
  auto k = st_kernel<D, RND, VAR, PH>;
  StArgs b = a;
  b.counter += PH == 2 ? 1 : 0;  // the selection pass hands out the items afresh
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kWsLaunchRegs) return cudaErrorInvalidConfiguration;  // the register split assumes this pool
  const size_t smem = (size_t)st_plan<D>().total + 1024;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, WS_NT, smem, st>>>(b, tmV);
  return cudaGetLastError();
}

template <int D, int RND>
cudaError_t st_launch_var(const StArgs& a, const CUtensorMap& tmV, int grid, cudaStream_t st) {
  if (a.p.variant == LAMP_GIVEN_MASK) return st_launch_one<D, RND, LAMP_GIVEN_MASK, 0>(a, tmV, grid, st);
  if (a.p.variant == LAMP_RELAXED) return st_launch_one<D, RND, LAMP_RELAXED, 0>(a, tmV, grid, st);
  // strict: the scores-and-statistics pass, then the selection pass
  cudaError_t e = st_launch_one<D, RND, LAMP_STRICT, 1>(a, tmV, grid, st);
  if (e != cudaSuccess) return e;
  return st_launch_one<D, RND, LAMP_STRICT, 2>(a, tmV, grid, st);
}

}  // namespace

size_t stream_slab_ld(int n_k) { return (size_t)((n_k + ST_T - 1) / ST_T) * ST_T; }

size_t stream_smem_bytes(int d) {  // dynamic shared memory of a launch (with the alignment slack)
  return (d == 64 ? (size_t)st_plan<64>().total : (size_t)st_plan<128>().total) + 1024;
}

cudaError_t launch_stream(const Problem& p, const Workspace& ws, char* base, int num_sms, cudaStream_t st) {
  StArgs a;
  a.p = p;
  a.stats = reinterpret_cast<const int*>(base + ws.stats);
  a.counter = reinterpret_cast<unsigned*>(base + ws.counters);
  a.nchunk = ws.nchunk;
  a.n_rb = (p.n_q + WS_BM - 1) / WS_BM;
  a.n_items = a.n_rb * p.B * p.H;
  a.slab = reinterpret_cast<float*>(base + ws.st_slab);
  a.ld = stream_slab_ld(p.n_k);
  a.rows = reinterpret_cast<RowStat*>(base + ws.st_rows);
  CUtensorMap tmV;
  const cudaError_t e = make_tmap_bf16(&tmV, p.V, p.d, p.n_k, p.B * p.H, 64, WS_VKEYS, 128);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  if (p.d == 64) {
    if (rnd == kRndFast) return st_launch_var<64, kRndFast>(a, tmV, grid, st);
    if (rnd == kRndNone) return st_launch_var<64, kRndNone>(a, tmV, grid, st);
    return st_launch_var<64, kRndExact>(a, tmV, grid, st);
  }
  if (rnd == kRndFast) return st_launch_var<128, kRndFast>(a, tmV, grid, st);
  if (rnd == kRndNone) return st_launch_var<128, kRndNone>(a, tmV, grid, st);
  return st_launch_var<128, kRndExact>(a, tmV, grid, st);
}

}  // namespace lamp
