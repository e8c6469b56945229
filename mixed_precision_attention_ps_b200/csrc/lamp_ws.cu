// LAMP attention, warp-specialised row kernel (strict, relaxed, given mask) for
// rows short enough that two blocks of 16 complete score rows fit in shared
// memory at once (n_k up to 1024 keys at d = 64, 896 at d = 128; the GPT-2 XL
// attention shape).
//
// Method ("LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models",
// technical summary, gist.science paper 2601.21623): section "Implementation
// strategy", steps 1-3; section "Theoretical basis", item 3, softmax bullet (the
// strict test 2 z (1 - z) |y| > tau on the whole probability row); section
// "Experimental results" (PS(mu), relaxed relative threshold, random control).
//
// One persistent CTA of 640 threads (5 warpgroups) per SM works through items
// (b, h, block of 16 query rows) that it claims at run time from a work counter,
// heaviest causal blocks first. Two row buffers alternate between three warp
// roles, each warpgroup with its own register budget (setmaxnreg):
//
//   producers (warps 0-7): PS(mu) scores of item k into buffer k & 1. The item's
//     keys are cut into 64-key units dealt round-robin to the producer warps,
//     continuing across items. Each warp stages its own K slices (8 head
//     dimensions x 64 keys, binary32, double buffered). A lane holds 8 rows x 4
//     keys as sixteen packed binary32 pairs (two rows of one key per 64-bit
//     register): one accumulation step is fma.rn.f32x2 plus the two-instruction
//     PS(mu) rounding (or the exact integer rounding).
//   consumers (warps 8-15): for item k, two rows per warp, four keys per lane:
//     row maximum and first argmax, S_rest in double (strict), the criterion with
//     a double re-evaluation near tau, mask words, warp-compacted FP32 recompute,
//     then the softmax numerators of the mixed row written in place as bf16 hi/lo
//     parts in the tensor-core operand layout (sw_off / p_off).
//   tensor-core warpgroup (warps 16-19): one thread streams V tiles of 64 keys by
//     TMA into a ring of shared-memory slots (running ahead across items) and, for
//     each item once its P is in place, issues O^T = V^T P^T by tcgen05.mma into
//     one of two TMEM accumulators (lamp_umma.cuh); tcgen05.commit frees each V
//     slot and signals the item's completion. Then the four warps (one per TMEM
//     lane quarter) read the accumulator, scale by 1 / l and store the output
//     with 16-byte stores through a shared-memory tile. Warp 17 also hands out
//     the items: it claims item k + 3, reads its head's exponent statistics,
//     stages its Q into slot k % 3 and publishes it in a ring in shared memory
//     once the output of item k is stored.
//
// Hand-offs use mbarriers: full[b] (256 producer arrivals: the scores are in
// place), pready[b] (256 consumer arrivals: P in place), empty[b] (the item's
// MMAs have completed), tfree[b] (128 epilogue arrivals: accumulator and row
// statistics read, so the buffer may be refilled), vfull/vempty per V slot; and
// the ring's published count (polled).
// Every wait is bounded; a wait that gives up records LAMP_ERR_TIMEOUT in the
// caller's status word (when given) and ends the kernel after the tensor-core
// work in flight has drained and the tensor memory is released.
#include <cfloat>

#include "lamp_ws_common.cuh"

namespace lamp {
namespace {

template <int D>
__host__ __device__ constexpr int ws_vslots() { return D == 64 ? 6 : 3; }  // V tiles in the ring
template <int D>
__host__ __device__ constexpr int ws_vtile_bytes() { return WS_VKEYS * D * 2; }  // 64 keys x D dimensions, bf16

// mbarrier indices
constexpr int BAR_FULL = 0, BAR_PREADY = 2, BAR_EMPTY = 4, BAR_TFREE = 6, BAR_VFULL = 8;
template <int D>
__host__ __device__ constexpr int bar_vempty() { return BAR_VFULL + ws_vslots<D>(); }
template <int D>
__host__ __device__ constexpr int bar_drain() { return BAR_VFULL + 2 * ws_vslots<D>(); }
constexpr int BAR_EPI = 3;   // named barrier of the tensor-core warpgroup (output epilogue)

struct WsSmem {  // byte offsets from a 1024-byte aligned base
  int rows;   // score rows [2][sw_bytes(n_k)] (block layout of lamp_ws_common.cuh)
  int v;      // V ring [S][D / 64][64 keys][64 dims] bf16, as the TMA leaves it (128-byte swizzle)
  int ks;     // producer K slices [8 warps][2][8][64] f32
  int q;      // Q [3][D][16] f32 (item k in slot k % 3)
  int list;   // consumer mask-word buffers [8][2][32] uint32
  int stats;  // per buffer and row: softmax max, normaliser [2][16][2] f32
  int otile;  // output tile of an item [16][D] bf16 (epilogue)
  int bars;   // mbarriers
  int sched;  // item ring [8] and its published count (ItemRing)
  int tmem;   // TMEM base address (written by tcgen05.alloc)
  int total;
};

template <int D>
__host__ __device__ inline WsSmem ws_plan(int n_k) {
  WsSmem s{};
  s.rows = 0;
  s.v = 2 * sw_bytes(n_k);
  s.ks = s.v + ws_vslots<D>() * ws_vtile_bytes<D>();
  s.q = s.ks + WS_NP * 2 * WS_DS * WS_UNIT * 4;
  s.list = s.q + 3 * ws_qfloats<D>() * 4;
  s.stats = s.list + WS_NC * 2 * SEL_WMAX * 4;
  s.otile = s.stats + 2 * WS_BM * 2 * 4;
  s.bars = s.otile + WS_BM * D * 2;
  s.sched = s.bars + (bar_drain<D>() + 1) * 8;
  s.tmem = s.sched + 16 * 4;
  s.total = s.tmem + 16;
  return s;
}

struct WsArgs {
  Problem p;
  const int* stats;   // per-(b, h) exponent statistics
  unsigned* counter;  // next item to hand out (zeroed by the preparation kernel)
  int nchunk;
  int n_items;
  int n_rb;
};


// Ring entries of this kernel: 2 q + f for item q (f = 1: the head's products
// admit the two-instruction rounding and the fused recompute), -1 for none left.
__device__ __forceinline__ int ring_q(int v) { return v >> 1; }
__device__ __forceinline__ bool ring_fast(int v) { return (v & 1) != 0; }

// ---------------------------------------------------------------------------
// Hand-out of the CTA's k-th item, by one warp of the tensor-core warpgroup:
// claims it from the work counter (heaviest first), reads its head's exponent
// statistics, stages its Q into slot k % 3 and publishes it in the ring. Items
// 0-2 go out at the start, item k + 3 after the output of item k, when every
// role is done with item k and so with slot k % 3; that is still an item ahead of
// the producers (they cannot store item k + 2 before that output is read). None
// of the global-memory latency of a hand-out sits on the path of the roles that
// wait for it. Returns false once no item is left (-1 published).
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ bool ws_hand_out(const WsArgs& a, unsigned char* smem, const WsSmem& L, int k, int lane) {
  const Problem& p = a.p;
  const ItemRing sched{smem_u32(smem + L.sched)};
  int q = lane == 0 ? claim_item(a.counter, a.n_items) : 0;
  q = __shfl_sync(0xFFFFFFFFu, q, 0);
  if (q < 0) {
    if (lane == 0) publish_item(sched, k, -1);
    return false;
  }
  const ItemInfo it = ws_decode(q, p, a.n_rb);
  const bool fast = head_fast_ok(a.stats + (size_t)it.bh * a.nchunk * 4, a.nchunk, p.emax_sum_limit);
  ws_stage_q<D>(reinterpret_cast<float*>(smem + L.q) + (k % 3) * ws_qfloats<D>(), p, it, lane, 32);
  __threadfence_block();
  __syncwarp();
  if (lane == 0) publish_item(sched, k, 2 * q + (fast ? 1 : 0));
  return true;
}

// ---------------------------------------------------------------------------
// Producers: PS(mu) scores of every item into the item's row buffer.
// ---------------------------------------------------------------------------
template <int D, int RND>
__device__ __forceinline__ void ws_producer(const WsArgs& a, unsigned char* smem, const WsSmem& L, int warp,
                                            int lane) {
  const Problem& p = a.p;
  const int s = 23 - p.mu;
  const u64 negc = pack2(-(float)((1u << s) - 1u), -(float)((1u << s) - 1u));
  const u64 pow2s = pack2((float)(1u << s), (float)(1u << s));
  const u64 scale2 = pack2(p.scale, p.scale);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  float* ksw = reinterpret_cast<float*>(smem + L.ks) + warp * 2 * WS_DS * WS_UNIT;
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  const int rb = sw_bytes(p.n_k);
  // failure-path tests: hand over nothing, so that every other warp's bounded wait runs out
  if (p.debug_stall == LAMP_DEBUG_STALL_PRODUCERS) return;
  const ItemRing sched{smem_u32(smem + L.sched)};
  int deal = 0;     // producer warp that takes the next unit
  for (int k = 0;; ++k) {
    const int buf = k & 1;
    const uint32_t ph = ((k - 2) >> 1) & 1;
    // item k, published with its Q staged by the hand-out (one decision per
    // warp: the tile routine synchronises the whole warp)
    int v = lane == 0 ? wait_published(sched, k) : 0;
    v = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (v == -2) {
      ws_timeout(p);
      return;
    }
    if (v < 0) break;
    const ItemInfo it = ws_decode(ring_q(v), p, a.n_rb);
    const float* sQ = qbase + (k % 3) * ws_qfloats<D>();
    const bool fast = (RND != kRndExact) && ring_fast(v);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    float* rows = reinterpret_cast<float*>(smem + L.rows + buf * rb);
    const int U = (it.kv_end + WS_UNIT - 1) / WS_UNIT;
    // the buffer itself is free once item k - 2's P.V has completed and its
    // output has been read (tfree): the tile routine waits for that only before
    // its first store. A warp without a unit in this item waits for it before its
    // arrival, so that no arrival on full[b] runs two items ahead of another's.
    const int first = (warp - deal + WS_NP) % WS_NP;
    if (!ws_produce_tile<D, RND, 2>(p, it, 0, it.kv_end, sQ, rows, ksw, lane, first, fast, Kh, negc, pow2s, scale2, s,
                                 k >= 2 ? bars + BAR_TFREE + buf : nullptr, ph) ||
        (first >= U && k >= 2 && !__all_sync(0xFFFFFFFFu, mbar_wait(bars + BAR_TFREE + buf, ph)))) {
      ws_timeout(p);
      return;
    }
    deal = (deal + U) % WS_NP;
    mbar_arrive(bars + BAR_FULL + buf);  // this thread's scores of item k are in place
  }
}

// ---------------------------------------------------------------------------
// Output of item k by the tensor-core warpgroup (warp 16 + ew reads TMEM lane
// quarter ew: head dimensions 32 ew + lane, or 16 ew + lane in lanes 0-15 for the
// M = 64 shape of d = 64). It waits for the item's MMAs, reads the accumulator
// (columns P_hi rows, then P_lo rows) and the rows' normalisers l, releases the
// buffer (tfree), then stores O / l as bf16 through a shared-memory tile with
// 16-byte stores. False when a bounded wait gave up (agreed by all 128 threads).
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ bool ws_epilogue(const Problem& p, const ItemInfo& it, uint64_t* bars, int k, uint32_t tbase,
                                            const float* stats, uint16_t* otile, int ew, int lane) {
  const int buf = k & 1;
  const bool ok = mbar_wait(bars + BAR_EMPTY + buf, (k >> 1) & 1);
  if (named_or(BAR_EPI, 128, !ok)) return false;
  tc_fence_after();
  const float* st = stats + buf * WS_BM * 2;
  const uint32_t ta = tbase + 32 * buf + ((uint32_t)(32 * ew) << 16);
  float o[WS_BM];
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // rows 8h .. 8h + 7
    float hi[8], lo[8];
    tmem_ld8(ta + 8 * h, hi);
    tmem_ld8(ta + 16 + 8 * h, lo);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float lv = st[2 * (8 * h + j) + 1];
      o[8 * h + j] = lv > 0.f ? __fadd_rn(hi[j], lo[j]) * (1.f / lv) : 0.f;
    }
  }
  tc_fence_before();
  mbar_arrive(bars + BAR_TFREE + buf);  // accumulator, row statistics and row buffer are free
  const int dim = D == 128 ? 32 * ew + lane : 16 * ew + lane;
  if (D == 128 || lane < 16) {
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
  return true;
}

// ---------------------------------------------------------------------------
// Consumers: selection, recompute, softmax and the output of every item.
// ---------------------------------------------------------------------------
template <int D, int RND, int VAR>
__device__ __forceinline__ void ws_consumer(const WsArgs& a, unsigned char* smem, const WsSmem& L, int cw, int lane) {
  constexpr int NCT = WS_NC * 32;  // consumer threads
  const Problem& p = a.p;
  const int nwords = (p.n_k + 31) >> 5;
  const bool refine_ok = VAR != LAMP_GIVEN_MASK && isfinite(p.tau) && p.tau >= 0.f;
  const float band = WS_BAND * p.tau;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(smem + L.list) + cw * 2 * SEL_WMAX;
  float* qbase = reinterpret_cast<float*>(smem + L.q);
  const int rb = sw_bytes(p.n_k);
  const ItemRing sched{smem_u32(smem + L.sched)};
  long long nsel = 0;
  for (int k = 0;; ++k) {
    // item k (published before the producers started it), then its scores; the
    // barrier also makes all threads agree on a wait that gave up
    const int v = wait_published(sched, k);
    const int buf = k & 1;
    const bool ok = v != -2 && (v == -1 || mbar_wait(bars + BAR_FULL + buf, (k >> 1) & 1));
    if (named_or(BAR_CONS, NCT, !ok)) {
      ws_timeout(p);
      return;
    }
    if (v < 0) break;
    const int q = ring_q(v);
    const ItemInfo it = ws_decode(q, p, a.n_rb);
    const uint16_t* Kh = p.K + (size_t)it.bh * p.n_k * D;
    const bool fast = (RND != kRndExact) && ring_fast(v);
    const float* sQ = qbase + (k % 3) * ws_qfloats<D>();
    float* rows = reinterpret_cast<float*>(smem + L.rows + buf * rb);
    float* st = reinterpret_cast<float*>(smem + L.stats) + buf * WS_BM * 2;
    const int written = ((it.kv_end + WS_UNIT - 1) / WS_UNIT) * WS_UNIT;  // keys the producers wrote

    // ---- selection and recompute, rows 2cw and 2cw + 1 ------------------------------
    // Keys past a row's valid range hold -inf: their criterion is NaN, which no
    // comparison selects, so the hot loops need no validity test.
    int rr_[2], nv[2];
    size_t grow[2];
    SelRows S;
    S.base = rows;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      rr_[t] = 2 * cw + t;
      nv[t] = rr_[t] < it.rows ? ws_valid_keys(it.i0 + rr_[t], p) : 0;
      grow[t] = (size_t)it.bh * p.n_q + it.i0 + rr_[t];
      S.rr[t] = rr_[t];
      S.off[t] = sw_off(rr_[t], lane);
      S.nv[t] = nv[t];
      S.word0[t] = grow[t] * nwords;
      S.live[t] = rr_[t] < it.rows;
      S.mx[t] = -INFINITY;
      S.mrun[t] = -INFINITY;
    }
    // keys 128 i4 + 4 lane .. + 3 of row rr_[t]: scores at ob[t] + 2048 i4, P_hi at pbo[t] + 2048 i4
    const int ob[2] = {sw_off(rr_[0], 4 * lane), sw_off(rr_[1], 4 * lane)};
    const int pbo[2] = {p_off(rr_[0], 4 * lane), p_off(rr_[1], 4 * lane)};
    const int nvmax = max(nv[0], nv[1]);
    const int nit = (nvmax + 127) >> 7;
    if (p.ps_out) {  // dump of the low-precision scores (before any recompute)
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (rr_[t] < it.rows)
          for (int j = lane; j < p.n_k; j += 32)
            p.ps_out[grow[t] * p.n_k + j] = j < written ? rows[sw_off(rr_[t], j)] : -INFINITY;
    }
    if (VAR == LAMP_STRICT) {
      // A: maximum and first argmax of each row
      float m[2] = {-INFINITY, -INFINITY};
      int am[2] = {0x7FFFFFFF, 0x7FFFFFFF};
      for (int i4 = 0; i4 < nit; ++i4) {
        const int j0 = 128 * i4 + 4 * lane;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const float4 v = lds4_or_ninf(rows + ob[t] + 2048 * i4, j0 < written);
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
          float4 v = lds4_or_ninf(rows + ob[t] + 2048 * i4, j0 < written);
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
      rows[sw_off(2 * cw + t, j)] = v;
      if (t == 0) S.mx[0] = fmaxf(S.mx[0], v);
      else S.mx[1] = fmaxf(S.mx[1], v);
    });
    __syncwarp();
    if (p.mixed_out) {  // dump of the mixed scores
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (rr_[t] < it.rows)
          for (int j = lane; j < p.n_k; j += 32)
            p.mixed_out[grow[t] * p.n_k + j] = j < written ? rows[sw_off(rr_[t], j)] : -INFINITY;
    }

    // D: softmax numerators of the mixed rows, written in place as the bf16 hi and
    // lo parts of the P.V operand; the maximum m' of each mixed row was tracked
    // through the selection and the recompute
    const int nitw = (written + 127) >> 7;
    float mm[2], mL[2], l[2] = {0.f, 0.f};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      mm[t] = warp_max_redux(S.mx[t]);
      mL[t] = mm[t] == -INFINITY ? 0.f : mm[t] * kLog2e;
    }
    for (int i4 = 0; i4 < nitw; ++i4) {
      const int j0 = 128 * i4 + 4 * lane;
      const bool act = j0 < written;
      float4 v[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) v[t] = act ? *reinterpret_cast<const float4*>(rows + ob[t] + 2048 * i4)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
      __syncwarp();  // the 128 keys of both rows are read before any lane overwrites them
      if (act) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const float vv[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
          uint32_t pw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float pj;  // exp(y - m'), 0 for -inf
            asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(pj) : "f"(fmaf(vv[e], kLog2e, -mL[t])));
            l[t] += pj;
            pw[e] = p_pair_cvt(pj);  // low half bf16(P), high half bf16(P - bf16(P))
          }
          float* dst = rows + pbo[t] + 2048 * i4;
          *reinterpret_cast<uint2*>(dst) = make_uint2(__byte_perm(pw[0], pw[1], 0x5410), __byte_perm(pw[2], pw[3], 0x5410));
          *reinterpret_cast<uint2*>(dst + 512) =
              make_uint2(__byte_perm(pw[0], pw[1], 0x7632), __byte_perm(pw[2], pw[3], 0x7632));
        }
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
    fence_async_smem();  // P (generic-proxy stores) becomes visible to the tensor core
    named_sync(BAR_CONS, NCT);  // every P row of the item is in place; Q of the item is no longer read
    mbar_arrive(bars + BAR_PREADY + buf);  // P of item k in place
  }
  if (lane == 0 && nsel && p.nsel_out) atomicAdd(p.nsel_out, (unsigned long long)nsel);
}

// ---------------------------------------------------------------------------
// Tensor-core warpgroup (warps 16-19, ew = warp - 16). Per item, lane 0 of warp
// 16 streams the V tiles by TMA and issues P.V by tcgen05.mma, then the four
// warps run the item's output epilogue.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void ws_tensor_warpgroup(const WsArgs& a, const CUtensorMap* tmV, unsigned char* smem,
                                                    const WsSmem& L, uint32_t tbase, int ew, int lane) {
  constexpr int S = ws_vslots<D>();
  constexpr uint32_t TB = ws_vtile_bytes<D>();
  const Problem& p = a.p;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  unsigned char* vring = smem + L.v;
  const uint32_t vbase = smem_u32(vring), rbase = smem_u32(smem + L.rows);
  const int rb = sw_bytes(p.n_k);
  const uint32_t idesc = umma_idesc_bf16(D, 32);
  const bool issuer = ew == 0 && lane == 0;
  bool ok = true;
  // V tiles form one sequence over the CTA's items: tile tl of item kl is number gl
  int kl = 0, tl = 0, Tl = -1, bhl = 0;
  int gl = 0, gm = 0;  // next tile to load, next tile to multiply
  const ItemRing sched{smem_u32(smem + L.sched)};
  auto next_tile = [&]() -> bool {  // false: no further tile known yet (or none left)
    for (;;) {
      if (Tl < 0) {
        if (sched.count() <= kl) return false;  // item kl is not claimed yet
        __threadfence_block();
        const int v = sched.get(kl);
        if (v < 0) return false;
        const ItemInfo it = ws_decode(ring_q(v), p, a.n_rb);
        Tl = (it.kv_end + WS_VKEYS - 1) / WS_VKEYS;
        bhl = it.bh;
        tl = 0;
      }
      if (tl < Tl) return true;
      ++kl;
      Tl = -1;
    }
  };
  auto load_upto = [&](int limit) {  // start the loads of tiles gl .. limit - 1
    while (ok && gl < limit && next_tile()) {
      const int slot = gl % S;
      if (gl >= S && !mbar_wait(bars + bar_vempty<D>() + slot, ((gl / S) - 1) & 1)) {  // its MMAs have read it
        ok = false;
        break;
      }
      mbar_expect_tx(bars + BAR_VFULL + slot, TB);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(vring + slot * TB + h * 8192, tmV, 64 * h, WS_VKEYS * tl, bhl, bars + BAR_VFULL + slot);
      ++tl;
      ++gl;
    }
  };
  // P.V of item k (the issuing thread only)
  auto mma_item = [&](int k, const ItemInfo& it) {
    const int buf = k & 1;
    const int T = (it.kv_end + WS_VKEYS - 1) / WS_VKEYS;
    load_upto(gm + S);
    if (!ok || !mbar_wait(bars + BAR_PREADY + buf, (k >> 1) & 1)) {
      ok = false;
      return;
    }
    tc_fence_after();
    const uint32_t dcol = tbase + 32 * buf;
    const uint32_t pb = rbase + buf * rb;
    for (int t = 0; t < T; ++t, ++gm) {
      load_upto(gm + S - 1);  // keep the ring full (waits for the MMAs two tiles back)
      const int slot = gm % S;
      if (!ok || !mbar_wait(bars + BAR_VFULL + slot, (gm / S) & 1)) {
        ok = false;
        return;
      }
      tc_fence_after();
      const uint32_t va = vbase + slot * TB, pa = pb + t * 4096;
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) {  // 16 keys per MMA
        const uint64_t ad = umma_desc_sw128(va + s4 * 2048, D == 128 ? 8192u : 0u, 1024);
        const uint64_t bd = umma_desc_sw128(pa + s4 * 32, 16, 1024);
        umma_bf16(dcol, ad, bd, idesc, (t | s4) != 0);
      }
      umma_commit(bars + bar_vempty<D>() + slot);  // V slot free once these MMAs are done
    }
    umma_commit(bars + BAR_EMPTY + buf);  // the item's P.V is complete
  };
  const float* stats = reinterpret_cast<const float*>(smem + L.stats);
  uint16_t* otile = reinterpret_cast<uint16_t*>(smem + L.otile);
  bool good = true;
  // items 0-2 at the start, item k + 3 after item k's output
  const bool handler = ew == 1;
  bool more = true;
  for (int k0 = 0; handler && more && k0 < 3; ++k0) more = ws_hand_out<D>(a, smem, L, k0, lane);
  for (int k = 0;; ++k) {
    const int v = wait_published(sched, k);
    if (named_or(BAR_EPI, 128, v == -2)) {  // the wait gave up (all four warps agree)
      good = false;
      break;
    }
    if (v < 0) break;
    const ItemInfo it = ws_decode(ring_q(v), p, a.n_rb);
    if (issuer && ok) mma_item(k, it);
    __syncwarp();
    // a failed issue leaves the item's accumulator incomplete: the epilogue's
    // bounded wait then gives up, and all four warps agree on it
    if (!ws_epilogue<D>(p, it, bars, k, tbase, stats, otile, ew, lane)) {
      good = false;
      break;
    }
    if (handler && more) more = ws_hand_out<D>(a, smem, L, k + 3, lane);
  }
  if (issuer) {
    // drain: every MMA issued and every V load in flight completes before the
    // tensor memory is released and the CTA exits
    umma_commit(bars + bar_drain<D>());
    bool drained = mbar_wait(bars + bar_drain<D>(), 0);
    for (int g = gm; g < gl; ++g) drained = mbar_wait(bars + BAR_VFULL + g % S, (g / S) & 1) && drained;
    if (!ok || !drained) good = false;
  }
  if (!good && lane == 0) ws_timeout(p);
}

template <int D, int RND, int VAR>
__global__ void __launch_bounds__(WS_NT, 1) ws_kernel(const WsArgs a, const __grid_constant__ CUtensorMap tmV) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + smem_align1k_pad(smem_raw);
  const WsSmem L = ws_plan<D>(a.p.n_k);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L.tmem);
  if (threadIdx.x == 0) {
    mbar_init(bars + BAR_FULL + 0, WS_NP * 32);
    mbar_init(bars + BAR_FULL + 1, WS_NP * 32);
    mbar_init(bars + BAR_PREADY + 0, WS_NC * 32);
    mbar_init(bars + BAR_PREADY + 1, WS_NC * 32);
    mbar_init(bars + BAR_EMPTY + 0, 1);
    mbar_init(bars + BAR_EMPTY + 1, 1);
    mbar_init(bars + BAR_TFREE + 0, 128);
    mbar_init(bars + BAR_TFREE + 1, 128);
    for (int i = 0; i < ws_vslots<D>(); ++i) {
      mbar_init(bars + BAR_VFULL + i, 1);
      mbar_init(bars + bar_vempty<D>() + i, 1);
    }
    mbar_init(bars + bar_drain<D>(), 1);
    mbar_fence_init();
    const ItemRing sched{smem_u32(smem + L.sched)};
    sched.set_count(0);  // no item published yet
  }
  if (warp == WS_MW) tmem_alloc(tslot, WS_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  if (warp < WS_NP) {
    regs_inc<kWsProdRegs>();
    ws_producer<D, RND>(a, smem, L, warp, lane);
  } else if (warp < WS_MW) {
    regs_inc<kWsConsRegs>();
    ws_consumer<D, RND, VAR>(a, smem, L, warp - WS_NP, lane);
  } else {
    regs_dec<kWsMmaRegs>();
    ws_tensor_warpgroup<D>(a, &tmV, smem, L, tbase, warp - WS_MW, lane);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WS_MW) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, WS_TMEM_COLS);
  }
}

template <int D, int RND, int VAR>
cudaError_t ws_launch_one(const WsArgs& a, const CUtensorMap& tmV, int grid, size_t smem, cudaStream_t st) {
  auto k = ws_kernel<D, RND, VAR>;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k);
  if (e != cudaSuccess) return e;
  // the register split assumes this pool, and the block must be launchable with it
  if (fa.numRegs != kWsLaunchRegs || fa.maxThreadsPerBlock < WS_NT) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, WS_NT, smem, st>>>(a, tmV);
  return cudaGetLastError();
}

template <int D, int RND>
cudaError_t ws_launch_var(const WsArgs& a, const CUtensorMap& tmV, int grid, size_t smem, cudaStream_t st) {
  if (a.p.variant == LAMP_RELAXED) return ws_launch_one<D, RND, LAMP_RELAXED>(a, tmV, grid, smem, st);
  if (a.p.variant == LAMP_GIVEN_MASK) return ws_launch_one<D, RND, LAMP_GIVEN_MASK>(a, tmV, grid, smem, st);
  return ws_launch_one<D, RND, LAMP_STRICT>(a, tmV, grid, smem, st);
}

}  // namespace

size_t ws_smem_bytes(int d, int n_k) {  // dynamic shared memory of a launch (with the 1024-byte alignment slack)
  return (d == 64 ? (size_t)ws_plan<64>(n_k).total : (size_t)ws_plan<128>(n_k).total) + 1024;
}

bool ws_fits(int d, int n_k, size_t smem_optin) {
  return n_k <= 32 * SEL_WMAX && ws_smem_bytes(d, n_k) + kStaticSmemReserve <= smem_optin;
}

cudaError_t launch_ws(const Problem& p, const Workspace& ws, char* base, int num_sms, cudaStream_t st) {
  WsArgs a;
  a.p = p;
  a.stats = reinterpret_cast<const int*>(base + ws.stats);
  a.counter = reinterpret_cast<unsigned*>(base + ws.counters);
  a.nchunk = ws.nchunk;
  a.n_rb = (p.n_q + WS_BM - 1) / WS_BM;
  a.n_items = a.n_rb * p.B * p.H;
  CUtensorMap tmV;
  cudaError_t e = make_tmap_bf16(&tmV, p.V, p.d, p.n_k, p.B * p.H, 64, WS_VKEYS, 128);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  const size_t smem = ws_smem_bytes(p.d, p.n_k);
  const int rnd = p.mu == 23 ? kRndNone : (p.mu <= 10 ? kRndFast : kRndExact);
  if (p.d == 64) {
    if (rnd == kRndFast) return ws_launch_var<64, kRndFast>(a, tmV, grid, smem, st);
    if (rnd == kRndNone) return ws_launch_var<64, kRndNone>(a, tmV, grid, smem, st);
    return ws_launch_var<64, kRndExact>(a, tmV, grid, smem, st);
  }
  if (rnd == kRndFast) return ws_launch_var<128, kRndFast>(a, tmV, grid, smem, st);
  if (rnd == kRndNone) return ws_launch_var<128, kRndNone>(a, tmV, grid, smem, st);
  return ws_launch_var<128, kRndExact>(a, tmV, grid, smem, st);
}

}  // namespace lamp
