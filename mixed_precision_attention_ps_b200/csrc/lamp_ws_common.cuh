// Device pieces shared by the warp-specialised LAMP kernels (whole-row and
// streamed): work order, Q staging, the layout of the score rows in shared
// memory, the producer's score tile and the FP32 recompute. Method: "LAMP: Look-Ahead Mixed-Precision Inference of Large
// Language Models" (technical summary, gist.science paper 2601.21623), sections
// "Implementation strategy" (steps 1 and 3) and "Experimental results" (PS(mu)).
#pragma once

#include <type_traits>

#include "lamp.h"
#include "lamp_device.cuh"
#include "lamp_kernels.h"
#include "lamp_umma.cuh"

namespace lamp {
namespace {

constexpr int WS_BM = 16;              // query rows per item
constexpr int WS_NT = kWsThreads;      // 640
constexpr int WS_NP = 8;               // producer warps
constexpr int WS_NC = 8;               // consumer warps
constexpr int WS_MW = WS_NP + WS_NC;   // the tensor-core warp (V tiles by TMA, P.V by tcgen05.mma), first of its warpgroup
constexpr int WS_UNIT = 64;            // keys per producer unit
constexpr int WS_DS = 8;               // head dimensions per K slice
constexpr float WS_BAND = 8e-6f;       // relative band around tau re-evaluated in double
constexpr int BAR_CONS = 1;            // named barrier of the consumer group
constexpr int WS_VKEYS = 64;           // keys per V tile (one TMA box of 64 keys x 64 dimensions per half)
constexpr int WS_TMEM_COLS = 64;       // two P.V accumulators of N = 32 columns (P_hi rows, P_lo rows)
// Per-warpgroup register budgets (setmaxnreg; every warp of a warpgroup executes
// the same one).
template <int N>
__device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

// Q of an item in shared memory: [D][16 rows] f32 (dimension-major, so a 16-byte
// load gives four rows of one dimension: the packed pairs of two row pairs)
template <int D>
__host__ __device__ constexpr int ws_qfloats() { return D * WS_BM; }

// ---------------------------------------------------------------------------
// Score rows of an item (16 query rows) in shared memory: blocks of 64 keys, 4096
// bytes each, laid out so that the softmax numerators can be written in place as
// the B operand of the P.V tensor-core product (K-major, 128-byte swizzle; see
// lamp_umma.cuh):
//   block b = j / 64 at 4096 b; half h = (j / 32) % 2 at 2048 h holds the fp32
//   scores of keys 32h .. 32h + 31 of the block; row r is the 128-byte line at
//   1024 (r / 8) + 128 (r % 8) of the half, and its 16-byte chunk c = (j % 32) / 4
//   sits at position c ^ (r % 8).
// After the softmax pass the same two lines of row r hold the block's 64 P_hi
// values (half 0) and P_lo values (half 1) as bf16, chunk (j % 64) / 8 at position
// ((j % 64) / 8) ^ (r % 8): a row's P overwrites only that row's own scores. A
// warp reading one row touches 32 consecutive keys per 128-byte line (no bank
// conflicts), and 4 consecutive keys are one 16-byte chunk.
// ---------------------------------------------------------------------------
constexpr int SW_BLOCK_FLOATS = 1024;  // one 64-key block of 16 rows

// Float index of score (r, j).
__device__ __forceinline__ int sw_off(int r, int j) {
  return ((j >> 6) << 10) | (((j >> 5) & 1) << 9) | ((r >> 3) << 8) | ((r & 7) << 5) |
         ((((j >> 2) & 7) ^ (r & 7)) << 2) | (j & 3);
}
// Float index of the 8 bytes that hold P_hi of keys j .. j + 3 (j a multiple of
// 4) of row r; P_lo follows at + 512 floats (2048 bytes).
__device__ __forceinline__ int p_off(int r, int j) {
  return ((j >> 6) << 10) | ((r >> 3) << 8) | ((r & 7) << 5) | ((((j >> 3) & 7) ^ (r & 7)) << 2) | ((j & 4) >> 1);
}
// Bytes of the score rows of an item with n keys.
__host__ __device__ constexpr int sw_bytes(int n) { return ((n + 63) / 64) * 4096; }

// Items are handed out at run time, heaviest first, from a global counter, so
// that CTAs which run slower (two SMs share a TPC's resources) take fewer. A
// CTA's k-th item goes to ring[k % 8] in shared memory (-1: none left), then the
// published count ring[8] (zeroed at kernel start) rises to k + 1; readers poll
// the count (bounded) or follow a barrier that orders them after the write.
// Who claims: in the streamed kernel items 0 and 1 by the producers at the start
// and item k + 2 by the consumers when they begin item k; in the whole-row
// kernel one warp of the tensor-core warpgroup, three items ahead (lamp_ws.cu).
constexpr int kRing = 8;
// Volatile 32-bit shared-memory accesses by shared-window address (the ring is
// polled by other warps of the CTA).
__device__ __forceinline__ int ld_volatile_shared(uint32_t addr) {
  int v;
  asm volatile("ld.volatile.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_volatile_shared(uint32_t addr, int v) {
  asm volatile("st.volatile.shared.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// The ring, addressed through its 32-bit shared-window address: ring[0..7] and
// the published count at [8].
struct ItemRing {
  uint32_t a;  // address of ring[0]
  __device__ __forceinline__ int get(int k) const { return ld_volatile_shared(a + 4 * (k & (kRing - 1))); }
  __device__ __forceinline__ int count() const { return ld_volatile_shared(a + 4 * kRing); }
  __device__ __forceinline__ void put(int k, int q) const { st_volatile_shared(a + 4 * (k & (kRing - 1)), q); }
  __device__ __forceinline__ void set_count(int n) const { st_volatile_shared(a + 4 * kRing, n); }
};
__device__ __forceinline__ int claim_item(unsigned* counter, int n_items) {
  const unsigned q = atomicAdd(counter, 1u);
  return q < (unsigned)n_items ? (int)q : -1;
}
__device__ __forceinline__ void publish_item(ItemRing r, int k, int q) {
  r.put(k, q);
  __threadfence_block();
  r.set_count(k + 1);
}
// Bounded wait until the CTA's k-th item is published: its number (-1: none),
// or -2 when the wait gave up.
__device__ __forceinline__ int wait_published(ItemRing r, int k) {
  if (r.count() <= k) {
    const uint64_t t0 = global_ns();
    while (r.count() <= k) {
      if (global_ns() - t0 > kWaitLimitNs) return -2;
      __nanosleep(32);
    }
  }
  __threadfence_block();
  return r.get(k);
}

struct ItemInfo {
  int bh, i0, rows, kv_end;
};

__device__ __forceinline__ ItemInfo ws_decode(int q, const Problem& p, int n_rb) {
  const int BH = p.B * p.H;
  ItemInfo it;
  const int rb = p.causal ? n_rb - 1 - q / BH : q / BH;
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

__device__ __forceinline__ void ws_timeout(const Problem& p) {
  if (p.status_out) atomicExch(p.status_out, LAMP_ERR_TIMEOUT);
}

// Q rows of an item as binary32 [D][16] (rows past the problem are zero).
// Thread u takes row u % 16 of the 8-dimension group u / 16, so that the 16
// lanes of a half-warp write 16 consecutive floats of each dimension.
template <int D>
__device__ __forceinline__ void ws_stage_q(float* sQ, const Problem& p, const ItemInfo& it, int t, int nthreads) {
  for (int u = t; u < WS_BM * D / 8; u += nthreads) {
    const int r = u % WS_BM, c8 = (u / WS_BM) * 8;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (r < it.rows) w = __ldg(reinterpret_cast<const uint4*>(p.Q + ((size_t)it.bh * p.n_q + it.i0 + r) * D + c8));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sQ[(c8 + 2 * e) * WS_BM + r] = bf16_lo(ws[e]);
      sQ[(c8 + 2 * e + 1) * WS_BM + r] = bf16_hi(ws[e]);
    }
  }
}

// WS_DS accumulation steps of a lane's 8-row x 4-key tile; the packed pairs run
// over rows: acc[rp][i] holds rows 8gr + 2rp, 8gr + 2rp + 1 at key 4gk + i.
//   qs: Q of this slice, [WS_DS][16] f32 (lane rows 8gr..8gr+7 at qoff = 8gr);
//   ks: warp's K slice, [WS_DS][64] f32 (lane keys at koff = 4gk).
// KU: steps unrolled together. The whole-row kernel takes 2: its producer loop
// then fits the instruction cache that the five warp roles of an SM share
// (GPT-2 XL strict 0.219 -> 0.211 ms, batch 8 relaxed 1.62 -> 1.39 ms against
// all 8); the streamed kernel at d = 128 keeps all 8 (2 was 1.5 % slower there).
template <int MODE, int KU>
__device__ __forceinline__ void ws_score_slice(const float* __restrict__ qs, const float* __restrict__ ks, int qoff,
                                               int koff, u64 (&acc)[4][4], u64 negc, u64 pow2s, int s) {
#pragma unroll KU
  for (int dd = 0; dd < WS_DS; ++dd) {
    const ulonglong2 qa = *reinterpret_cast<const ulonglong2*>(qs + dd * WS_BM + qoff);
    const ulonglong2 qb = *reinterpret_cast<const ulonglong2*>(qs + dd * WS_BM + qoff + 4);
    const float4 kk = *reinterpret_cast<const float4*>(ks + dd * WS_UNIT + koff);
    const u64 q[4] = {qa.x, qa.y, qb.x, qb.y};
    const u64 k[4] = {pack2(kk.x, kk.x), pack2(kk.y, kk.y), pack2(kk.z, kk.z), pack2(kk.w, kk.w)};
#pragma unroll
    for (int rp = 0; rp < 4; ++rp)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[rp][i] = ps_step<MODE>(q[rp], k[i], acc[rp][i], negc, pow2s, s);
  }
}

// Scores of one tile of an item, keys t0 .. t0 + tlen - 1, by one producer warp:
// the tile's 64-key units j = first, first + 8, ... (the others belong to the other
// producer warps). The scores of key t0 + c go to rows[sw_off(r, c)] for the 16
// rows r of the item (the block layout above); keys past a row's valid range hold
// -inf.
// K slices travel global -> registers -> shared memory (binary32) two stream
// positions ahead of their use, so an L2 round trip hides behind two slices of
// arithmetic. (A TMA load of each bf16 slice, a box of 64 rows of 16 bytes, into
// a ring that the warp then widens was measured 15 % slower on the streamed
// kernel.) The buffer may still be read by the tensor core when the call
// starts: the warp waits for free_bar's phase free_phase (when free_bar is not
// null) only before its first store, one unit of arithmetic later. Returns false
// when that bounded wait gave up.
template <int D, int RND, int KU>
__device__ __forceinline__ bool ws_produce_tile(const Problem& p, const ItemInfo& it, int t0, int tlen,
                                                const float* sQ, float* rows, float* ksw, int lane, int first,
                                                bool fast, const uint16_t* Kh, u64 negc, u64 pow2s, u64 scale2,
                                                int s, uint64_t* free_bar, uint32_t free_phase) {
  constexpr int NSL = D / WS_DS;  // K slices per unit
  const int gr = lane & 1, gk = lane >> 1;  // rows 8gr..8gr+7, keys 4gk..4gk+3 of a unit
  const int qoff = 8 * gr, koff = 4 * gk;
  const int U = (tlen + WS_UNIT - 1) / WS_UNIT;
  const int mine = first < U ? (U - first + WS_NP - 1) / WS_NP : 0;
  const int total = mine * NSL;
  uint4 kra[2], krb[2];
  auto load = [&](int pos, uint4 (&kr)[2]) {  // keys lane and lane + 32 of the slice at pos
    const int j = first + WS_NP * (pos / NSL), sl = pos % NSL;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int key = t0 + j * WS_UNIT + lane + 32 * h;
      kr[h] = make_uint4(0u, 0u, 0u, 0u);
      if (key < it.kv_end) kr[h] = __ldg(reinterpret_cast<const uint4*>(Kh + (size_t)key * D + sl * WS_DS));
    }
  };
  auto widen = [&](int b2, const uint4 (&kr)[2]) {  // binary32 [8 dims][64 keys] into slice buffer b2
    float* dst = ksw + b2 * WS_DS * WS_UNIT + lane;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t ws[4] = {kr[h].x, kr[h].y, kr[h].z, kr[h].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dst[(2 * e) * WS_UNIT + 32 * h] = bf16_lo(ws[e]);
        dst[(2 * e + 1) * WS_UNIT + 32 * h] = bf16_hi(ws[e]);
      }
    }
  };
  bool failed = false;
  u64 acc[4][4];
  // one stream position: compute slice pos, then stage slice pos + 1 into the free
  // binary32 buffer and start the load of slice pos + 3 into `cur` (the register
  // set of pos + 1; two sets alternate, so no load is waited on early)
  auto body = [&](auto mode, int pos, uint4 (&cur)[2]) {
    const int j = first + WS_NP * (pos / NSL), sl = pos % NSL;
    if (sl == 0) {
#pragma unroll
      for (int rp = 0; rp < 4; ++rp)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[rp][i] = 0ull;
    }
    const float* qs = sQ + sl * WS_DS * WS_BM;
    const float* ks = ksw + (pos & 1) * WS_DS * WS_UNIT;
    ws_score_slice<decltype(mode)::value, KU>(qs, ks, qoff, koff, acc, negc, pow2s, s);
    if (sl == NSL - 1) {
      if (free_bar) {  // first store of the call: the buffer's previous contents are no longer read
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(free_bar, free_phase))) {
          failed = true;
          return;
        }
        free_bar = nullptr;
      }
      const int c0 = j * WS_UNIT + koff;  // lane's first column, relative to the tile
      const int j0 = t0 + c0;             // ... and as an absolute key
#pragma unroll
      for (int rp = 0; rp < 4; ++rp) {
        const int r0 = 8 * gr + 2 * rp;
        const int nv0 = r0 < it.rows ? ws_valid_keys(it.i0 + r0, p) : 0;
        const int nv1 = r0 + 1 < it.rows ? ws_valid_keys(it.i0 + r0 + 1, p) : 0;
        float4 y0, y1;
        const u64 a0 = mul2u(acc[rp][0], scale2), a1 = mul2u(acc[rp][1], scale2);
        const u64 a2 = mul2u(acc[rp][2], scale2), a3 = mul2u(acc[rp][3], scale2);
        y0.x = j0 < nv0 ? lo_f(a0) : -INFINITY;
        y0.y = j0 + 1 < nv0 ? lo_f(a1) : -INFINITY;
        y0.z = j0 + 2 < nv0 ? lo_f(a2) : -INFINITY;
        y0.w = j0 + 3 < nv0 ? lo_f(a3) : -INFINITY;
        y1.x = j0 < nv1 ? hi_f(a0) : -INFINITY;
        y1.y = j0 + 1 < nv1 ? hi_f(a1) : -INFINITY;
        y1.z = j0 + 2 < nv1 ? hi_f(a2) : -INFINITY;
        y1.w = j0 + 3 < nv1 ? hi_f(a3) : -INFINITY;
        *reinterpret_cast<float4*>(rows + sw_off(r0, c0)) = y0;
        *reinterpret_cast<float4*>(rows + sw_off(r0 + 1, c0)) = y1;
      }
    }
    __syncwarp();  // every lane is done reading slice pos - 1's buffer
    if (pos + 1 < total) widen((pos + 1) & 1, cur);
    if (pos + 3 < total) load(pos + 3, cur);
    __syncwarp();
  };
  if (total > 0) {
    load(0, kra);
    widen(0, kra);
  }
  if (total > 1) load(1, kra);
  if (total > 2) load(2, krb);
  __syncwarp();
  // one step form for the whole tile: the exact rounding's loop is a separate
  // copy, so that its code does not sit inside the fast loop (with the branch in
  // the loop, 3 % of a GPT-2 XL call went to the instruction fetch of the other
  // warp roles)
  auto run = [&](auto mode) {
    for (int pos = 0; pos < total && !failed; pos += 2) {
      body(mode, pos, kra);
      if (pos + 1 < total && !failed) body(mode, pos + 1, krb);
    }
  };
  if (RND != kRndExact && fast) run(std::integral_constant<int, RND == kRndFast ? kStepFast : kStepF32>{});
  else run(std::integral_constant<int, kStepExact>{});
  return !failed;  // (a warp with no unit of its own writes nothing and so needs no wait)
}

// FP32 recompute of score (row r, key j): the sequential binary32 sum over
// k = 0..D-1 (a fused multiply-add when the head's products are exact), then the scale.
template <int D>
__device__ __forceinline__ float ws_recompute(const float* __restrict__ sQ, int r, const uint16_t* __restrict__ krow,
                                              float scale, bool fused) {
  float acc = 0.f;
#pragma unroll
  for (int kk = 0; kk < D; kk += 8) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(krow + kk));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float k0 = bf16_lo(ws[e]), k1 = bf16_hi(ws[e]);
      const float q0 = sQ[(kk + 2 * e) * WS_BM + r], q1 = sQ[(kk + 2 * e + 1) * WS_BM + r];
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

__device__ __forceinline__ float4 lds4_or_ninf(const float* ptr, bool ok) {
  return ok ? *reinterpret_cast<const float4*>(ptr) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
}

// ---------------------------------------------------------------------------
// Selection pass of a consumer warp: the look-ahead test on its two rows, 128 keys
// per step. Lane l takes keys kb + 32 m + l (m = 0..3) of step kb, so the ballot
// of key column m over the lanes is mask word kb / 32 + m itself. The words go to
// a per-warp buffer in shared memory; after the pass one scan over the buffer
// gives every selected key its recompute slot and the words leave for mask_out
// in one coalesced store per row.
// ---------------------------------------------------------------------------
constexpr int SEL_WMAX = 32;  // mask words per row a pass holds (1024 keys)

struct SelRows {
  float* base;       // the item's score rows (block layout, sw_off)
  int rr[2];         // the warp's two rows (key j of the pass at base[sw_off(rr[t], j)])
  int off[2];        // sw_off(rr[t], lane): key kb + 32 m + lane (kb a multiple of 128) is at off + 16 kb + 512 m
  int nv[2];         // valid keys of each row, counted from the pass's key 0
  size_t word0[2];   // mask word of the pass's key 0 in mask_out / mask_in
  bool live[2];      // the row exists (only live rows write mask words)
  float mx[2];       // running maximum of the mixed row (kept and recomputed scores)
  float mrun[2];     // relaxed: running maximum of the low-precision scores over 64-key tiles
  // strict: statistics of the low-precision row (maximum m, first argmax am,
  // S = 1 + S_rest in double and binary32, 2 / S^2 in binary32)
  float mL[2], Sf[2], c2[2], srest_f[2], m[2];
  double Sd[2], srest[2];
  int am[2];
};

// One step (keys kb .. kb + 127 of the pass). `written` bounds the keys holding
// scores (a multiple of 64); keys at or past it read as -inf. wbuf is the warp's
// [2][SEL_WMAX] word buffer.
template <int VAR>
__device__ __forceinline__ void sel_step(const Problem& p, SelRows& S, int kb, int written, int nwords_left,
                                         float tlo, float thi, int lane, uint32_t* wbuf, long long& nsel) {
  float y[2][4];
  uint32_t sel[2] = {0u, 0u}, nearb[2] = {0u, 0u};
  float mh[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // relaxed: running maximum for columns 0-1 and 2-3
#pragma unroll
  for (int t = 0; t < 2; ++t) {
#pragma unroll
    for (int m = 0; m < 4; ++m) y[t][m] = kb + 32 * m < written ? S.base[S.off[t] + 16 * kb + 512 * m] : -INFINITY;
    if (VAR == LAMP_GIVEN_MASK) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int w = (kb >> 5) + m;
        const uint32_t word = w < nwords_left ? __ldg(p.mask_in + S.word0[t] + w) : 0u;
        sel[t] |= (uint32_t)(((word >> lane) & 1u) && kb + 32 * m + lane < S.nv[t]) << m;
      }
    } else if (VAR == LAMP_RELAXED) {
      // 64-key tiles: columns 0-1 form one, columns 2-3 the next
      const float ta = warp_max_redux(fmaxf(y[t][0], y[t][1]));
      const float tb = warp_max_redux(fmaxf(y[t][2], y[t][3]));
      mh[t][0] = fmaxf(S.mrun[t], ta);
      mh[t][1] = fmaxf(mh[t][0], tb);
      S.mrun[t] = mh[t][1];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float ex;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ex) : "f"(fmaf(y[t][m], kLog2e, -(mh[t][m >> 1] * kLog2e))));
        const float cr = 2.f * fabsf(y[t][m]) * ex;
        sel[t] |= (uint32_t)(cr > p.tau) << m;
        nearb[t] |= (uint32_t)(cr >= tlo && cr <= thi) << m;
      }
    } else {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float ex;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ex) : "f"(fmaf(y[t][m], kLog2e, -S.mL[t])));
        const float om = __fsub_rn(S.Sf[t], ex);
        const float cr = (fabsf(y[t][m]) * ex) * (om * S.c2[t]);
        sel[t] |= (uint32_t)(cr > p.tau) << m;
        nearb[t] |= (uint32_t)(cr >= tlo && cr <= thi) << m;
      }
      const int da = S.am[t] - kb;
      if (da >= 0 && da < 128 && (da & 31) == lane) {  // the argmax: z = 1 / S, 1 - z = S_rest / S
        const int ma = da >> 5;
        const float ya = ma == 0 ? y[t][0] : (ma == 1 ? y[t][1] : (ma == 2 ? y[t][2] : y[t][3]));
        const float cr = fabsf(ya) * (S.srest_f[t] * S.c2[t]);
        sel[t] = (sel[t] & ~(1u << ma)) | ((uint32_t)(cr > p.tau) << ma);
        nearb[t] = (nearb[t] & ~(1u << ma)) | ((uint32_t)(cr >= tlo && cr <= thi) << ma);
      }
    }
  }
  if (VAR != LAMP_GIVEN_MASK && __any_sync(0xFFFFFFFFu, (nearb[0] | nearb[1]) != 0u)) {
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if ((nearb[t] >> m) & 1u) {  // close to tau: the test again in double
          const double yd = (double)y[t][m];
          double cd;
          if (VAR == LAMP_RELAXED) {
            cd = 2.0 * exp(yd - (double)mh[t][m >> 1]) * fabs(yd);
          } else {
            const bool isa = kb + 32 * m + lane == S.am[t];
            const double ed = isa ? 1.0 : exp(yd - (double)S.m[t]);
            const double z = ed / S.Sd[t];
            const double omz = isa ? S.srest[t] / S.Sd[t] : (S.Sd[t] - ed) / S.Sd[t];
            cd = 2.0 * z * omz * fabs(yd);
          }
          sel[t] = (sel[t] & ~(1u << m)) | ((uint32_t)(cd > (double)p.tau) << m);
        }
  }
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, (sel[t] >> m) & 1u);
      if (lane == 4 * t + m) wbuf[t * SEL_WMAX + (kb >> 5) + m] = bal;
      nsel += __popc(bal);
      if (!((sel[t] >> m) & 1u)) S.mx[t] = fmaxf(S.mx[t], y[t][m]);
    }
}

// After the pass: the first nw mask words of each row are in wbuf. Writes them
// (and zeros up to nwrite words) to mask_out, then hands every selected key to
// rec(t, j) (row t of the warp, key j of the pass), 32 keys per warp round.
template <typename Rec>
__device__ __forceinline__ void sel_finish(const Problem& p, const SelRows& S, const uint32_t* wbuf, int nw,
                                           int nwrite, int lane, Rec&& rec) {
  __syncwarp();
  const uint32_t w0 = lane < nw ? wbuf[lane] : 0u;
  const uint32_t w1 = lane < nw ? wbuf[SEL_WMAX + lane] : 0u;
  if (p.mask_out) {
    if (S.live[0])
      for (int w = lane; w < nwrite; w += 32) p.mask_out[S.word0[0] + w] = w == lane ? w0 : 0u;
    if (S.live[1])
      for (int w = lane; w < nwrite; w += 32) p.mask_out[S.word0[1] + w] = w == lane ? w1 : 0u;
  }
  const int c0 = __popc(w0), cnt = c0 + __popc(w1);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  for (int base = 0; base < total; base += 32) {
    const int e = base + lane;  // this lane's entry: owner lane L has incl[L - 1] <= e < incl[L]
    int L = 0;
#pragma unroll
    for (int step = 16; step > 0; step >>= 1)
      if (__shfl_sync(0xFFFFFFFFu, incl, L + step - 1) <= e) L += step;
    const uint32_t a0 = __shfl_sync(0xFFFFFFFFu, w0, L), a1 = __shfl_sync(0xFFFFFFFFu, w1, L);
    const int r = e - (__shfl_sync(0xFFFFFFFFu, incl, L) - __popc(a0) - __popc(a1));
    if (e < total) {
      const int ca = __popc(a0);
      const int t = r < ca ? 0 : 1;
      const uint32_t word = t == 0 ? a0 : a1;
      const int bit = __fns(word, 0, (t == 0 ? r : r - ca) + 1);
      rec(t, 32 * L + bit);
    }
  }
}

}  // namespace
}  // namespace lamp
