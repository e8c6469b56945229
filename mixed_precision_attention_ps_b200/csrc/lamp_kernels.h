// Host-side launch interface between the C ABI (lamp_api.cu) and the kernels.
// Plain pointers and sizes only.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "lamp.h"

namespace lamp {

// Rounding class of mu, fixed per launch:
//   kRndFast : mu in [1, 10]  (two-instruction rounding when the head allows it,
//                              exact integer rounding otherwise)
//   kRndExact: mu in [11, 22] (exact integer rounding only)
//   kRndNone : mu = 23        (plain binary32; fused multiply-add when allowed)
enum RoundClass { kRndFast = 0, kRndExact = 1, kRndNone = 2 };

struct Problem {
  int B, H, n_q, n_k, d;
  int causal;
  int mu;
  float tau;
  float scale;
  int variant;
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  uint16_t* out;
  uint32_t* mask_out;
  const uint32_t* mask_in;
  float* out_f32;
  float* ps_out;
  float* mixed_out;
  float* lse_out;
  unsigned long long* nsel_out;
  int* status_out;       // optional device status word (LAMP_ERR_TIMEOUT on a bounded wait that gave up)
  int debug_stall;       // LAMP_DEBUG_STALL_PRODUCERS: the whole-row producers hand over nothing (failure-path tests)
  int emax_sum_limit;  // largest e_q + e_k for which the fast score path is exact
};

// Workspace layout (bytes from the base, all 256-byte aligned).
struct Workspace {
  size_t counters;     // uint32 work counters [4]
  size_t stats;        // int32 [B*H][nchunk][4]
  size_t total;
  int nchunk;
  int use_ws;          // 1: warp-specialised whole-row kernel (two 16-row buffers fit on chip)
  int use_stream;      // 1: streamed kernel (rows too long for use_ws; strict rows in two passes)
  int use_decode;      // 1: split-key decode kernels (few query rows, long rows)
  int slab_too_large;  // 1: strict rows whose two-pass score slab would pass kStrictSlabCap
  size_t st_slab;      // strict rows on the streamed kernel: low-precision score slab [B*H][n_q][ld] f32
  size_t st_slab_bytes;
  size_t st_rows;      // ... and per-row statistics (maximum, first argmax, S_rest), 16 bytes each
  int dec_chunks;      // decode: 512-key chunks per row
  size_t dec_scores;   // decode: fp32 low-precision scores [B*H][n_q][dec_chunks * 512]
  size_t dec_stat;     // decode: per (row, chunk) maximum, first argmax, S_rest (16 bytes)
  size_t dec_part;     // decode: per (row, chunk) softmax maximum, normaliser, partial output [2 + d] f32
  size_t dec_flag;     // decode: per (b, h, chunk) int, the chunk's products are exact
  size_t dec_done;     // decode: per row, chunks whose partials are written (the last one combines)
};

// Warp-specialised kernels: 8 producer warps, 8 consumer warps and a warpgroup
// whose first warp drives the tensor core (MMA and TMA issue), 5 warpgroups.
constexpr int kWsThreads = 640;
// Registers per thread after setmaxnreg, per warpgroup role. The block launches
// with kWsLaunchRegs (65536 / 640 rounded down to a multiple of 8); the split
// must not need more than that pool: 256 P + 256 C + 128 M <= 640 * 96.
constexpr int kWsLaunchRegs = 96;
constexpr int kWsProdRegs = 112, kWsConsRegs = 96, kWsMmaRegs = 64;
static_assert(256 * kWsProdRegs + 256 * kWsConsRegs + 128 * kWsMmaRegs <= kWsThreads * kWsLaunchRegs,
              "register split above the launch pool");
// setmaxnreg.inc may only raise a warp's count and .dec only lower it (a lower
// .inc target is an illegal instruction); every budget is a multiple of 8 in [24, 256].
static_assert(kWsProdRegs >= kWsLaunchRegs && kWsConsRegs >= kWsLaunchRegs && kWsMmaRegs <= kWsLaunchRegs,
              "setmaxnreg.inc below, or .dec above, the launch count");
static_assert(kWsProdRegs % 8 == 0 && kWsConsRegs % 8 == 0 && kWsMmaRegs % 8 == 0 && kWsMmaRegs >= 24 &&
                  kWsProdRegs <= 256 && kWsConsRegs <= 256,
              "setmaxnreg counts are multiples of 8 in [24, 256]");
// Bytes of the opt-in shared memory left for the kernels' static __shared__ data.
constexpr size_t kStaticSmemReserve = 256;

Workspace plan_workspace(const Problem& p, int num_sms, size_t smem_optin);
// Tensor map of a [bh][n][d] bf16 tensor (row-major, this GPU's memory) for TMA
// boxes of box_x dimensions x box_y rows of one (b, h); rows past n read as zero.
// swizzle: 0, 32 or 128 (bytes of the shared-memory swizzle pattern).
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int d, int n, int bh, int box_x, int box_y,
                           int swizzle);
cudaError_t launch_prep(const Problem& p, const Workspace& ws, char* base, cudaStream_t st);
cudaError_t launch_ws(const Problem& p, const Workspace& ws, char* base, int num_sms, cudaStream_t st);
bool ws_fits(int d, int n_k, size_t smem_optin);
cudaError_t launch_stream(const Problem& p, const Workspace& ws, char* base, int num_sms, cudaStream_t st);
cudaError_t launch_decode(const Problem& p, const Workspace& ws, char* base, cudaStream_t st);
constexpr int kDecodeMaxQ = 4;       // query rows per (b, h) the decode kernels take
constexpr int kDecodeMinKeys = 512;  // shortest rows routed to them
constexpr int kDecodeChunk = 512;    // keys per chunk (one CTA)
constexpr size_t kStrictSlabCap = (size_t)LAMP_MAX_SCORE_SLAB_BYTES;  // largest two-pass strict score slab
size_t stream_smem_bytes(int d);
size_t stream_slab_ld(int n_k);  // slab row stride: keys rounded up to whole 512-key tiles
cudaError_t launch_ps_round(const float* x, float* y, size_t n, int mu, int path, cudaStream_t st);

// LAMP GELU(scale * x W^T): x [M, K], W [N, K] bf16, out [M, N].
struct GeluProblem {
  int M, N, K;
  int mu;
  float tau;
  float scale;
  int variant;  // LAMP_STRICT (the kappa test) or LAMP_GIVEN_MASK
  const uint16_t* x;
  const uint16_t* W;
  uint16_t* out;
  uint32_t* mask_out;
  const uint32_t* mask_in;
  float* out_f32;
  float* ps_out;
  float* mixed_out;
  unsigned long long* nsel_out;
  int emax_sum_limit;  // largest e_x + e_w for which the two-instruction rounding is exact
};
cudaError_t launch_gelu(const GeluProblem& p, cudaStream_t st);
// The PS(mu) linear map alone: fl32(scale * x W^T) written to p.ps_out [M, N].
cudaError_t launch_linear_ps(const GeluProblem& p, cudaStream_t st);
int gelu_max_rows();

// LAMP LayerNorm((y_hat -> greedy recompute) of scale * x W^T), per row, after
// launch_linear_ps has written y_hat.
struct LnProblem {
  int M, N, K;
  float tau;
  float scale;
  float eps;
  int variant;  // LAMP_STRICT (the greedy selection) or LAMP_GIVEN_MASK
  const uint16_t* x;
  const uint16_t* W;
  const float* yhat;  // [M, N], written by launch_linear_ps
  uint16_t* out;
  uint32_t* mask_out;
  const uint32_t* mask_in;
  float* out_f32;
  float* ps_out;      // the caller's copy of y_hat, when it is not yhat itself
  float* mixed_out;
  unsigned long long* nsel_out;
};
cudaError_t launch_ln_rows(const LnProblem& p, cudaStream_t st);
constexpr int kLnMaxN = 8192;

}  // namespace lamp
