// C ABI of the LAMP attention library: argument checks, workspace planning and
// the launch sequence (preparation kernel, then the strict or relaxed kernel).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "lamp.h"
#include "lamp_kernels.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = '\0';
  return LAMP_OK;
}

struct DeviceInfo {
  int dev = 0;
  int num_sms = 0;
  size_t smem_optin = 0;
};

// Per-device attributes, queried once per device.
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];
cudaMemPool_t g_pool[kMaxDevices];  // scratch pool of each device; keeps its memory between calls
cudaError_t g_pool_err[kMaxDevices];
std::once_flag g_pool_once[kMaxDevices];

cudaError_t device_info(DeviceInfo& out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_dev_once[dev], [&]() {
    int sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      sms = optin = 0;
    g_dev[dev].dev = dev;
    g_dev[dev].num_sms = sms;
    g_dev[dev].smem_optin = (size_t)optin;
  });
  out = g_dev[dev];
  if (out.num_sms <= 0) return cudaErrorInvalidDevice;
  return cudaSuccess;
}

// The library's scratch pool of the current device (created on first use).
cudaError_t scratch_pool(int dev, cudaMemPool_t& pool) {
  std::call_once(g_pool_once[dev], [&]() {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pl = nullptr;
    cudaError_t pe = cudaMemPoolCreate(&pl, &props);
    if (pe == cudaSuccess) {
      uint64_t keep = ~0ull;  // never hand freed scratch back to the driver
      pe = cudaMemPoolSetAttribute(pl, cudaMemPoolAttrReleaseThreshold, &keep);
    }
    g_pool[dev] = pe == cudaSuccess ? pl : nullptr;
    g_pool_err[dev] = pe;
  });
  pool = g_pool[dev];
  return g_pool_err[dev];
}

bool aligned(const void* ptr, size_t a) { return ((uintptr_t)ptr % a) == 0; }

// Largest e_q + e_k (unbiased exponents of the largest |q| and |k| of a head)
// for which every partial sum x of every PS(mu) score stays below
// 2^(127 - s): |x| <= d * 2^(e_q + 1) * 2^(e_k + 1) * ((1 + 2^-24)(1 + 2^-(mu+1)))^d.
int emax_sum_limit(int mu, int d) {
  const int s = 23 - mu;
  const double growth = (double)d * std::log2((1.0 + std::ldexp(1.0, -24)) * (1.0 + std::ldexp(1.0, -(mu + 1))));
  const double lim = 127.0 - s - 2.0 - std::log2((double)d) - growth;
  return (int)std::floor(lim) - 1;
}

int check_args(const lamp_args* a) {
  if (!a) return fail(LAMP_ERR_ARG, "args is NULL");
  const lamp_dims& d = a->dims;
  if (d.B <= 0 || d.H <= 0 || d.n_q <= 0 || d.n_k <= 0 || d.d <= 0)
    return fail(LAMP_ERR_ARG, "dimensions must be positive (B=%d H=%d n_q=%d n_k=%d d=%d)", d.B, d.H,
                d.n_q, d.n_k, d.d);
  if (!a->Q || !a->K || !a->V || !a->out) return fail(LAMP_ERR_ARG, "Q, K, V and out must be non-NULL");
  if (a->mu < 1 || a->mu > 23) return fail(LAMP_ERR_ARG, "mu must be in [1, 23] (got %d)", a->mu);
  if (a->variant < 0 || a->variant > 2) return fail(LAMP_ERR_ARG, "unknown variant %d", a->variant);
  if (a->variant != LAMP_GIVEN_MASK && std::isnan(a->tau)) return fail(LAMP_ERR_ARG, "tau is NaN");
  if (a->variant == LAMP_GIVEN_MASK && !a->mask_in)
    return fail(LAMP_ERR_ARG, "LAMP_GIVEN_MASK needs mask_in");
  if (a->causal != 0 && a->causal != 1) return fail(LAMP_ERR_ARG, "causal must be 0 or 1");
  if (std::isnan(a->scale) || a->scale < 0.f || std::isinf(a->scale))
    return fail(LAMP_ERR_ARG, "scale must be 0 (default) or a positive finite value");
  if (a->debug_stall != 0 && a->debug_stall != LAMP_DEBUG_STALL_PRODUCERS)
    return fail(LAMP_ERR_ARG, "debug_stall must be 0 or LAMP_DEBUG_STALL_PRODUCERS");
  if (d.d != 64 && d.d != 128) return fail(LAMP_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d.d);
  const long long rows = (long long)d.B * d.H * d.n_q;
  if ((long long)d.B * d.H > 65535 || rows > (1LL << 40))
    return fail(LAMP_ERR_UNSUPPORTED, "problem too large for the index space");
  if (!aligned(a->Q, 16) || !aligned(a->K, 16) || !aligned(a->V, 16) || !aligned(a->out, 16))
    return fail(LAMP_ERR_UNSUPPORTED, "Q, K, V and out must be 16-byte aligned");
  if ((a->mask_out && !aligned(a->mask_out, 4)) || (a->mask_in && !aligned(a->mask_in, 4)) ||
      (a->out_f32 && !aligned(a->out_f32, 8)) || (a->ps_scores_out && !aligned(a->ps_scores_out, 4)) ||
      (a->mixed_scores_out && !aligned(a->mixed_scores_out, 4)) || (a->lse_out && !aligned(a->lse_out, 4)) ||
      (a->n_selected_out && !aligned(a->n_selected_out, 8)) || (a->status_out && !aligned(a->status_out, 4)))
    return fail(LAMP_ERR_UNSUPPORTED, "optional outputs must be naturally aligned (out_f32: 8 bytes)");
  return LAMP_OK;
}

lamp::Problem make_problem(const lamp_args* a) {
  lamp::Problem p;
  p.B = a->dims.B; p.H = a->dims.H; p.n_q = a->dims.n_q; p.n_k = a->dims.n_k; p.d = a->dims.d;
  p.causal = a->causal;
  p.mu = a->mu;
  p.tau = a->tau;
  p.scale = a->scale > 0.f ? a->scale : (float)(1.0 / std::sqrt((double)a->dims.d));
  p.variant = a->variant;
  p.Q = static_cast<const uint16_t*>(a->Q);
  p.K = static_cast<const uint16_t*>(a->K);
  p.V = static_cast<const uint16_t*>(a->V);
  p.out = static_cast<uint16_t*>(a->out);
  p.mask_out = a->mask_out;
  p.mask_in = a->mask_in;
  p.out_f32 = a->out_f32;
  p.ps_out = a->ps_scores_out;
  p.mixed_out = a->mixed_scores_out;
  p.lse_out = a->lse_out;
  p.nsel_out = a->n_selected_out;
  p.status_out = a->status_out;
  p.debug_stall = a->debug_stall;
  p.emax_sum_limit = emax_sum_limit(a->mu, a->dims.d);
  return p;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The launch sequence of one call: exponent statistics, then the whole-row or
// the streamed kernel (or the two decode kernels on their own).
cudaError_t run_kernels(const lamp::Problem& p, const lamp::Workspace& ws, char* base, const DeviceInfo& info,
                        cudaStream_t st) {
  // the decode kernels fold their own exponent statistics and reset the count
  if (ws.use_decode) return lamp::launch_decode(p, ws, base, st);
  cudaError_t e = lamp::launch_prep(p, ws, base, st);
  if (e != cudaSuccess) return e;
  if (ws.use_ws) return lamp::launch_ws(p, ws, base, info.num_sms, st);
  return lamp::launch_stream(p, ws, base, info.num_sms, st);
}

// Scratch of lamp_attention_noalloc: one fixed array in the device memory of
// every GPU that loads the library, held until the process exits. In host code
// the name stands for a host-side shadow, not for a device address: kernels get
// the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LAMP_NOALLOC_SCRATCH_BYTES];
std::atomic<char*> g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on device dev (the current device). Only a
// successful lookup is kept: a failed one (for instance while another thread
// holds a stream capture open) is retried on the next call, and its error is
// cleared from the runtime's last-error state.
cudaError_t noalloc_scratch(int dev, char*& ptr) {
  ptr = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (ptr) return cudaSuccess;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ptr = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
  if (ptr) return cudaSuccess;
  void* addr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
  if (e != cudaSuccess || !addr) {
    (void)cudaGetLastError();
    return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
  }
  ptr = static_cast<char*>(addr);
  g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
  return cudaSuccess;
}

}  // namespace

namespace lamp {

Workspace plan_workspace(const Problem& p, int num_sms, size_t smem_optin) {
  Workspace w{};
  const int BH = p.B * p.H;
  int nchunk = (2 * num_sms + BH - 1) / BH;
  if (nchunk < 1) nchunk = 1;
  if (nchunk > 64) nchunk = 64;
  const int maxrows = p.n_q > p.n_k ? p.n_q : p.n_k;
  if (nchunk > maxrows) nchunk = maxrows;
  w.nchunk = nchunk;
  w.counters = 0;
  w.stats = 256;
  size_t off = align256(w.stats + (size_t)BH * nchunk * 16);
  // decode shapes (a few query rows per head, long rows): split over the keys
  if (p.n_q <= kDecodeMaxQ && p.n_k >= kDecodeMinKeys) {
    w.use_decode = 1;
    w.dec_chunks = (p.n_k + kDecodeChunk - 1) / kDecodeChunk;
    const size_t rows = (size_t)BH * p.n_q;
    w.dec_scores = off;
    off = align256(off + rows * w.dec_chunks * kDecodeChunk * 4);
    w.dec_stat = off;
    off = align256(off + rows * w.dec_chunks * 16);
    w.dec_part = off;
    off = align256(off + rows * w.dec_chunks * (2 + (size_t)p.d) * 4);
    w.dec_flag = off;
    off = align256(off + (size_t)BH * w.dec_chunks * 4);
    w.dec_done = off;
    off = align256(off + rows * 4);
    w.total = off;
    return w;
  }
  w.use_ws = ws_fits(p.d, p.n_k, smem_optin) ? 1 : 0;
  // rows too long for the whole-row kernel stream through 512-key tiles instead
  w.use_stream = (!w.use_ws && stream_smem_bytes(p.d) + kStaticSmemReserve <= smem_optin) ? 1 : 0;
  if (w.use_stream && p.variant == LAMP_STRICT) {
    // strict rows take two passes over a score slab in HBM (the strict test needs
    // the whole row's statistics before it selects anything)
    const size_t slab = (size_t)BH * p.n_q * stream_slab_ld(p.n_k) * 4;
    w.st_slab_bytes = slab;
    if (slab > kStrictSlabCap) {
      w.slab_too_large = 1;
    } else {
      w.st_slab = off;
      off = align256(off + slab);
      w.st_rows = off;
      off = align256(off + (size_t)BH * p.n_q * 16);
    }
  }
  w.total = off;
  return w;
}

}  // namespace lamp

// The plan's kernels must be able to serve the problem: a strict problem's
// two-pass score slab must stay within LAMP_MAX_SCORE_SLAB_BYTES, and the
// kernel's shared memory must fit the device.
int check_plan(const lamp::Problem& p, const lamp::Workspace& ws, const DeviceInfo& info) {
  (void)info;
  if (ws.slab_too_large)
    return fail(LAMP_ERR_UNSUPPORTED,
                "strict rows of %d keys need a two-pass score slab of %zu bytes, more than "
                "LAMP_MAX_SCORE_SLAB_BYTES (%llu)",
                p.n_k, ws.st_slab_bytes, (unsigned long long)LAMP_MAX_SCORE_SLAB_BYTES);
  if (!ws.use_decode && !ws.use_ws && !ws.use_stream)
    return fail(LAMP_ERR_UNSUPPORTED, "device shared memory too small for the attention kernels");
  return LAMP_OK;
}

extern "C" {

const char* lamp_last_error(void) { return g_err; }

const char* lamp_version(void) { return "lamp-b200 0.1 (sm_100a)"; }

size_t lamp_args_size(void) { return sizeof(lamp_args); }

size_t lamp_workspace_size(const lamp_dims* dims, int variant) {
  if (!dims || dims->B <= 0 || dims->H <= 0 || dims->n_q <= 0 || dims->n_k <= 0 ||
      (dims->d != 64 && dims->d != 128) || variant < 0 || variant > 2)
    return 0;
  DeviceInfo info;
  if (device_info(info) != cudaSuccess) return 0;
  lamp::Problem p{};
  p.B = dims->B; p.H = dims->H; p.n_q = dims->n_q; p.n_k = dims->n_k; p.d = dims->d;
  p.variant = variant;
  const lamp::Workspace w = lamp::plan_workspace(p, info.num_sms, info.smem_optin);
  if (w.slab_too_large || (!w.use_decode && !w.use_ws && !w.use_stream)) return 0;
  return w.total;
}

int lamp_attention_ex(const lamp_args* a) {
  int rc = check_args(a);
  if (rc != LAMP_OK) return rc;
  DeviceInfo info;
  cudaError_t e = device_info(info);
  if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "no usable CUDA device: %s", cudaGetErrorString(e));
  lamp::Problem p = make_problem(a);
  lamp::Workspace ws = lamp::plan_workspace(p, info.num_sms, info.smem_optin);
  rc = check_plan(p, ws, info);
  if (rc != LAMP_OK) return rc;
  if (a->workspace && a->workspace_bytes < ws.total)
    return fail(LAMP_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu bytes needed",
                a->workspace_bytes, ws.total);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(a->stream);
  char* base = static_cast<char*>(a->workspace);
  bool owned = false;
  if (!base) {
    cudaMemPool_t pool = nullptr;
    e = scratch_pool(info.dev, pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&base), ws.total, pool, st);
    if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "workspace allocation failed: %s", cudaGetErrorString(e));
    owned = true;
  }
  e = run_kernels(p, ws, base, info, st);
  if (owned) {
    cudaError_t fe = cudaFreeAsync(base, st);
    if (e == cudaSuccess) e = fe;
  }
  if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return ok();
}

int lamp_attention_noalloc(const lamp_args* a) {
  int rc = check_args(a);
  if (rc != LAMP_OK) return rc;
  if (a->workspace || a->workspace_bytes)
    return fail(LAMP_ERR_ARG, "lamp_attention_noalloc uses its own scratch: workspace must be NULL and 0");
  DeviceInfo info;
  cudaError_t e = device_info(info);
  if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "no usable CUDA device: %s", cudaGetErrorString(e));
  lamp::Problem p = make_problem(a);
  lamp::Workspace ws = lamp::plan_workspace(p, info.num_sms, info.smem_optin);
  rc = check_plan(p, ws, info);
  if (rc != LAMP_OK) return rc;
  if (ws.total > (size_t)LAMP_NOALLOC_SCRATCH_BYTES)
    return fail(LAMP_ERR_WORKSPACE,
                "this problem needs %zu bytes of scratch, more than the %u bytes lamp_attention_noalloc "
                "holds; use lamp_attention_ex",
                ws.total, (unsigned)LAMP_NOALLOC_SCRATCH_BYTES);
  char* base = nullptr;
  e = noalloc_scratch(info.dev, base);
  if (e != cudaSuccess || !base)
    return fail(LAMP_ERR_CUDA, "scratch array address unavailable: %s", cudaGetErrorString(e));
  e = run_kernels(p, ws, base, info, reinterpret_cast<cudaStream_t>(a->stream));
  if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return ok();
}

int lamp_attention(const lamp_dims* dims, const void* Q, const void* K, const void* V, void* out,
                   uint32_t* mask_out, int mu, float tau, int variant, int causal, lamp_stream_t stream) {
  if (!dims) return fail(LAMP_ERR_ARG, "dims is NULL");
  if (variant == LAMP_GIVEN_MASK) return fail(LAMP_ERR_ARG, "LAMP_GIVEN_MASK needs lamp_attention_ex (mask_in)");
  lamp_args a;
  std::memset(&a, 0, sizeof(a));
  a.dims = *dims;
  a.Q = Q; a.K = K; a.V = V; a.out = out; a.mask_out = mask_out;
  a.mu = mu; a.tau = tau; a.variant = variant; a.causal = causal; a.stream = stream;
  return lamp_attention_ex(&a);
}

size_t lamp_gelu_args_size(void) { return sizeof(lamp_gelu_args); }

int lamp_linear_gelu(const lamp_gelu_args* a) {
  if (!a) return fail(LAMP_ERR_ARG, "args is NULL");
  if (a->M <= 0 || a->N <= 0 || a->K <= 0)
    return fail(LAMP_ERR_ARG, "dimensions must be positive (M=%d N=%d K=%d)", a->M, a->N, a->K);
  if (!a->x || !a->W || !a->out) return fail(LAMP_ERR_ARG, "x, W and out must be non-NULL");
  if (a->mu < 1 || a->mu > 23) return fail(LAMP_ERR_ARG, "mu must be in [1, 23] (got %d)", a->mu);
  if (a->variant == LAMP_RELAXED)
    return fail(LAMP_ERR_ARG, "an activation's kappa test is exact per output; there is no relaxed variant");
  if (a->variant != LAMP_STRICT && a->variant != LAMP_GIVEN_MASK)
    return fail(LAMP_ERR_ARG, "unknown variant %d", a->variant);
  if (a->variant == LAMP_STRICT && std::isnan(a->tau)) return fail(LAMP_ERR_ARG, "tau is NaN");
  if (a->variant == LAMP_GIVEN_MASK && !a->mask_in) return fail(LAMP_ERR_ARG, "LAMP_GIVEN_MASK needs mask_in");
  if (std::isnan(a->scale) || a->scale < 0.f || std::isinf(a->scale))
    return fail(LAMP_ERR_ARG, "scale must be 0 (default 1) or a positive finite value");
  if (a->K % 8) return fail(LAMP_ERR_UNSUPPORTED, "K must be a multiple of 8 (got %d)", a->K);
  if (a->M > lamp::gelu_max_rows()) return fail(LAMP_ERR_UNSUPPORTED, "M must be at most %d", lamp::gelu_max_rows());
  if (!aligned(a->x, 16) || !aligned(a->W, 16)) return fail(LAMP_ERR_UNSUPPORTED, "x and W must be 16-byte aligned");
  if (!aligned(a->out, 2) || (a->mask_out && !aligned(a->mask_out, 4)) || (a->mask_in && !aligned(a->mask_in, 4)) ||
      (a->out_f32 && !aligned(a->out_f32, 4)) || (a->ps_out && !aligned(a->ps_out, 4)) ||
      (a->mixed_out && !aligned(a->mixed_out, 4)) || (a->n_selected_out && !aligned(a->n_selected_out, 8)))
    return fail(LAMP_ERR_UNSUPPORTED, "outputs must be naturally aligned");
  lamp::GeluProblem g;
  g.M = a->M; g.N = a->N; g.K = a->K;
  g.mu = a->mu;
  g.tau = a->variant == LAMP_GIVEN_MASK ? 0.f : a->tau;
  g.scale = a->scale == 0.f ? 1.f : a->scale;
  g.variant = a->variant;
  g.x = static_cast<const uint16_t*>(a->x);
  g.W = static_cast<const uint16_t*>(a->W);
  g.out = static_cast<uint16_t*>(a->out);
  g.mask_out = a->mask_out;
  g.mask_in = a->mask_in;
  g.out_f32 = a->out_f32;
  g.ps_out = a->ps_out;
  g.mixed_out = a->mixed_out;
  g.nsel_out = a->n_selected_out;
  g.emax_sum_limit = emax_sum_limit(a->mu, a->K);
  cudaError_t e = lamp::launch_gelu(g, reinterpret_cast<cudaStream_t>(a->stream));
  if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return ok();
}

size_t lamp_ln_args_size(void) { return sizeof(lamp_ln_args); }

size_t lamp_ln_workspace_size(int M, int N) { return (M > 0 && N > 0) ? (size_t)M * (size_t)N * 4 : 0; }

int lamp_linear_layernorm(const lamp_ln_args* a) {
  if (!a) return fail(LAMP_ERR_ARG, "args is NULL");
  if (a->M <= 0 || a->N <= 0 || a->K <= 0)
    return fail(LAMP_ERR_ARG, "dimensions must be positive (M=%d N=%d K=%d)", a->M, a->N, a->K);
  if (!a->x || !a->W || !a->out) return fail(LAMP_ERR_ARG, "x, W and out must be non-NULL");
  if (a->mu < 1 || a->mu > 23) return fail(LAMP_ERR_ARG, "mu must be in [1, 23] (got %d)", a->mu);
  if (a->variant == LAMP_RELAXED) return fail(LAMP_ERR_ARG, "LayerNorm's selection has no relaxed variant");
  if (a->variant != LAMP_STRICT && a->variant != LAMP_GIVEN_MASK)
    return fail(LAMP_ERR_ARG, "unknown variant %d", a->variant);
  if (a->variant == LAMP_STRICT && std::isnan(a->tau)) return fail(LAMP_ERR_ARG, "tau is NaN");
  if (a->variant == LAMP_GIVEN_MASK && !a->mask_in) return fail(LAMP_ERR_ARG, "LAMP_GIVEN_MASK needs mask_in");
  if (std::isnan(a->scale) || a->scale < 0.f || std::isinf(a->scale))
    return fail(LAMP_ERR_ARG, "scale must be 0 (default 1) or a positive finite value");
  if (std::isnan(a->eps) || a->eps < 0.f || std::isinf(a->eps))
    return fail(LAMP_ERR_ARG, "eps must be 0 (default 1e-5) or a positive finite value");
  if (a->K % 8) return fail(LAMP_ERR_UNSUPPORTED, "K must be a multiple of 8 (got %d)", a->K);
  if (a->N > lamp::kLnMaxN) return fail(LAMP_ERR_UNSUPPORTED, "N must be at most %d", lamp::kLnMaxN);
  if (a->M > lamp::gelu_max_rows()) return fail(LAMP_ERR_UNSUPPORTED, "M must be at most %d", lamp::gelu_max_rows());
  if (!aligned(a->x, 16) || !aligned(a->W, 16)) return fail(LAMP_ERR_UNSUPPORTED, "x and W must be 16-byte aligned");
  if (!aligned(a->out, 2) || (a->mask_out && !aligned(a->mask_out, 4)) || (a->mask_in && !aligned(a->mask_in, 4)) ||
      (a->out_f32 && !aligned(a->out_f32, 4)) || (a->ps_out && !aligned(a->ps_out, 4)) ||
      (a->mixed_out && !aligned(a->mixed_out, 4)) || (a->n_selected_out && !aligned(a->n_selected_out, 8)) ||
      (a->workspace && !aligned(a->workspace, 4)))
    return fail(LAMP_ERR_UNSUPPORTED, "outputs and workspace must be naturally aligned");
  const size_t need = lamp_ln_workspace_size(a->M, a->N);
  if (a->workspace && a->workspace_bytes < need)
    return fail(LAMP_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu bytes needed", a->workspace_bytes,
                need);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(a->stream);
  float* yhat = a->ps_out ? a->ps_out : static_cast<float*>(a->workspace);
  bool owned = false;
  if (!yhat) {
    DeviceInfo info;
    cudaError_t e = device_info(info);
    if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "no usable CUDA device: %s", cudaGetErrorString(e));
    cudaMemPool_t pool = nullptr;
    e = scratch_pool(info.dev, pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&yhat), need, pool, st);
    if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "workspace allocation failed: %s", cudaGetErrorString(e));
    owned = true;
  }
  lamp::GeluProblem g{};
  g.M = a->M; g.N = a->N; g.K = a->K;
  g.mu = a->mu;
  g.scale = a->scale == 0.f ? 1.f : a->scale;
  g.variant = LAMP_STRICT;
  g.x = static_cast<const uint16_t*>(a->x);
  g.W = static_cast<const uint16_t*>(a->W);
  g.ps_out = yhat;
  g.emax_sum_limit = emax_sum_limit(a->mu, a->K);
  lamp::LnProblem l{};
  l.M = a->M; l.N = a->N; l.K = a->K;
  l.tau = a->variant == LAMP_GIVEN_MASK ? 0.f : a->tau;
  l.scale = g.scale;
  l.eps = a->eps == 0.f ? 1e-5f : a->eps;
  l.variant = a->variant;
  l.x = g.x; l.W = g.W;
  l.yhat = yhat;
  l.out = static_cast<uint16_t*>(a->out);
  l.mask_out = a->mask_out;
  l.mask_in = a->mask_in;
  l.out_f32 = a->out_f32;
  l.mixed_out = a->mixed_out;
  l.nsel_out = a->n_selected_out;
  cudaError_t e = cudaSuccess;
  if (a->n_selected_out) e = cudaMemsetAsync(a->n_selected_out, 0, sizeof(unsigned long long), st);
  if (e == cudaSuccess) e = lamp::launch_linear_ps(g, st);
  if (e == cudaSuccess) e = lamp::launch_ln_rows(l, st);
  if (owned) {
    cudaError_t fe = cudaFreeAsync(yhat, st);
    if (e == cudaSuccess) e = fe;
  }
  if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return ok();
}

int lamp_ps_round(const float* x, float* y, size_t n, int mu, int path, lamp_stream_t stream) {
  if ((!x || !y) && n) return fail(LAMP_ERR_ARG, "x and y must be non-NULL");
  if (mu < 1 || mu > 23) return fail(LAMP_ERR_ARG, "mu must be in [1, 23] (got %d)", mu);
  if (path != 0 && path != 1) return fail(LAMP_ERR_ARG, "path must be 0 or 1");
  cudaError_t e = lamp::launch_ps_round(x, y, n, mu, path, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(LAMP_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return ok();
}

}  // extern "C"
