/*
 * lamp.h -- C ABI of the B200 (sm_100a) LAMP attention library (liblamp.so).
 *
 * LAMP = look-ahead mixed-precision inference ("LAMP: Look-Ahead Mixed-Precision
 * Inference of Large Language Models", technical summary on gist.science,
 * paper 2601.21623). The library computes attention in which every key-query
 * product is first accumulated in a simulated low-precision float PS(mu), a
 * look-ahead test picks the few products whose rounding error the softmax would
 * amplify most, only those are recomputed in FP32, and softmax and P.V follow:
 *   - section "Implementation strategy", steps 1-3: low-precision baseline of g,
 *     look-ahead selection from that baseline, recompute of the selection in
 *     higher precision before f;
 *   - section "Theoretical basis", item 3 (softmax bullet): the strict test
 *     2 z_j (1 - z_j) |y_j| > tau, z the softmax probabilities of the row;
 *   - section "Experimental results": PS(mu) (mu mantissa bits), the relaxed
 *     relative-threshold variant that needs no normalising constant and so fits
 *     a one-pass softmax, and the random-selection control.
 * The same look-ahead scheme serves the two other operators of "Theoretical
 * basis", item 3, each after a PS(mu) linear map y = scale * x W^T:
 * lamp_linear_gelu (an activation: a diagonal Jacobian, a per-output condition
 * number) and lamp_linear_layernorm (greedy recompute by sorted magnitude);
 * their conventions are given with them below.
 *
 * Conventions for every entry point (the operator calls state their own shapes):
 *   - All tensor pointers are DEVICE pointers owned by the caller. Q is
 *     [B, H, n_q, d], K and V are [B, H, n_k, d], out is [B, H, n_q, d]; all
 *     contiguous row-major bfloat16 given as raw 16-bit patterns, 16-byte aligned.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream). Outputs
 *     are valid once the stream has reached the end of the call.
 *   - Between calls the library keeps only per-device attributes and a scratch
 *     memory pool. It never traps on the device; errors are return codes
 *     (below), with a message from lamp_last_error().
 *   - Arguments are checked on the host before anything is launched; a rejected
 *     call launches nothing and writes nothing.
 *   - Key j is valid for query row i when causal == 0, or when
 *     j <= i + (n_k - n_q) (bottom-right aligned causal mask). A row with no
 *     valid key produces out = 0, lse = -inf and no mask bits.
 *
 * Numerical contract (fixed by this library's reading of the pages, which give
 * no kernel; see the oracle tests for the pins):
 *   - PS(mu), mu in [1, 23]: binary32 exponent range and subnormals, mu explicit
 *     fraction bits, round to nearest with ties to even. Score accumulation:
 *     acc = +0; for k = 0..d-1: acc = round_PS(fl32(acc + fl32(q_k * k_k)));
 *     y_hat = fl32(scale * acc). mu = 23 is plain binary32.
 *   - FP32 recompute: the same sequential binary32 sum without rounding, then
 *     the same scaling.
 *   - Strict (variant 0): the criterion c_j = 2 z_j (1 - z_j) |y_hat_j| over the
 *     valid keys of the row, with z = softmax(y_hat); select when c_j > tau.
 *   - Relaxed (variant 1): c_j = 2 exp(y_hat_j - M_t) |y_hat_j|, M_t the running
 *     maximum of y_hat over 64-key tiles counted from key 0 up to and including
 *     the tile of key j; select when c_j > tau. It selects a superset of strict.
 *   - Given mask (variant 2): select exactly the bits of mask_in (the random
 *     control of the experiments).
 *   - Mixed row y_j = FP32 value if selected, else y_hat_j; then P = softmax(y)
 *     and out = P.V with fp32 accumulation, stored as bf16 (round to nearest even).
 *   - The selection of an entry whose criterion lies within about 1e-6 relative
 *     of tau may differ from an exact double-precision evaluation; everything
 *     else in the scores and the mask is bit-exact with the definition above.
 */
#ifndef LAMP_H
#define LAMP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point is exported from liblamp.so with default visibility. */
#if defined(__GNUC__)
#define LAMP_API __attribute__((visibility("default")))
#else
#define LAMP_API
#endif

/* Same handle as cudaStream_t; declared here so that this header needs no CUDA headers. */
typedef struct CUstream_st *lamp_stream_t;

enum lamp_variant { LAMP_STRICT = 0, LAMP_RELAXED = 1, LAMP_GIVEN_MASK = 2 };

enum lamp_status {
  LAMP_OK = 0,
  LAMP_ERR_ARG = -1,          /* null required pointer, mu outside [1,23], tau NaN,
                                 unknown variant, a dimension <= 0, scale <= 0 or NaN */
  LAMP_ERR_UNSUPPORTED = -2,  /* d not in {64, 128}; pointer not 16-byte aligned;
                                 a strict problem whose score slab would pass
                                 LAMP_MAX_SCORE_SLAB_BYTES; B * H > 65535 */
  LAMP_ERR_WORKSPACE = -3,    /* workspace given but smaller than lamp_workspace_size() */
  LAMP_ERR_CUDA = -4,         /* a CUDA call failed (allocation, launch); see lamp_last_error() */
  LAMP_ERR_TIMEOUT = -5,      /* written to status_out by a kernel whose bounded wait gave up */
  LAMP_ERR_CHECK = -6         /* reserved: a device-side check failed (reported via status_out) */
};

/* Largest score slab of a strict call. Whole rows of up to 1024 keys (d = 64;
 * 896 at d = 128) stay in shared memory, relaxed and given-mask rows of any
 * length stream through 512-key tiles, and decode rows (n_q <= 4) split their
 * keys. Strict rows longer than that take two streamed passes over a score slab
 * of B*H*n_q*ceil(n_k/512)*512*4 bytes in the workspace; a problem whose slab
 * would be larger than this is LAMP_ERR_UNSUPPORTED (lamp_workspace_size
 * returns 0 for it). */
#define LAMP_MAX_SCORE_SLAB_BYTES (64ull << 30)

typedef struct {
  int B, H, n_q, n_k, d;
} lamp_dims;

/*
 * lamp_attention -- LAMP attention, basic form.
 *   dims      shapes (see conventions); d must be 64 or 128.
 *   Q, K, V   bf16 inputs; out bf16 [B, H, n_q, d].
 *   mask_out  nullable. uint32 words [B, H, n_q, ceil(n_k/32)]: bit (j % 32) of
 *             word j / 32 is 1 when score j of the row was recomputed in FP32.
 *             Bits of invalid keys and of the padding past n_k are 0.
 *   mu        PS(mu) mantissa bits, 1..23.
 *   tau       selection threshold (strict and relaxed); tau < 0 recomputes every
 *             valid score; tau = +inf recomputes none. Ignored for variant 2.
 *   variant   LAMP_STRICT or LAMP_RELAXED (LAMP_GIVEN_MASK needs lamp_attention_ex).
 *   causal    0 or 1.
 * Scratch memory comes from a stream-ordered memory pool that the library creates
 * for each device on first use and keeps (with the memory it has grown to) until
 * the process exits; it is returned to that pool when the call completes on the
 * stream. Returns LAMP_OK or a negative lamp_status.
 */
LAMP_API int lamp_attention(const lamp_dims *dims, const void *Q, const void *K, const void *V,
                   void *out, uint32_t *mask_out, int mu, float tau, int variant,
                   int causal, lamp_stream_t stream);

/* Extended call. Every field after `stream` is optional (NULL / 0 = off). */
typedef struct {
  lamp_dims dims;
  const void *Q, *K, *V;
  void *out;
  uint32_t *mask_out;
  int mu;
  float tau;
  int variant;
  int causal;
  lamp_stream_t stream;
  float scale;                 /* score scale; 0 = fl32(1/sqrt(d)) */
  const uint32_t *mask_in;     /* LAMP_GIVEN_MASK: words in the mask_out layout; bits of
                                  invalid keys are ignored */
  float *out_f32;              /* fp32 copy of out [B, H, n_q, d] before bf16 rounding */
  float *ps_scores_out;        /* fp32 [B, H, n_q, n_k]: y_hat (invalid keys: -inf) */
  float *mixed_scores_out;     /* fp32 [B, H, n_q, n_k]: y after recompute (invalid: -inf) */
  float *lse_out;              /* fp32 [B, H, n_q]: log-sum-exp of the mixed row */
  unsigned long long *n_selected_out; /* device word: set to the number of recomputed
                                         scores of this call */
  void *workspace;             /* device scratch; NULL = the library's per-device pool */
  size_t workspace_bytes;
  int *status_out;             /* device status word, may be NULL: set to LAMP_ERR_TIMEOUT when
                                  a bounded wait inside a kernel gave up (the outputs of the
                                  call are then undefined); never cleared by the library */
  int debug_stall;             /* 0 in normal use. LAMP_DEBUG_STALL_PRODUCERS (tests of the
                                  failure path only): in the whole-row kernel the score
                                  producers hand over nothing, so every other warp's bounded
                                  wait (about 2 s) runs out; the kernel then writes
                                  LAMP_ERR_TIMEOUT to status_out and returns, its outputs
                                  undefined. Other kernels ignore the field. */
} lamp_args;

#define LAMP_DEBUG_STALL_PRODUCERS 1

LAMP_API int lamp_attention_ex(const lamp_args *args);

/*
 * lamp_attention_noalloc -- lamp_attention_ex for callers that must not allocate
 * device memory: a program that has handed the device's memory to an allocator
 * of its own, or one that may allocate only at start-up and not on the path that
 * computes attention. (The LAMP pages have no counterpart of this entry point; it
 * is part of this library's interface only.)
 *   args       as for lamp_attention_ex, except that workspace must be NULL and
 *              workspace_bytes 0 (LAMP_ERR_ARG otherwise).
 *   scratch    a fixed array of LAMP_NOALLOC_SCRATCH_BYTES in the memory of every
 *              GPU that loads the library, held until the process exits. A problem
 *              is rejected with LAMP_ERR_WORKSPACE before anything is launched when
 *              lamp_workspace_size() for it exceeds LAMP_NOALLOC_SCRATCH_BYTES; the
 *              usual causes are the score slab of strict rows longer than the
 *              whole-row kernel takes (B*H*n_q*ceil(n_k/512)*512*4 bytes) and the
 *              per-chunk partials of long decode rows.
 *   first call on a device: looks up the device address of that array (no
 *              allocation; a failed lookup is retried by the next call); make it
 *              before capturing a stream into a graph.
 *   sharing    every call on a device uses the same array, and keeps nothing in it
 *              from one call to the next (the call clears what must start at zero).
 *              Calls whose kernels overlap on the GPU (work on two streams without
 *              an ordering between them) race on the array: order them.
 * The call makes no cudaMalloc, cudaFree or other allocating CUDA call.
 */
#define LAMP_NOALLOC_SCRATCH_BYTES (4u << 20)
LAMP_API int lamp_attention_noalloc(const lamp_args *args);

/* Bytes of device scratch lamp_attention_ex needs for these shapes and variant
 * (0 when dims is NULL or invalid). The content need not be initialised. */
LAMP_API size_t lamp_workspace_size(const lamp_dims *dims, int variant);

/* Message for the last non-zero return on the calling thread ("" if none). */
LAMP_API const char *lamp_last_error(void);

/*
 * lamp_ps_round -- elementwise PS(mu) rounding of n binary32 values on the
 * device (the rounding the score kernels apply after every add). x and y are
 * device pointers to n floats (may alias). path: 0 = the exact integer
 * sequence, 1 = the two-instruction floating-point sequence the score kernels
 * use when the inputs' magnitude range allows it (valid for mu <= 10 and
 * |x| in {0} U [2^-126, 2^(127 - (23 - mu)))); outside that domain path 1
 * returns what the hardware sequence computes, which is what the tests check.
 */
LAMP_API int lamp_ps_round(const float *x, float *y, size_t n, int mu, int path, lamp_stream_t stream);

/* Library version string. */
LAMP_API const char *lamp_version(void);

/* sizeof(lamp_args) as compiled into the library, so that a binding can check
 * that its copy of the struct has the same layout. */
LAMP_API size_t lamp_args_size(void);

/*
 * lamp_linear_gelu -- LAMP on an elementwise activation: out = GELU(y) with
 * y = scale * x W^T computed in PS(mu), and the outputs whose component-wise
 * condition number kappa_j = |y_j f'(y_j) / f(y_j)| exceeds tau recomputed in
 * binary32 before the activation. LAMP summary (gist.science paper 2601.21623):
 * "Theoretical basis" item 3 (for an activation the Jacobian is diagonal, so the
 * sensitive components are found directly) and "Implementation strategy" steps
 * 1-3. f is GELU in its tanh form (GPT-2's activation),
 * f(y) = y/2 (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))), and
 * kappa(y) = |1 + y u'(y) (1 - tanh u)| (1 at y = 0; +inf for a non-finite y).
 *
 *   M, N, K     x is [M, K], W is [N, K] (a linear layer's weight layout), out
 *               [M, N]; all row-major. K must be a multiple of 8; M <= 4194240.
 *   x, W        bf16 bit patterns, device pointers, 16-byte aligned.
 *   out         bf16 [M, N] (2-byte aligned): f(y) rounded to nearest even.
 *   mask_out    nullable: uint32 words [M][ceil(N/32)], bit j % 32 of word j / 32
 *               set when output j of the row was recomputed; padding bits 0.
 *   mu, tau     PS(mu) fraction bits (1..23); kappa threshold (tau < 0 recomputes
 *               every output, +inf none; ignored for LAMP_GIVEN_MASK). NaN is
 *               LAMP_ERR_ARG.
 *   variant     LAMP_STRICT (the kappa test; an activation has no relaxed form,
 *               LAMP_RELAXED is LAMP_ERR_ARG) or LAMP_GIVEN_MASK (mask_in).
 *   scale       multiplies each finished sum once in binary32; 0 = 1.
 *   mask_in     LAMP_GIVEN_MASK: words in the mask_out layout (bits past N ignored).
 *   out_f32     nullable fp32 [M, N]: f(y) before the bf16 rounding.
 *   ps_out      nullable fp32 [M, N]: the PS(mu) outputs y_hat.
 *   mixed_out   nullable fp32 [M, N]: y after the recompute.
 *   n_selected_out  nullable device word: set to the number of recomputed outputs.
 * Every pointer is caller-owned device memory; the call is asynchronous on
 * stream, allocates nothing, and launches one or two kernels (plus a memset of
 * n_selected_out). Returns LAMP_OK, LAMP_ERR_ARG or LAMP_ERR_UNSUPPORTED
 * (K % 8 != 0, misaligned pointers, M too large) before launching anything, or
 * LAMP_ERR_CUDA when the launch fails.
 */
typedef struct {
  int M, N, K;
  const void *x, *W;
  void *out;
  uint32_t *mask_out;
  int mu;
  float tau;
  int variant;
  float scale;
  const uint32_t *mask_in;
  float *out_f32;
  float *ps_out;
  float *mixed_out;
  unsigned long long *n_selected_out;
  lamp_stream_t stream;
} lamp_gelu_args;

LAMP_API int lamp_linear_gelu(const lamp_gelu_args *args);

/* sizeof(lamp_gelu_args) as compiled into the library. */
LAMP_API size_t lamp_gelu_args_size(void);

/*
 * lamp_linear_layernorm -- LAMP on LayerNorm: out = LN(y) over each row of
 * y = scale * x W^T, with y computed in PS(mu) and, per row, the largest
 * magnitudes recomputed in binary32 until ||(1 - q) o y_hat||_2 / sigma_hat <= tau
 * (sigma_hat the low-precision row's sqrt(var + eps)). LAMP summary
 * (gist.science paper 2601.21623): "Theoretical basis" item 3 (layer
 * normalisation: a nearly sparsest set by sorting the input magnitudes) and
 * "Implementation strategy" steps 1-3. LN has no affine part:
 * LN(y)_j = (y_j - mean(y)) / sqrt(var(y) + eps), var the biased variance.
 *
 *   M, N, K, x, W, out, mask_out, mu, scale, mask_in, out_f32, ps_out,
 *   mixed_out, n_selected_out: as for lamp_linear_gelu; N <= 8192.
 *   tau         the bound on ||(1 - q) o y_hat||_2 / sigma_hat (tau < 0 recomputes
 *               every output, +inf none). Equal magnitudes are taken in
 *               ascending column order. NaN is LAMP_ERR_ARG.
 *   variant     LAMP_STRICT (the greedy selection) or LAMP_GIVEN_MASK.
 *   eps         LayerNorm's epsilon; 0 = 1e-5.
 *   workspace   device scratch for y_hat of lamp_ln_workspace_size(M, N) bytes,
 *               or NULL: then ps_out holds y_hat when given, else the library's
 *               per-device pool (as lamp_attention_ex) provides it.
 * Asynchronous on stream; the linear map (one or two kernels), then one warp per row.
 * Returns LAMP_OK, LAMP_ERR_ARG / LAMP_ERR_UNSUPPORTED / LAMP_ERR_WORKSPACE
 * before launching anything, or LAMP_ERR_CUDA.
 */
typedef struct {
  int M, N, K;
  const void *x, *W;
  void *out;
  uint32_t *mask_out;
  int mu;
  float tau;
  int variant;
  float scale;
  float eps;
  const uint32_t *mask_in;
  float *out_f32;
  float *ps_out;
  float *mixed_out;
  unsigned long long *n_selected_out;
  void *workspace;
  size_t workspace_bytes;
  lamp_stream_t stream;
} lamp_ln_args;

LAMP_API int lamp_linear_layernorm(const lamp_ln_args *args);

/* Bytes of scratch lamp_linear_layernorm needs when ps_out is NULL (M * N * 4). */
LAMP_API size_t lamp_ln_workspace_size(int M, int N);

/* sizeof(lamp_ln_args) as compiled into the library. */
LAMP_API size_t lamp_ln_args_size(void);

#ifdef __cplusplus
}
#endif

#endif /* LAMP_H */
