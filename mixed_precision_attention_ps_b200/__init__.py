"""LAMP (look-ahead mixed-precision) attention for B200 (sm_100a).

The computation lives in liblamp.so (C ABI, include/lamp.h); this package is
its Python binding. ``attention()`` is a convenience wrapper that allocates the
outputs as torch tensors on the inputs' device and calls ``lamp_attention_ex``
on the current stream.

Method: "LAMP: Look-Ahead Mixed-Precision Inference of Large Language Models"
(technical summary, gist.science paper 2601.21623), sections "Implementation
strategy" (steps 1-3), "Theoretical basis" (item 3, softmax bullet) and
"Experimental results" (PS(mu), relaxed relative-threshold variant).
"""
from __future__ import annotations

from dataclasses import dataclass

from ._native import (LAMP_ERR_ARG, LAMP_ERR_CHECK, LAMP_ERR_CUDA, LAMP_ERR_TIMEOUT,  # noqa: F401
                      LAMP_DEBUG_STALL_PRODUCERS, LAMP_ERR_UNSUPPORTED, LAMP_ERR_WORKSPACE, LAMP_GIVEN_MASK, LAMP_MAX_SCORE_SLAB_BYTES,
                      LAMP_NOALLOC_SCRATCH_BYTES, LAMP_OK, LAMP_RELAXED, LAMP_STRICT, LampError, lamp_args,
                      lamp_args_size, lamp_attention, lamp_attention_ex, lamp_attention_noalloc, lamp_dims,
                      lamp_gelu_args, lamp_gelu_args_size, lamp_last_error, lamp_linear_gelu,
                      lamp_linear_layernorm, lamp_ln_args, lamp_ln_args_size, lamp_ln_workspace_size, lamp_ps_round,
                      lamp_version, lamp_workspace_size, load, make_args, make_gelu_args, make_ln_args)

__all__ = [
    "LAMP_STRICT", "LAMP_RELAXED", "LAMP_GIVEN_MASK", "LampError", "lamp_attention", "lamp_attention_ex",
    "lamp_attention_noalloc",
    "lamp_workspace_size", "lamp_last_error", "lamp_ps_round", "lamp_version", "lamp_args_size",
    "attention", "LampOutputs", "load", "lamp_linear_gelu", "lamp_gelu_args_size", "linear_gelu", "GeluOutputs",
    "lamp_linear_layernorm", "lamp_ln_args_size", "lamp_ln_workspace_size", "linear_layernorm",
]


@dataclass
class LampOutputs:
    out: "object"
    mask: "object | None" = None
    out_f32: "object | None" = None
    ps_scores: "object | None" = None
    mixed_scores: "object | None" = None
    lse: "object | None" = None
    n_selected: "object | None" = None


def attention(Q, K, V, *, mu: int = 4, tau: float = 0.0, variant: int = LAMP_STRICT, causal: bool = True,
              scale: float = 0.0, mask_in=None, want_mask: bool = True, want_out_f32: bool = False,
              want_scores: bool = False, want_lse: bool = False, want_count: bool = False,
              stream=None) -> LampOutputs:
    """LAMP attention on torch tensors.

    Q: [B, H, n_q, d], K and V: [B, H, n_k, d], all torch.bfloat16, contiguous,
    on one CUDA device. Returns the bf16 output and the requested extras
    (mask words int32 [B, H, n_q, ceil(n_k/32)], scores fp32 [B, H, n_q, n_k],
    lse fp32 [B, H, n_q], selected count int64 [1]).
    """
    import torch

    B, H, n_q, d = Q.shape
    n_k = K.shape[2]
    dev = Q.device
    for t in (Q, K, V):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != dev:
            raise ValueError("Q, K, V must be contiguous bfloat16 tensors on one device")
    nwords = (n_k + 31) // 32
    res = LampOutputs(out=torch.empty((B, H, n_q, d), dtype=torch.bfloat16, device=dev))
    if want_mask:
        res.mask = torch.empty((B, H, n_q, nwords), dtype=torch.int32, device=dev)
    if want_out_f32:
        res.out_f32 = torch.empty((B, H, n_q, d), dtype=torch.float32, device=dev)
    if want_scores:
        res.ps_scores = torch.empty((B, H, n_q, n_k), dtype=torch.float32, device=dev)
        res.mixed_scores = torch.empty((B, H, n_q, n_k), dtype=torch.float32, device=dev)
    if want_lse:
        res.lse = torch.empty((B, H, n_q), dtype=torch.float32, device=dev)
    if want_count:
        res.n_selected = torch.empty(1, dtype=torch.int64, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    lamp_attention_ex(dims=(B, H, n_q, n_k, d), Q=Q, K=K, V=V, out=res.out, mask_out=res.mask, mu=mu,
                      tau=tau, variant=variant, causal=int(bool(causal)), stream=stream, scale=scale,
                      mask_in=mask_in, out_f32=res.out_f32, ps_scores_out=res.ps_scores,
                      mixed_scores_out=res.mixed_scores, lse_out=res.lse, n_selected_out=res.n_selected)
    return res


@dataclass
class GeluOutputs:
    out: "object"
    mask: "object | None" = None
    out_f32: "object | None" = None
    ps: "object | None" = None
    mixed: "object | None" = None
    n_selected: "object | None" = None


def linear_gelu(x, W, *, mu: int = 4, tau: float = 0.0, variant: int = LAMP_STRICT, scale: float = 0.0,
                mask_in=None, want_mask: bool = True, want_out_f32: bool = False, want_scores: bool = False,
                want_count: bool = False, stream=None) -> GeluOutputs:
    """LAMP GELU(scale * x W^T) on torch tensors ("Theoretical basis", item 3:
    an activation's diagonal Jacobian).

    x: [M, K], W: [N, K] (a linear layer's weight), both torch.bfloat16,
    contiguous, on one CUDA device, K a multiple of 8. Returns the bf16 output
    [M, N] and the requested extras (mask words int32 [M, ceil(N/32)], the PS(mu)
    and mixed pre-activations fp32 [M, N], selected count int64 [1]).
    """
    import torch

    M, K = x.shape
    N = W.shape[0]
    dev = x.device
    for t in (x, W):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != dev:
            raise ValueError("x and W must be contiguous bfloat16 tensors on one device")
    if W.shape[1] != K:
        raise ValueError("x and W disagree on K")
    res = GeluOutputs(out=torch.empty((M, N), dtype=torch.bfloat16, device=dev))
    if want_mask:
        res.mask = torch.empty((M, (N + 31) // 32), dtype=torch.int32, device=dev)
    if want_out_f32:
        res.out_f32 = torch.empty((M, N), dtype=torch.float32, device=dev)
    if want_scores:
        res.ps = torch.empty((M, N), dtype=torch.float32, device=dev)
        res.mixed = torch.empty((M, N), dtype=torch.float32, device=dev)
    if want_count:
        res.n_selected = torch.empty(1, dtype=torch.int64, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    lamp_linear_gelu(M=M, N=N, K=K, x=x, W=W, out=res.out, mask_out=res.mask, mu=mu, tau=tau, variant=variant,
                     scale=scale, mask_in=mask_in, out_f32=res.out_f32, ps_out=res.ps, mixed_out=res.mixed,
                     n_selected_out=res.n_selected, stream=stream)
    return res


def linear_layernorm(x, W, *, mu: int = 4, tau: float = 0.0, variant: int = LAMP_STRICT, scale: float = 0.0,
                     eps: float = 0.0, mask_in=None, want_mask: bool = True, want_out_f32: bool = False,
                     want_scores: bool = False, want_count: bool = False, stream=None) -> GeluOutputs:
    """LAMP LayerNorm(scale * x W^T) on torch tensors ("Theoretical basis", item 3:
    layer normalisation, greedy by sorted magnitude). Shapes and extras as for
    linear_gelu; N <= 8192. y_hat goes to the returned ps tensor when want_scores,
    else to the library's scratch pool."""
    import torch

    M, K = x.shape
    N = W.shape[0]
    dev = x.device
    for t in (x, W):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device != dev:
            raise ValueError("x and W must be contiguous bfloat16 tensors on one device")
    if W.shape[1] != K:
        raise ValueError("x and W disagree on K")
    res = GeluOutputs(out=torch.empty((M, N), dtype=torch.bfloat16, device=dev))
    if want_mask:
        res.mask = torch.empty((M, (N + 31) // 32), dtype=torch.int32, device=dev)
    if want_out_f32:
        res.out_f32 = torch.empty((M, N), dtype=torch.float32, device=dev)
    if want_scores:
        res.ps = torch.empty((M, N), dtype=torch.float32, device=dev)
        res.mixed = torch.empty((M, N), dtype=torch.float32, device=dev)
    if want_count:
        res.n_selected = torch.empty(1, dtype=torch.int64, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    lamp_linear_layernorm(M=M, N=N, K=K, x=x, W=W, out=res.out, mask_out=res.mask, mu=mu, tau=tau,
                          variant=variant, scale=scale, eps=eps, mask_in=mask_in, out_f32=res.out_f32,
                          ps_out=res.ps, mixed_out=res.mixed, n_selected_out=res.n_selected, stream=stream)
    return res
