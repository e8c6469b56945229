"""Seeded synthetic inputs for LAMP attention.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It holds no LAMP arithmetic: it only turns (seed, stream, index)
counters into bf16 tensors and random key subsets. Both sides receive the same
bytes.

Generator (counter based, so any element can be produced on its own):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): the i-th output of a generator whose state starts
  at ``k`` is ``mix64(k + (i + 1) * GOLDEN)``.
* A stream ``s`` of seed ``seed`` starts at ``k = mix64(seed * GOLDEN + s + 1)``.
* Normal samples use Box-Muller in double on two 53-bit uniforms
  (outputs ``2n`` and ``2n+1`` of the stream for element ``n``), are optionally
  scaled, rounded to float32, then to bfloat16 (both round-to-nearest-even).

Streams: 0 = Q, 1 = K, 2 = V, 3 = outlier channel choice, 4 = random-control
subset keys, 5 = x and 6 = W of the activation workloads (GELU after a linear
map; x is [M, K], W is [N, K] like a linear layer's weight).

The workloads stand in for GPT-2 XL activations on OpenWebText (LAMP summary,
"Experimental results"), which are not available here: iid N(0,1) entries, and
for the peaked/outlier workload one head-dim channel in every (b, h) of Q and K
scaled by 20 before rounding to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_Q, STREAM_K, STREAM_V, STREAM_OUTLIER, STREAM_RANDOM = 0, 1, 2, 3, 4
STREAM_X, STREAM_W = 5, 6


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_start(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        k = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) * GOLDEN + np.uint64(stream + 1)
    return mix64(np.array([k], dtype=np.uint64))[0]


def stream_values(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """Outputs number ``index`` (uint64 array) of the given stream."""
    k = stream_start(seed, stream)
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(k + (idx + np.uint64(1)) * GOLDEN)


def _uniform53(r: np.ndarray) -> np.ndarray:
    return (r >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_f64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Elements ``start .. start+count-1`` of a N(0,1) stream, in double."""
    n = np.arange(start, start + count, dtype=np.uint64)
    u1 = _uniform53(stream_values(seed, stream, n * np.uint64(2)))
    u2 = _uniform53(stream_values(seed, stream, n * np.uint64(2) + np.uint64(1)))
    return np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * math.pi * u2)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """double -> float32 (RNE) -> bfloat16 (RNE), returned as uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic LAMP attention problem."""

    B: int
    H: int
    n_q: int
    n_k: int
    d: int
    causal: bool = True
    outlier_frac: float = 0.0   # fraction of head-dim channels of Q and K scaled up
    outlier_scale: float = 20.0
    seed: int = 0

    @property
    def n_outlier(self) -> int:
        return int(math.ceil(self.outlier_frac * self.d)) if self.outlier_frac > 0 else 0

    def valid_keys(self, i: int) -> int:
        """Number of valid keys of query row i (keys 0 .. n-1 are valid)."""
        if not self.causal:
            return self.n_k
        return max(0, min(self.n_k, i + 1 + (self.n_k - self.n_q)))

    def valid_scores(self) -> int:
        per_head = sum(self.valid_keys(i) for i in range(self.n_q))
        return per_head * self.B * self.H


def outlier_channels(w: Workload) -> np.ndarray:
    """[B*H, n_outlier] distinct channel indices per (b, h)."""
    n_out = w.n_outlier
    out = np.zeros((w.B * w.H, n_out), dtype=np.int64)
    for bh in range(w.B * w.H):
        chosen: list[int] = []
        t = 0
        while len(chosen) < n_out:
            c = int(stream_values(w.seed, STREAM_OUTLIER, np.array([bh * 64 + t]))[0] % np.uint64(w.d))
            t += 1
            if c not in chosen:
                chosen.append(c)
        out[bh] = chosen
    return out


def make_tensor(w: Workload, stream: int, n: int) -> np.ndarray:
    """bf16 bits [B, H, n, d] for stream Q (n = n_q), K or V (n = n_k)."""
    count = w.B * w.H * n * w.d
    x = normal_f64(w.seed, stream, 0, count).reshape(w.B * w.H, n, w.d)
    if w.n_outlier and stream in (STREAM_Q, STREAM_K):
        ch = outlier_channels(w)
        for bh in range(w.B * w.H):
            x[bh][:, ch[bh]] *= w.outlier_scale
    return to_bf16_bits(x.reshape(-1)).reshape(w.B, w.H, n, w.d)


def make_qkv(w: Workload) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Q, K, V as uint16 bf16 bit patterns, contiguous [B, H, n, d]."""
    return (make_tensor(w, STREAM_Q, w.n_q), make_tensor(w, STREAM_K, w.n_k),
            make_tensor(w, STREAM_V, w.n_k))


def random_control_mask(w: Workload, counts: np.ndarray, bh_list=None) -> np.ndarray:
    """Bit-packed mask choosing, per query row, ``counts[bh, i]`` valid keys uniformly
    without replacement (the random-selection control at a matched per-row count).

    Each valid key gets a 64-bit stream value and the row keeps the ``count`` keys
    with the smallest values (ties to the lower key index): a uniform random subset.
    Returns uint32 words [len(bh_list), n_q, ceil(n_k/32)], bit j%32 of word j//32.
    """
    if bh_list is None:
        bh_list = range(w.B * w.H)
    nwords = (w.n_k + 31) // 32
    bh_list = list(bh_list)
    out = np.zeros((len(bh_list), w.n_q, nwords), dtype=np.uint32)
    jj = np.arange(w.n_k, dtype=np.uint64)
    nvalid = np.array([w.valid_keys(i) for i in range(w.n_q)])
    for t, bh in enumerate(bh_list):
        base = np.uint64(bh) * np.uint64(w.n_q) * np.uint64(w.n_k)
        rows = np.arange(w.n_q, dtype=np.uint64)[:, None] * np.uint64(w.n_k)
        keys = stream_values(w.seed, STREAM_RANDOM, base + rows + jj[None, :])
        keys[jj[None, :].astype(np.int64) >= nvalid[:, None]] = np.uint64(0xFFFFFFFFFFFFFFFF)
        order = np.argsort(keys, axis=1, kind="stable")
        c = np.asarray(counts[t], dtype=np.int64)
        if np.any(c > nvalid):
            raise ValueError("count exceeds the number of valid keys")
        rank = np.empty_like(order)
        np.put_along_axis(rank, order, np.arange(w.n_k)[None, :].repeat(w.n_q, 0), axis=1)
        out[t] = pack_mask(rank < c[:, None])
    return out


def pack_mask(bits: np.ndarray) -> np.ndarray:
    """bool [..., n_k] -> uint32 words [..., ceil(n_k/32)] (bit j%32 of word j//32)."""
    bits = np.asarray(bits, dtype=bool)
    n_k = bits.shape[-1]
    nwords = (n_k + 31) // 32
    pad = np.zeros(bits.shape[:-1] + (nwords * 32,), dtype=bool)
    pad[..., :n_k] = bits
    w = pad.reshape(bits.shape[:-1] + (nwords, 32)).astype(np.uint64)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (w * weights).sum(axis=-1).astype(np.uint32)


def unpack_mask(words: np.ndarray, n_k: int) -> np.ndarray:
    """uint32 words [..., nwords] -> bool [..., n_k]."""
    words = np.asarray(words, dtype=np.uint32)
    b = (words[..., :, None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    return b.reshape(words.shape[:-1] + (-1,))[..., :n_k].astype(bool)


# The five workloads of the benchmark/parity suite: the GPT-2 XL attention shape
# and its neighbours (a single head, a batch of 8, a 16K-token context with
# d=128, and a peaked/outlier variant).
WORKLOADS = {
    "single_head_128": Workload(1, 1, 128, 128, 64),
    "gpt2xl_1x25x1024x64": Workload(1, 25, 1024, 1024, 64),
    "batch8_8x25x1024x64": Workload(8, 25, 1024, 1024, 64),
    "long_1x32x16384x128": Workload(1, 32, 16384, 16384, 128),
    # a smaller case of the streamed relaxed kernel, sized for profiling captures
    "long_1x8x4096x128": Workload(1, 8, 4096, 4096, 128),
    # decode: one new query per head against a 16K-token key/value cache
    "decode_1x32x1x16384x128": Workload(1, 32, 1, 16384, 128),
    "outlier_4x25x4096x64": Workload(4, 25, 4096, 4096, 64, outlier_frac=0.01),
}


@dataclass(frozen=True)
class LinearWorkload:
    """One synthetic activation problem: GELU(scale * x W^T), x [M, K], W [N, K],
    iid N(0,1) bf16 entries; scale = fl32(1/sqrt(K)) makes the pre-activations
    about N(0,1)."""

    M: int
    N: int
    K: int
    seed: int = 0

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.K)))

    def outputs(self) -> int:
        return self.M * self.N

    def as_rows(self) -> Workload:
        """The same shape as a one-head non-causal attention workload (rows of x
        against rows of W), for the row-wise random-control masks."""
        return Workload(1, 1, self.M, self.N, self.K, causal=False, seed=self.seed)


def make_linear(lw: LinearWorkload) -> tuple[np.ndarray, np.ndarray]:
    """x [M, K] and W [N, K] as uint16 bf16 bit patterns."""
    x = to_bf16_bits(normal_f64(lw.seed, STREAM_X, 0, lw.M * lw.K)).reshape(lw.M, lw.K)
    W = to_bf16_bits(normal_f64(lw.seed, STREAM_W, 0, lw.N * lw.K)).reshape(lw.N, lw.K)
    return x, W


def linear_random_mask(lw: LinearWorkload, counts: np.ndarray) -> np.ndarray:
    """Mask [M, ceil(N/32)] choosing ``counts[i]`` of the N outputs of row i
    uniformly without replacement (the random control at a matched row count)."""
    return random_control_mask(lw.as_rows(), np.asarray(counts)[None, :])[0]


LINEAR_WORKLOADS = {
    "gelu_small_96x300x200": LinearWorkload(96, 300, 200),
    # GPT-2 XL's first MLP layer (1600 -> 6400) on 1024 tokens
    "gelu_gpt2xl_fc_1024x6400x1600": LinearWorkload(1024, 6400, 1600),
    # LayerNorm after a linear map
    "ln_small_64x300x128": LinearWorkload(64, 300, 128),
    # GPT-2 XL's attention output projection (1600 -> 1600) on 1024 tokens
    "ln_gpt2xl_proj_1024x1600x1600": LinearWorkload(1024, 1600, 1600),
}
