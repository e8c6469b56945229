"""ctypes binding of the CPU oracle (``lamp_oracle.c``: attention;
``lamp_oracle_act.c``: GELU after a PS(mu) linear map; ``lamp_oracle_ln.c``:
LayerNorm after a PS(mu) linear map).

Test infrastructure only: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs use it; the CUDA library and its
Python binding never import it. The C library is single threaded; callers that
want several cores run disjoint row lists from Python threads (ctypes releases
the GIL during the call).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, f) for f in ("lamp_oracle.c", "lamp_oracle_act.c", "lamp_oracle_ln.c")]
_LIB = os.path.join(_HERE, "liblamp_oracle.so")
_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c99"]

STRICT, RELAXED, GIVEN_MASK = 0, 1, 2
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C, no contraction of a*b+c)."""
    if force or not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(f) for f in _SRCS):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, *_SRCS, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.c_void_p
            L.lamp_oracle_round_ps.restype = ctypes.c_float
            L.lamp_oracle_round_ps.argtypes = [ctypes.c_float, ctypes.c_int]
            L.lamp_oracle_round_ps_array.restype = None
            L.lamp_oracle_round_ps_array.argtypes = [P, P, ctypes.c_int64, ctypes.c_int]
            L.lamp_oracle_ps_dot.restype = ctypes.c_float
            L.lamp_oracle_ps_dot.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_float]
            L.lamp_oracle_fp32_dot.restype = ctypes.c_float
            L.lamp_oracle_fp32_dot.argtypes = [P, P, ctypes.c_int, ctypes.c_float]
            L.lamp_oracle_strict_criterion.restype = None
            L.lamp_oracle_strict_criterion.argtypes = [P, ctypes.c_int, P]
            L.lamp_oracle_relaxed_criterion.restype = None
            L.lamp_oracle_relaxed_criterion.argtypes = [P, ctypes.c_int, P]
            L.lamp_oracle_softmax_pv.restype = None
            L.lamp_oracle_softmax_pv.argtypes = [P, ctypes.c_int, P, ctypes.c_int, P, P, P]
            L.lamp_oracle_rows.restype = ctypes.c_int
            L.lamp_oracle_rows.argtypes = [P, ctypes.c_int, P, P, P, ctypes.c_float, ctypes.c_int,
                                           ctypes.c_double, ctypes.c_int, P, P, ctypes.c_int64,
                                           P, P, P, P, P, P, P, P]
            L.lamp_oracle_row_kl.restype = ctypes.c_double
            L.lamp_oracle_row_kl.argtypes = [P, P, ctypes.c_int]
            L.lamp_oracle_kl_rows.restype = None
            L.lamp_oracle_kl_rows.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int64, P]
            L.lamp_oracle_gelu.restype = ctypes.c_double
            L.lamp_oracle_gelu.argtypes = [ctypes.c_double]
            L.lamp_oracle_gelu_kappa.restype = ctypes.c_double
            L.lamp_oracle_gelu_kappa.argtypes = [ctypes.c_double]
            L.lamp_oracle_layernorm.restype = ctypes.c_double
            L.lamp_oracle_layernorm.argtypes = [P, ctypes.c_int64, ctypes.c_double, P]
            L.lamp_oracle_ln_select.restype = ctypes.c_int64
            L.lamp_oracle_ln_select.argtypes = [P, ctypes.c_int64, ctypes.c_double, ctypes.c_double, P, P]
            L.lamp_oracle_ln_thresholds.restype = None
            L.lamp_oracle_ln_thresholds.argtypes = [P, ctypes.c_int64, ctypes.c_double, P]
            L.lamp_oracle_linear_ln_rows.restype = ctypes.c_int
            L.lamp_oracle_linear_ln_rows.argtypes = [P, P, P, ctypes.c_float, ctypes.c_int, ctypes.c_double,
                                                     ctypes.c_double, ctypes.c_int, P, P, ctypes.c_int64, P, P, P,
                                                     P, P, P, P]
            L.lamp_oracle_linear_gelu_rows.restype = ctypes.c_int
            L.lamp_oracle_linear_gelu_rows.argtypes = [P, P, P, ctypes.c_float, ctypes.c_int, ctypes.c_double,
                                                       ctypes.c_int, P, P, ctypes.c_int64, P, P, P, P, P, P]
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_scale(d: int) -> float:
    """fl32(1/sqrt(d)): 1/sqrt(d) in double, rounded once to binary32."""
    return float(np.float32(1.0 / np.sqrt(np.float64(d))))


def round_ps(x, mu: int) -> np.ndarray:
    """Elementwise PS(mu) rounding of a float32 array."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(x)
    lib().lamp_oracle_round_ps_array(_ptr(x), _ptr(out), x.size, int(mu))
    return out


def ps_dot(q_bits, k_bits, mu: int, scale: float) -> np.float32:
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    return np.float32(lib().lamp_oracle_ps_dot(_ptr(q), _ptr(k), q.size, mu, scale))


def fp32_dot(q_bits, k_bits, scale: float) -> np.float32:
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    return np.float32(lib().lamp_oracle_fp32_dot(_ptr(q), _ptr(k), q.size, scale))


def strict_criterion(ps) -> np.ndarray:
    ps = np.ascontiguousarray(ps, dtype=np.float32)
    c = np.zeros(ps.size, dtype=np.float64)
    lib().lamp_oracle_strict_criterion(_ptr(ps), ps.size, _ptr(c))
    return c


def relaxed_criterion(ps) -> np.ndarray:
    ps = np.ascontiguousarray(ps, dtype=np.float32)
    c = np.zeros(ps.size, dtype=np.float64)
    lib().lamp_oracle_relaxed_criterion(_ptr(ps), ps.size, _ptr(c))
    return c


def softmax_pv(y, V_bits):
    """Softmax of a score row and P.V (double). Returns (out[d], lse, P[n])."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    n, d = V.shape
    out = np.zeros(d, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    P = np.zeros(n, dtype=np.float64)
    lib().lamp_oracle_softmax_pv(_ptr(y), n, _ptr(V), d, _ptr(out), _ptr(lse), _ptr(P))
    return out, float(lse[0]), P


class RowResult:
    """Per-row oracle outputs for a list of query rows."""

    def __init__(self, nrows, n_k, d, want_scores=True, want_crit=False):
        nw = (n_k + 31) // 32
        self.ps = np.empty((nrows, n_k), np.float32) if want_scores else None
        self.y32 = np.empty((nrows, n_k), np.float32) if want_scores else None
        self.mixed = np.empty((nrows, n_k), np.float32) if want_scores else None
        self.mask = np.zeros((nrows, nw), np.uint32)
        self.crit = np.empty((nrows, n_k), np.float64) if want_crit else None
        self.out = np.empty((nrows, d), np.float64)
        self.lse = np.empty(nrows, np.float64)
        self.nsel = np.zeros(nrows, np.int64)


def attention_rows(Q, K, V, *, causal=True, scale=None, mu=4, tau=0.0, variant=STRICT,
                   mask_in=None, rows=None, want_scores=True, want_crit=False,
                   threads: int = 1) -> RowResult:
    """Oracle LAMP attention for selected query rows.

    Q: uint16 [B, H, n_q, d]; K, V: uint16 [B, H, n_k, d] (bf16 bit patterns).
    rows: flat row ids (b*H + h)*n_q + i, or None for every row.
    """
    Q = np.ascontiguousarray(Q, dtype=np.uint16)
    K = np.ascontiguousarray(K, dtype=np.uint16)
    V = np.ascontiguousarray(V, dtype=np.uint16)
    B, H, n_q, d = Q.shape
    n_k = K.shape[2]
    if scale is None:
        scale = default_scale(d)
    if rows is None:
        rows = np.arange(B * H * n_q, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    res = RowResult(rows.size, n_k, d, want_scores, want_crit)
    dims = np.array([B, H, n_q, n_k, d], dtype=np.int64)
    if mask_in is not None:
        mask_in = np.ascontiguousarray(mask_in, dtype=np.uint32)
    L = lib()

    def run(lo, hi):
        sub = slice(lo, hi)
        rc = L.lamp_oracle_rows(
            _ptr(dims), int(causal), _ptr(Q), _ptr(K), _ptr(V), float(scale), int(mu), float(tau),
            int(variant), _ptr(mask_in), _ptr(rows[sub]), hi - lo,
            None if res.ps is None else _ptr(res.ps[sub]),
            None if res.y32 is None else _ptr(res.y32[sub]),
            None if res.mixed is None else _ptr(res.mixed[sub]),
            _ptr(res.mask[sub]), None if res.crit is None else _ptr(res.crit[sub]),
            _ptr(res.out[sub]), _ptr(res.lse[sub]), _ptr(res.nsel[sub]))
        if rc != 0:
            raise ValueError(f"oracle rejected its arguments (rc={rc})")

    n = rows.size
    if threads <= 1 or n < 2 * threads:
        run(0, n)
    else:
        # interleaved chunks so that causal rows of different lengths spread evenly
        chunk = max(1, n // (threads * 8))
        bounds = [(lo, min(n, lo + chunk)) for lo in range(0, n, chunk)]
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda b: run(*b), bounds))
    return res


def kl_rows(y_ref, y_x, n_valid) -> np.ndarray:
    y_ref = np.ascontiguousarray(y_ref, dtype=np.float32)
    y_x = np.ascontiguousarray(y_x, dtype=np.float32)
    nv = np.ascontiguousarray(n_valid, dtype=np.int32)
    nrows, n_k = y_ref.shape
    kl = np.zeros(nrows, dtype=np.float64)
    lib().lamp_oracle_kl_rows(_ptr(y_ref), _ptr(y_x), _ptr(nv), nrows, n_k, _ptr(kl))
    return kl


def calibrate_tau(crit: np.ndarray, n_valid_per_row, rate: float) -> float:
    """tau giving round(rate * valid) selections: the (k+1)-th largest criterion
    value among valid entries (entries strictly above it are selected)."""
    vals = np.concatenate([crit[r, :n] for r, n in enumerate(n_valid_per_row)])
    k = int(round(rate * vals.size))
    if k >= vals.size:
        return -1.0
    return float(np.partition(vals, vals.size - 1 - k)[vals.size - 1 - k])


# --------------------------------------------------------------------------------------
# LAMP on an elementwise activation: GELU(scale * x W^T) with a PS(mu) linear map
# --------------------------------------------------------------------------------------

def gelu(y) -> np.ndarray:
    """GELU (tanh form) in double, elementwise."""
    y = np.asarray(y, dtype=np.float64)
    f = np.vectorize(lambda v: lib().lamp_oracle_gelu(float(v)), otypes=[np.float64])
    return f(y)


def gelu_kappa(y) -> np.ndarray:
    """Component-wise condition number |y f'(y) / f(y)| of the tanh-form GELU, in double."""
    y = np.asarray(y, dtype=np.float64)
    f = np.vectorize(lambda v: lib().lamp_oracle_gelu_kappa(float(v)), otypes=[np.float64])
    return f(y)


class ActResult:
    """Per-row oracle outputs of LAMP GELU(scale * x W^T) for a list of rows."""

    def __init__(self, nrows, N):
        self.ps = np.empty((nrows, N), np.float32)
        self.mixed = np.empty((nrows, N), np.float32)
        self.kappa = np.empty((nrows, N), np.float64)
        self.mask = np.zeros((nrows, (N + 31) // 32), np.uint32)
        self.out = np.empty((nrows, N), np.float64)
        self.nsel = np.zeros(nrows, np.int64)


def linear_gelu_rows(x, W, *, scale=1.0, mu=4, tau=0.0, variant=STRICT, mask_in=None, rows=None,
                     threads: int = 1) -> ActResult:
    """Oracle LAMP GELU(scale * x W^T) for selected rows of x.

    x: uint16 [M, K], W: uint16 [N, K] (bf16 bit patterns). variant STRICT is the
    kappa test; GIVEN_MASK takes mask_in [M, ceil(N/32)]. rows: row ids of x, or
    None for every row.
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    W = np.ascontiguousarray(W, dtype=np.uint16)
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("x and W disagree on K")
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    res = ActResult(rows.size, N)
    dims = np.array([M, N, K], dtype=np.int64)
    if mask_in is not None:
        mask_in = np.ascontiguousarray(mask_in, dtype=np.uint32).reshape(M, -1)
    L = lib()

    def run(lo, hi):
        sub = slice(lo, hi)
        rc = L.lamp_oracle_linear_gelu_rows(
            _ptr(dims), _ptr(x), _ptr(W), float(scale), int(mu), float(tau), int(variant), _ptr(mask_in),
            _ptr(rows[sub]), hi - lo, _ptr(res.ps[sub]), _ptr(res.mixed[sub]), _ptr(res.kappa[sub]),
            _ptr(res.mask[sub]), _ptr(res.out[sub]), _ptr(res.nsel[sub]))
        if rc != 0:
            raise ValueError(f"oracle rejected its arguments (rc={rc})")

    n = rows.size
    if threads <= 1 or n < 2 * threads:
        run(0, n)
    else:
        chunk = max(1, n // (threads * 4))
        bounds = [(lo, min(n, lo + chunk)) for lo in range(0, n, chunk)]
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda b: run(*b), bounds))
    return res


def act_errors(out_x, y_x, out_ref, y_ref) -> dict:
    """Errors of activation outputs against the all-FP32 ones.

    l1_rel : l1 error relative to the l1 norm of the reference outputs;
    max_rel: the largest component-wise relative output error;
    max_amp, p99_amp: the largest (99th percentile) realised amplification of a
             component's relative input error into its relative output error,
             |f(y_x) - f(y)| / |f(y)| over |y_x - y| / |y|, over the components
             whose input differs from the FP32 one (the quantity that the
             component-wise condition number bounds to first order).
    """
    a = np.asarray(out_x, dtype=np.float64)
    r = np.asarray(out_ref, dtype=np.float64)
    yx = np.asarray(y_x, dtype=np.float64)
    yr = np.asarray(y_ref, dtype=np.float64)
    diff = np.abs(a - r)
    nz = r != 0.0
    rel = diff[nz] / np.abs(r[nz])
    m = (yx != yr) & nz & (yr != 0.0)
    amp = (diff[m] / np.abs(r[m])) / (np.abs(yx[m] - yr[m]) / np.abs(yr[m]))
    return {"l1_rel": float(diff.sum() / np.abs(r).sum()), "max_rel": float(rel.max()) if rel.size else 0.0,
            "max_amp": float(amp.max()) if amp.size else 0.0,
            "p99_amp": float(np.percentile(amp, 99)) if amp.size else 0.0}


# --------------------------------------------------------------------------------------
# LAMP on LayerNorm: LN(scale * x W^T) with a PS(mu) linear map
# --------------------------------------------------------------------------------------
LN_EPS = float(np.float32(1e-5))  # GPT-2's layer-norm epsilon, as the binary32 the C ABI takes


def layernorm(y, eps: float = LN_EPS):
    """LayerNorm of one row (no affine part) in double. Returns (out, sigma)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty_like(y)
    sigma = lib().lamp_oracle_layernorm(_ptr(y), y.size, float(eps), _ptr(out))
    return out, sigma


def ln_select(ps_row, tau: float, eps: float = LN_EPS):
    """Greedy selection of one row: (0/1 int32 mask, k, unselected sum of squares)."""
    ps_row = np.ascontiguousarray(ps_row, dtype=np.float32)
    sel = np.zeros(ps_row.size, dtype=np.int32)
    rest = np.zeros(1, dtype=np.float64)
    k = lib().lamp_oracle_ln_select(_ptr(ps_row), ps_row.size, float(eps), float(tau), _ptr(sel), _ptr(rest))
    return sel, int(k), float(rest[0])


def ln_thresholds(ps_row, eps: float = LN_EPS) -> np.ndarray:
    """The tau values at which one row's greedy count changes (non-decreasing)."""
    ps_row = np.ascontiguousarray(ps_row, dtype=np.float32)
    t = np.empty(ps_row.size, dtype=np.float64)
    lib().lamp_oracle_ln_thresholds(_ptr(ps_row), ps_row.size, float(eps), _ptr(t))
    return t


class LnResult:
    """Per-row oracle outputs of LAMP LayerNorm(scale * x W^T)."""

    def __init__(self, nrows, N):
        self.ps = np.empty((nrows, N), np.float32)
        self.mixed = np.empty((nrows, N), np.float32)
        self.out = np.empty((nrows, N), np.float64)
        self.mask = np.zeros((nrows, (N + 31) // 32), np.uint32)
        self.nsel = np.zeros(nrows, np.int64)
        self.sigma = np.zeros(nrows, np.float64)
        self.rest = np.zeros(nrows, np.float64)


def linear_ln_rows(x, W, *, scale=1.0, mu=4, tau=0.0, eps=LN_EPS, variant=STRICT, mask_in=None, rows=None,
                   threads: int = 1) -> LnResult:
    """Oracle LAMP LayerNorm(scale * x W^T) for selected rows of x (x [M, K],
    W [N, K] bf16 bits). variant STRICT is the greedy selection; GIVEN_MASK
    takes mask_in [M, ceil(N/32)]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    W = np.ascontiguousarray(W, dtype=np.uint16)
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("x and W disagree on K")
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    res = LnResult(rows.size, N)
    dims = np.array([M, N, K], dtype=np.int64)
    if mask_in is not None:
        mask_in = np.ascontiguousarray(mask_in, dtype=np.uint32).reshape(M, -1)
    L = lib()

    def run(lo, hi):
        sub = slice(lo, hi)
        rc = L.lamp_oracle_linear_ln_rows(
            _ptr(dims), _ptr(x), _ptr(W), float(scale), int(mu), float(tau), float(eps), int(variant),
            _ptr(mask_in), _ptr(rows[sub]), hi - lo, _ptr(res.ps[sub]), _ptr(res.mixed[sub]), _ptr(res.out[sub]),
            _ptr(res.mask[sub]), _ptr(res.nsel[sub]), _ptr(res.sigma[sub]), _ptr(res.rest[sub]))
        if rc != 0:
            raise ValueError(f"oracle rejected its arguments (rc={rc})")

    n = rows.size
    if threads <= 1 or n < 2 * threads:
        run(0, n)
    else:
        chunk = max(1, n // (threads * 4))
        bounds = [(lo, min(n, lo + chunk)) for lo in range(0, n, chunk)]
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda b: run(*b), bounds))
    return res


def ln_errors(out_x, out_ref) -> dict:
    """Row errors of LayerNorm outputs against the all-FP32 ones: the mean and the
    largest l2 error of a row (the quantity the norm-wise bound controls)."""
    d = np.linalg.norm(np.asarray(out_x, np.float64) - np.asarray(out_ref, np.float64), axis=-1)
    return {"mean_l2": float(d.mean()), "max_l2": float(d.max())}
