"""fp64 CPU oracle for Kimi Delta Attention (KDA) -- TEST INFRASTRUCTURE.

This package is the independent checker for libkda. Only the test suite, the
smoke check and the benchmark's CPU-baseline leg may import it; the product
path (the CUDA library and its Python binding) never does. It shares no code
with the CUDA side: the arithmetic lives in ``kda_oracle.c`` (plain C, fp64,
token by token) and this module only marshals numpy arrays into it.

What it computes follows the pages about the AliceAI-Foundation-80B-A3B-Base
model: the sarnas.ru article, section "Что именно изменилось" (fixed-size state,
read-out / compare / write-only-the-correction, one forgetting coefficient per
state row), and the m.lqnn.cn/news/205170 article, section
"KDA 与 Gated Attention：每 4 层只留 1 层全注意力" (kernel-4 causal conv with an
incremental cache, ``state = state * exp(gate) + delta`` with delta the
prediction residual times sigmoid(beta)). The readings where the pages are
silent are listed at the top of ``kda_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def compile_oracle(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile ``src`` into a shared library with plain gcc (no -march tuning)."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c99", *extra_flags, src, "-o", out,
           "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return out


def _declare(lib):
    lib.kda_oracle_fwd.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_double, _dp, _dp, _dp,
                                   _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int]
    lib.kda_oracle_fwd.restype = None
    lib.kda_oracle_gdn_fwd.argtypes = lib.kda_oracle_fwd.argtypes
    lib.kda_oracle_gdn_fwd.restype = None
    lib.kda_oracle_conv_silu.argtypes = [_dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int]
    lib.kda_oracle_conv_silu.restype = None
    lib.kda_oracle_l2norm.argtypes = [_dp, ctypes.c_int64, ctypes.c_int, ctypes.c_double]
    lib.kda_oracle_l2norm.restype = None
    lib.kda_oracle_gate.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
    lib.kda_oracle_gate.restype = None
    lib.kda_oracle_sigmoid.argtypes = [_dp, _dp, ctypes.c_int64]
    lib.kda_oracle_sigmoid.restype = None
    lib.kda_oracle_gated_rmsnorm.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int,
                                             ctypes.c_double]
    lib.kda_oracle_gated_rmsnorm.restype = None
    lib.kda_oracle_transition.argtypes = [_dp, _dp, _dp, _dp, _i64p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int]
    lib.kda_oracle_transition.restype = None
    return lib


def load(path: str | None = None):
    """Load the oracle library, compiling it first if it is missing or stale."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            stale = (not os.path.exists(_LIB_PATH)
                     or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
            if stale:
                compile_oracle()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _cu(cu_seqlens, T_tot):
    if cu_seqlens is None:
        return np.array([0, T_tot], dtype=np.int64)
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))


def kda_fwd(q, k, v, g, beta, scale=1.0, h0=None, cu_seqlens=None, nthreads=None,
            with_state=True, lib=None):
    """Token-by-token KDA over packed sequences.

    q, k, g: [T_tot, H, dk]; v: [T_tot, H, dv]; beta: [T_tot, H];
    h0: [N, H, dk, dv] or None (zero); cu_seqlens: [N+1] or None (one sequence).
    Returns (o [T_tot, H, dv], ht [N, H, dk, dv] or None), both float64.
    """
    lib = lib or load()
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    cu = _cu(cu_seqlens, T_tot)
    N = cu.shape[0] - 1
    h0 = None if h0 is None else _f64(h0)
    o = np.zeros((T_tot, H, dv), dtype=np.float64)
    ht = np.zeros((N, H, dk, dv), dtype=np.float64) if with_state else None
    nthreads = nthreads or os.cpu_count() or 1
    lib.kda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(h0),
                       _ptr(ht), _ptr(o), cu.ctypes.data_as(_i64p), N, H, dk, dv, int(nthreads))
    return o, ht


def transition(k, g, beta, cu_seqlens=None, nthreads=None, lib=None):
    """Transition M of each (sequence, head): the product over its tokens, latest on the left,
    of (I - beta k k^T) diag(exp(g)), so that the sequence started from S ends in
    M S + (the state it ends in from zero). k, g: [T_tot, H, dk]; beta: [T_tot, H].
    Returns m [N, H, dk, dk] (float64)."""
    lib = lib or load()
    k, g, beta = map(_f64, (k, g, beta))
    T_tot, H, dk = k.shape
    cu = _cu(cu_seqlens, T_tot)
    N = cu.shape[0] - 1
    m = np.zeros((N, H, dk, dk), dtype=np.float64)
    nthreads = nthreads or os.cpu_count() or 1
    lib.kda_oracle_transition(_ptr(k), _ptr(g), _ptr(beta), _ptr(m), cu.ctypes.data_as(_i64p), N,
                              H, dk, int(nthreads))
    return m


def gdn_fwd(q, k, v, alpha, beta, scale=1.0, h0=None, cu_seqlens=None, nthreads=None, lib=None):
    """Scalar-gated DeltaNet (Householder form); alpha, beta: [T_tot, H]."""
    lib = lib or load()
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    cu = _cu(cu_seqlens, T_tot)
    N = cu.shape[0] - 1
    h0 = None if h0 is None else _f64(h0)
    o = np.zeros((T_tot, H, dv), dtype=np.float64)
    ht = np.zeros((N, H, dk, dv), dtype=np.float64)
    nthreads = nthreads or os.cpu_count() or 1
    lib.kda_oracle_gdn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), float(scale),
                           _ptr(h0), _ptr(ht), _ptr(o), cu.ctypes.data_as(_i64p), N, H, dk, dv,
                           int(nthreads))
    return o, ht


def conv_silu(x, w, cache_in=None, cu_seqlens=None, lib=None):
    """Causal depthwise conv (no bias) + SiLU per sequence.

    x: [T_tot, C]; w: [C, K]; cache_in: [N, C, K-1] or None.
    Returns (y [T_tot, C], cache_out [N, C, K-1]).
    """
    lib = lib or load()
    x, w = _f64(x), _f64(w)
    T_tot, C = x.shape
    K = w.shape[1]
    cu = _cu(cu_seqlens, T_tot)
    N = cu.shape[0] - 1
    cache_in = None if cache_in is None else _f64(cache_in)
    y = np.zeros_like(x)
    cache_out = np.zeros((N, C, K - 1), dtype=np.float64)
    lib.kda_oracle_conv_silu(_ptr(x), _ptr(w), _ptr(cache_in), _ptr(y), _ptr(cache_out),
                             cu.ctypes.data_as(_i64p), N, C, K)
    return y, cache_out


def l2norm(x, eps, lib=None):
    """x / sqrt(sum x^2 + eps) over the last axis; returns a new float64 array."""
    lib = lib or load()
    x = _f64(x).copy()
    d = x.shape[-1]
    lib.kda_oracle_l2norm(_ptr(x), int(x.size // d), d, float(eps))
    return x


def prologue(q_raw, k_raw, v_raw, w_q, w_k, w_v, conv_state=None, cu_seqlens=None,
             l2_eps=1e-6, lib=None):
    """The fused prologue: conv+SiLU on q, k, v, then L2 norm on q and k.

    q_raw, k_raw: [T_tot, H, dk]; v_raw: [T_tot, H, dv]; w_*: [H*d, K];
    conv_state: [N, H*(2dk+dv), K-1] (q channels, then k, then v) or None.
    Returns (q, k, v, conv_state_out) in float64 with the input shapes.
    """
    lib = lib or load()
    T_tot, H, dk = np.shape(q_raw)
    dv = np.shape(v_raw)[2]
    Cq, Cv = H * dk, H * dv
    cs = None if conv_state is None else _f64(conv_state)
    parts = []
    outs_cache = []
    for x, w, lo, hi in ((q_raw, w_q, 0, Cq), (k_raw, w_k, Cq, 2 * Cq),
                         (v_raw, w_v, 2 * Cq, 2 * Cq + Cv)):
        xin = _f64(x).reshape(T_tot, -1)
        cin = None if cs is None else cs[:, lo:hi, :]
        y, cout = conv_silu(xin, w, cin, cu_seqlens, lib=lib)
        parts.append(y)
        outs_cache.append(cout)
    q = l2norm(parts[0].reshape(T_tot, H, dk), l2_eps, lib=lib)
    k = l2norm(parts[1].reshape(T_tot, H, dk), l2_eps, lib=lib)
    v = parts[2].reshape(T_tot, H, dv)
    return q, k, v, np.concatenate(outs_cache, axis=1)


def gate(x, A_log, dt_bias, lib=None):
    """Per-channel log-decay from raw gate logits: g = -exp(A_log[h]) softplus(x + dt_bias).
    x: [T_tot, H, dk]; A_log: [H]; dt_bias: [H*dk] (or [H, dk]). Returns g (float64)."""
    lib = lib or load()
    x = _f64(x)
    T_tot, H, dk = x.shape
    A_log, dt_bias = _f64(A_log).reshape(H), _f64(dt_bias).reshape(H * dk)
    g = np.zeros_like(x)
    lib.kda_oracle_gate(_ptr(x), _ptr(A_log), _ptr(dt_bias), _ptr(g), T_tot, H, dk)
    return g


def sigmoid(b_raw, lib=None):
    """beta = sigmoid(b_raw), elementwise (float64)."""
    lib = lib or load()
    b = _f64(b_raw)
    out = np.zeros_like(b)
    lib.kda_oracle_sigmoid(_ptr(b), _ptr(out), b.size)
    return out


def gated_rmsnorm(o, z, w, eps=1e-6, lib=None):
    """y = o / sqrt(mean(o^2) + eps) * w * sigmoid(z) over the last axis (dv); w: [dv]."""
    lib = lib or load()
    o, z, w = _f64(o), _f64(z), _f64(w)
    dv = o.shape[-1]
    y = np.zeros_like(o)
    lib.kda_oracle_gated_rmsnorm(_ptr(o), _ptr(z), _ptr(w), _ptr(y), o.size // dv, dv, float(eps))
    return y
