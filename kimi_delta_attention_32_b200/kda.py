"""Thin ctypes binding of libkda (the C ABI in include/kda.h).

Argument marshalling only: every step of the computation runs in libkda's CUDA
kernels. Tensors are torch CUDA tensors (torch provides device memory and
streams); the current torch stream is passed unless one is given. If libkda.so
is missing this module raises on first use -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_ERR_CUDA, \
    KDA_ERR_TIMEOUT = range(6)
KDA_IO_F32, KDA_IO_BF16 = 0, 1

EXPORTED = ("kda_status_string", "kda_version", "kda_conv_fwd", "kda_chunk_fwd_workspace_size",
            "kda_chunk_fwd", "kda_chunk_fwd_fused", "kda_chunk_fwd_noalloc", "kda_recurrent_step",
            "kda_conv_recurrent_step", "kda_fused_recurrent_step", "kda_set_wait_limit",
            "kda_last_device_error", "kda_chunk_states", "kda_state_scan",
            "kda_chunk_fwd_split_workspace_size", "kda_chunk_fwd_split", "kda_output_correct",
            "kda_chunk_fwd_split_plan")

_lock = threading.Lock()
_lib = None


class KdaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


def load_library(path: str = LIB_PATH):
    """Load libkda.so and declare its signatures. Raises if it is missing."""
    global _lib
    with _lock:
        if _lib is not None and path == LIB_PATH:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"libkda.so not found at {path}; build it with "
                               "`python -m kimi_delta_attention_32_b200.build`")
        lib = ctypes.CDLL(path)
        vp, i32p, fp = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
        ci, cf, cs = ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.kda_status_string.argtypes = [ci]
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_version.argtypes = []
        lib.kda_version.restype = ci
        lib.kda_conv_fwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, vp, vp, i32p,
                                     ctypes.POINTER(ctypes.c_int32), ci, ci, ci, ci, ci, ci, ci,
                                     cf, ci, vp]
        lib.kda_conv_fwd.restype = ci
        lib.kda_chunk_fwd_workspace_size.argtypes = [ci, ctypes.c_int64, ci, ci, ci, ci, ci,
                                                     ctypes.POINTER(cs)]
        lib.kda_chunk_fwd_workspace_size.restype = ci
        lib.kda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, cf, fp, fp, vp, i32p,
                                      ctypes.POINTER(ctypes.c_int32), ci, ci, ci, ci, ci, ci, ci,
                                      ci, vp, cs, vp]
        lib.kda_chunk_fwd.restype = ci
        lib.kda_chunk_fwd_fused.argtypes = [vp, vp, vp, fp, fp, fp, vp, cf, fp, fp, vp, vp, fp, fp, vp,
                                            fp, cf, cf, fp, fp, vp, i32p,
                                            ctypes.POINTER(ctypes.c_int32), ci, ci, ci, ci, ci, ci,
                                            ci, ci, ci, vp, cs, vp]
        lib.kda_chunk_fwd_fused.restype = ci
        lib.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, fp, fp, cf, fp, fp, vp, i32p,
                                              ctypes.POINTER(ctypes.c_int32), ci, ci, ci, ci, ci, ci,
                                              ci, ci, vp]
        lib.kda_chunk_fwd_noalloc.restype = ci
        lib.kda_recurrent_step.argtypes = [vp, vp, vp, fp, fp, cf, fp, vp, ci, ci, ci, ci, ci, vp]
        lib.kda_recurrent_step.restype = ci
        lib.kda_conv_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, fp, cf, fp, vp, ci,
                                                ci, ci, ci, ci, cf, ci, vp]
        lib.kda_conv_recurrent_step.restype = ci
        lib.kda_fused_recurrent_step.argtypes = [vp, vp, vp, vp, vp, fp, fp, fp, vp, fp, fp, vp, fp,
                                                 cf, cf, fp, vp, ci, ci, ci, ci, ci, cf, ci, vp]
        lib.kda_fused_recurrent_step.restype = ci
        lib.kda_set_wait_limit.argtypes = [ctypes.c_int64]
        lib.kda_set_wait_limit.restype = ci
        lib.kda_last_device_error.argtypes = [vp]
        lib.kda_last_device_error.restype = ci
        cip = ctypes.POINTER(ctypes.c_int32)
        lib.kda_chunk_states.argtypes = [vp, vp, vp, fp, fp, cf, fp, fp, vp, fp, vp, i32p, cip, ci,
                                         ci, ci, ci, ci, ci, ci, ci, vp, cs, vp]
        lib.kda_chunk_states.restype = ci
        lib.kda_state_scan.argtypes = [fp, fp, fp, fp, fp, ci, ci, ci, ci, ci, ctypes.c_int64,
                                       ctypes.c_int64, vp]
        lib.kda_state_scan.restype = ci
        lib.kda_chunk_fwd_split_workspace_size.argtypes = [cip, ci, ci, ci, ci, ci, ci, ci, ci, ci,
                                                           ctypes.POINTER(ci), ctypes.POINTER(cs)]
        lib.kda_chunk_fwd_split_workspace_size.restype = ci
        lib.kda_chunk_fwd_split.argtypes = [vp, vp, vp, fp, fp, cf, fp, fp, vp, i32p, cip, ci, ci,
                                            ci, ci, ci, ci, ci, ci, ci, vp, cs, vp]
        lib.kda_chunk_fwd_split.restype = ci
        lib.kda_output_correct.argtypes = [vp, fp, vp, i32p, cip, ci, ci, ci, ci, ci, ci, ci, vp]
        lib.kda_output_correct.restype = ci
        lib.kda_chunk_fwd_split_plan.argtypes = [cip, ci, ci, ci, ci, ci, ci, ci, ci, ci, ci,
                                                 ctypes.POINTER(ci), ctypes.POINTER(cs)]
        lib.kda_chunk_fwd_split_plan.restype = ci
        if path == LIB_PATH:
            _lib = lib
        return lib


def _check(fn: str, status: int):
    if status != KDA_OK:
        raise KdaError(fn, status, load_library().kda_status_string(status).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _io(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_IO_BF16
    if t.dtype == torch.float32:
        return KDA_IO_F32
    raise TypeError(f"unsupported I/O dtype {t.dtype}")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _host_cu(cu_host):
    if cu_host is None:
        return None, None
    arr = (ctypes.c_int32 * len(cu_host))(*[int(x) for x in cu_host])
    return arr, ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))


def conv_fwd(q_raw, k_raw, v_raw, w_q, w_k, w_v, q_out=None, k_out=None, v_out=None,
             conv_state=None, cu_seqlens=None, cu_host=None, l2_eps=1e-6, K=4, stream=None):
    """Fused causal conv (kernel K) + SiLU + L2 norm of q, k. Shapes: x [T_tot,H,d] for the
    packed form (cu_seqlens given) or [B,T,H,d] for the padded form. Returns (q, k, v)."""
    lib = load_library()
    q_out = torch.empty_like(q_raw) if q_out is None else q_out
    k_out = torch.empty_like(k_raw) if k_out is None else k_out
    v_out = torch.empty_like(v_raw) if v_out is None else v_out
    if cu_seqlens is None:
        B, T, H, dk = q_raw.shape if q_raw.dim() == 4 else (1, *q_raw.shape)
        N = B
    else:
        B, T = 1, 0
        _, H, dk = q_raw.shape
        N = len(cu_host) - 1
    dv = v_raw.shape[-1]
    keep, cuh = _host_cu(cu_host)
    st = lib.kda_conv_fwd(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(w_q), _ptr(w_k), _ptr(w_v),
                          _ptr(q_out), _ptr(k_out), _ptr(v_out), _ptr(conv_state),
                          _ptr(cu_seqlens), cuh, B, T, N, H, dk, dv, K, float(l2_eps),
                          _io(q_raw), _stream(stream))
    del keep
    _check("kda_conv_fwd", st)
    return q_out, k_out, v_out


def chunk_fwd_workspace_size(N, T_tot, H, dk, dv, chunk=64, io=KDA_IO_BF16) -> int:
    lib = load_library()
    out = ctypes.c_size_t(0)
    _check("kda_chunk_fwd_workspace_size",
           lib.kda_chunk_fwd_workspace_size(N, T_tot, H, dk, dv, chunk, io, ctypes.byref(out)))
    return out.value


def chunk_fwd(q, k, v, g, beta, scale=1.0, h0=None, ht=None, o=None, cu_seqlens=None,
              cu_host=None, chunk=64, output_final_state=True, workspace=None, stream=None):
    """Chunked prefill. Packed: q [T_tot,H,dk] with cu_seqlens (device int32) and cu_host
    (list); padded: q [B,T,H,dk]. Returns (o, ht) (ht None if not requested)."""
    lib = load_library()
    if cu_seqlens is None:
        B, T, H, dk = q.shape if q.dim() == 4 else (1, *q.shape)
        N = B
        T_tot = B * T
    else:
        B, T = 1, 0
        T_tot, H, dk = q.shape
        N = len(cu_host) - 1
    dv = v.shape[-1]
    o = torch.empty_like(v) if o is None else o
    if ht is None and output_final_state:
        ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    io = _io(q)
    need = chunk_fwd_workspace_size(N, T_tot, H, dk, dv, chunk, io)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    keep, cuh = _host_cu(cu_host)
    st = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(h0),
                           _ptr(ht), _ptr(o), _ptr(cu_seqlens), cuh, B, T, N, H, dk, dv, chunk,
                           io, _ptr(workspace), 0 if workspace is None else workspace.numel(),
                           _stream(stream))
    del keep
    _check("kda_chunk_fwd", st)
    return o, ht


def _batch(q, cu_seqlens, cu_host):
    if cu_seqlens is None:
        B, T, H, dk = q.shape if q.dim() == 4 else (1, *q.shape)
        return B, T, B, B * T, H, dk
    T_tot, H, dk = q.shape
    return 1, 0, len(cu_host) - 1, T_tot, H, dk


def chunk_states(q, k, v, g, beta, scale=1.0, h0=None, cu_seqlens=None, cu_host=None, chunk=64,
                 end_state=True, transition=True, output=False, carried_queries=False,
                 workspace=None, stream=None):
    """Per (sequence, head): the end state started from h0 (or zero), the transition M, the
    output (as chunk_fwd), and the queries carried back to the start, scale M_t^T q_t.
    Returns (ht [N,H,dk,dv], m [N,H,dk,dk], o [T,H,dv], w [T,H,dk]); each None unless asked."""
    lib = load_library()
    B, T, N, T_tot, H, dk = _batch(q, cu_seqlens, cu_host)
    dv = v.shape[-1]
    ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device) if end_state else None
    m = torch.empty((N, H, dk, dk), dtype=torch.float32, device=q.device) if transition else None
    o = torch.empty_like(v) if output else None
    w = torch.empty_like(q) if carried_queries else None
    io = _io(q)
    if workspace is None:
        need = chunk_fwd_workspace_size(N, T_tot, H, dk, dv, chunk, io)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    keep, cuh = _host_cu(cu_host)
    st = lib.kda_chunk_states(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                              _ptr(h0), _ptr(ht), _ptr(o), _ptr(m), _ptr(w), _ptr(cu_seqlens), cuh,
                              B, T, N, H, dk, dv, chunk, io, _ptr(workspace), workspace.numel(),
                              _stream(stream))
    del keep
    _check("kda_chunk_states", st)
    return ht, m, o, w


def state_scan(m, s_zero, h0=None, *, N, P, seq_stride, seg_stride, h_start=None, ht=None,
               stream=None):
    """Joins stretches: H_0 = h0, H_{p+1} = M_p H_p + Z_p, stretch p of sequence n at index
    n * seq_stride + p * seg_stride of m [*,H,dk,dk] and s_zero [*,H,dk,dv].
    Returns (h_start [*,H,dk,dv], ht [N,H,dk,dv])."""
    lib = load_library()
    H, dk, dv = s_zero.shape[1], s_zero.shape[2], s_zero.shape[3]
    if h_start is None:
        h_start = torch.empty_like(s_zero)
    if ht is None:
        ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=s_zero.device)
    _check("kda_state_scan", lib.kda_state_scan(_ptr(m), _ptr(s_zero), _ptr(h0), _ptr(h_start),
                                                _ptr(ht), N, P, H, dk, dv, seq_stride, seg_stride,
                                                _stream(stream)))
    return h_start, ht


def output_correct(w, h, o, cu_seqlens, cu_host, stream=None):
    """o[t] += h[n]^T w[t] for the tokens t of every sequence n (packed batch, in place)."""
    lib = load_library()
    T_tot, H, dk = w.shape
    keep, cuh = _host_cu(cu_host)
    st = lib.kda_output_correct(_ptr(w), _ptr(h), _ptr(o), _ptr(cu_seqlens), cuh, 1, 0,
                                len(cu_host) - 1, H, dk, o.shape[-1], _io(o), _stream(stream))
    del keep
    _check("kda_output_correct", st)
    return o


def chunk_fwd_split_plan(q, v, cu_seqlens=None, cu_host=None, n_split=0, chunk=64):
    """(stretches per sequence, workspace bytes) of chunk_fwd_split for this batch."""
    lib = load_library()
    B, T, N, _, H, dk = _batch(q, cu_seqlens, cu_host)
    keep, cuh = _host_cu(cu_host)
    P, nbytes = ctypes.c_int(0), ctypes.c_size_t(0)
    st = lib.kda_chunk_fwd_split_workspace_size(cuh, B, T, N, H, dk, v.shape[-1], chunk, _io(q),
                                                n_split, ctypes.byref(P), ctypes.byref(nbytes))
    del keep
    _check("kda_chunk_fwd_split_workspace_size", st)
    return P.value, nbytes.value


def chunk_fwd_split(q, k, v, g, beta, scale=1.0, h0=None, ht=None, o=None, cu_seqlens=None,
                    cu_host=None, n_split=0, chunk=64, workspace=None, stream=None):
    """chunk_fwd with every sequence split into stretches that run side by side (n_split = 0:
    chosen for the batch). Returns (o, ht)."""
    lib = load_library()
    B, T, N, _, H, dk = _batch(q, cu_seqlens, cu_host)
    dv = v.shape[-1]
    o = torch.empty_like(v) if o is None else o
    if ht is None:
        ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        _, need = chunk_fwd_split_plan(q, v, cu_seqlens, cu_host, n_split, chunk)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    keep, cuh = _host_cu(cu_host)
    st = lib.kda_chunk_fwd_split(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                 _ptr(h0), _ptr(ht), _ptr(o), _ptr(cu_seqlens), cuh, B, T, N, H,
                                 dk, dv, chunk, _io(q), n_split, _ptr(workspace), workspace.numel(),
                                 _stream(stream))
    del keep
    _check("kda_chunk_fwd_split", st)
    return o, ht


def chunk_fwd_fused(q, k, v, g=None, beta=None, *, w_q=None, w_k=None, w_v=None,
                    conv_state=None, l2_eps=1e-6, g_raw=None, beta_raw=None, A_log=None,
                    dt_bias=None, z=None, w_norm=None, norm_eps=1e-6, scale=1.0, h0=None, ht=None,
                    o=None, cu_seqlens=None, cu_host=None, chunk=64, K=4, workspace=None,
                    stream=None):
    """Chunked prefill with optional fused steps: the conv prologue (w_q, w_k, w_v given: q, k, v
    are raw projections; conv_state is read as the history and overwritten with the new one),
    the gate from raw logits (g_raw, beta_raw, A_log, dt_bias given; else g and beta are used),
    and the gated RMSNorm of the output (z, w_norm given). Returns (o, ht)."""
    lib = load_library()
    if cu_seqlens is None:
        B, T, H, dk = q.shape if q.dim() == 4 else (1, *q.shape)
        N, T_tot = B, B * T
    else:
        B, T = 1, 0
        T_tot, H, dk = q.shape
        N = len(cu_host) - 1
    dv = v.shape[-1]
    o = torch.empty_like(v) if o is None else o
    if ht is None:
        ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    need = chunk_fwd_workspace_size(N, T_tot, H, dk, dv, chunk, _io(q))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    keep, cuh = _host_cu(cu_host)
    st = lib.kda_chunk_fwd_fused(
        _ptr(q), _ptr(k), _ptr(v), _ptr(w_q), _ptr(w_k), _ptr(w_v), _ptr(conv_state),
        float(l2_eps), _ptr(g), _ptr(beta), _ptr(g_raw), _ptr(beta_raw), _ptr(A_log),
        _ptr(dt_bias), _ptr(z), _ptr(w_norm), float(norm_eps), float(scale), _ptr(h0), _ptr(ht),
        _ptr(o), _ptr(cu_seqlens), cuh, B, T, N, H, dk, dv, K, chunk, _io(q), _ptr(workspace),
        0 if workspace is None else workspace.numel(), _stream(stream))
    del keep
    _check("kda_chunk_fwd_fused", st)
    return o, ht


def chunk_fwd_noalloc(q, k, v, g, beta, scale=1.0, h0=None, ht=None, o=None, cu_seqlens=None,
                      cu_host=None, chunk=64, stream=None):
    """chunk_fwd through kda_chunk_fwd_noalloc: no workspace is allocated for the call (o and
    ht are, unless given). Returns (o, ht)."""
    lib = load_library()
    if cu_seqlens is None:
        B, T, H, dk = q.shape if q.dim() == 4 else (1, *q.shape)
        N = B
    else:
        B, T = 1, 0
        _, H, dk = q.shape
        N = len(cu_host) - 1
    dv = v.shape[-1]
    o = torch.empty_like(v) if o is None else o
    if ht is None:
        ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    keep, cuh = _host_cu(cu_host)
    st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                   _ptr(h0), _ptr(ht), _ptr(o), _ptr(cu_seqlens), cuh, B, T, N, H,
                                   dk, dv, chunk, _io(q), _stream(stream))
    del keep
    _check("kda_chunk_fwd_noalloc", st)
    return o, ht


def recurrent_step(q, k, v, g, beta, state, scale=1.0, o=None, stream=None):
    """One decode token per (sequence, head); q,k,g [N,H,dk], v [N,H,dv], beta [N,H],
    state [N,H,dk,dv] fp32 updated in place. Returns o [N,H,dv]."""
    lib = load_library()
    N, H, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty_like(v) if o is None else o
    st = lib.kda_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                _ptr(state), _ptr(o), N, H, dk, dv, _io(q), _stream(stream))
    _check("kda_recurrent_step", st)
    return o


def conv_recurrent_step(q_raw, k_raw, v_raw, w_q, w_k, w_v, conv_state, g, beta, state,
                        scale=1.0, o=None, l2_eps=1e-6, K=4, stream=None):
    """One decode token from raw q, k, v: conv (cache advanced in place) + SiLU + L2 norm and
    the state update in one kernel. Shapes: raw q, k, g [N,H,dk], v [N,H,dv], beta [N,H],
    conv_state [N, H*(2dk+dv), K-1], state [N,H,dk,dv] fp32 (in place). Returns o [N,H,dv]."""
    lib = load_library()
    N, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    o = torch.empty_like(v_raw) if o is None else o
    st = lib.kda_conv_recurrent_step(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(w_q), _ptr(w_k),
                                     _ptr(w_v), _ptr(conv_state), _ptr(g), _ptr(beta),
                                     float(scale), _ptr(state), _ptr(o), N, H, dk, dv, K,
                                     float(l2_eps), _io(q_raw), _stream(stream))
    _check("kda_conv_recurrent_step", st)
    return o


def fused_recurrent_step(q_raw, k_raw, v_raw, g_raw, beta_raw, w_q, w_k, w_v, conv_state, A_log,
                         dt_bias, state, z=None, w_norm=None, norm_eps=1e-6, scale=1.0, o=None,
                         l2_eps=1e-6, K=4, stream=None):
    """The whole decode step from raw projections: conv (cache in place), gate and beta from raw
    logits, state update, and the gated RMSNorm of the output when z is given. Shapes: raw q, k,
    g [N,H,dk], v, z [N,H,dv], beta_raw [N,H]; A_log [H], dt_bias [H*dk], w_norm [dv].
    Returns o [N,H,dv]."""
    lib = load_library()
    N, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    o = torch.empty_like(v_raw) if o is None else o
    st = lib.kda_fused_recurrent_step(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(g_raw),
                                      _ptr(beta_raw), _ptr(w_q), _ptr(w_k), _ptr(w_v),
                                      _ptr(conv_state), _ptr(A_log), _ptr(dt_bias), _ptr(z),
                                      _ptr(w_norm), float(norm_eps), float(scale), _ptr(state),
                                      _ptr(o), N, H, dk, dv, K, float(l2_eps), _io(q_raw),
                                      _stream(stream))
    _check("kda_fused_recurrent_step", st)
    return o


def set_wait_limit(cycles: int) -> None:
    """Bound (SM cycles) of every device-side wait of later prefill launches; 0 = default."""
    _check("kda_set_wait_limit", load_library().kda_set_wait_limit(int(cycles)))


def last_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device-side error status."""
    return load_library().kda_last_device_error(_stream(stream))
