"""Shared helpers of the GPU parity tests: run libkda on seeded inputs and compare the
results with the fp64 oracle, which reads back the exact bytes the GPU consumed."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from conftest import rel_l2
from kimi_delta_attention_32_b200 import kda

# Tolerances of the parity bar: relative L2 error (fp64, whole tensor).
TOL_F32 = 1e-4        # fp32 I/O
TOL_BF16 = 1e-2       # bf16 I/O with fp32 gates, beta and state


def tol_for(io: str) -> float:
    return TOL_F32 if io == "f32" else TOL_BF16


def to64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def oracle_prefill(d, q, k, v, pairs=None, nthreads=None):
    """Oracle o and ht for a prefill input dict; q, k, v are the tensors the GPU consumed.
    pairs: optional list of (sequence, head) to restrict the check to. Returns
    (o_ref, ht_ref, select) where select(o, ht) cuts the GPU results to the same pairs."""
    cu = d["cu_host"]
    if pairs is None:
        o, ht = oracle.kda_fwd(to64(q), to64(k), to64(v), to64(d["g"]), to64(d["beta"]),
                               d["scale"], to64(d["h0"]), cu, nthreads=nthreads)
        return o, ht, (lambda og, hg: (to64(og), to64(hg)))
    o_parts, h_parts, idx = [], [], []
    for n, h in pairs:
        sl = slice(cu[n], cu[n + 1])
        h0 = None if d["h0"] is None else to64(d["h0"][n:n + 1, h:h + 1])
        o, ht = oracle.kda_fwd(to64(q[sl, h:h + 1]), to64(k[sl, h:h + 1]), to64(v[sl, h:h + 1]),
                               to64(d["g"][sl, h:h + 1]), to64(d["beta"][sl, h:h + 1]),
                               d["scale"], h0, None, nthreads=1)
        o_parts.append(o)
        h_parts.append(ht)
        idx.append((sl, n, h))

    def select(og, hg):
        oo = np.concatenate([to64(og[sl, h:h + 1]) for sl, n, h in idx])
        hh = np.concatenate([to64(hg[n:n + 1, h:h + 1]) for sl, n, h in idx])
        return oo, hh

    return np.concatenate(o_parts), np.concatenate(h_parts), select


def check_prefill(d, q, k, v, o, ht, pairs=None, tol=None, nthreads=None):
    tol = tol if tol is not None else tol_for(d["io"])
    o_ref, h_ref, select = oracle_prefill(d, q, k, v, pairs, nthreads)
    og, hg = select(o, ht)
    eo, eh = rel_l2(og, o_ref), rel_l2(hg, h_ref)
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(hg))
    assert eo <= tol, f"o rel-L2 {eo:.3e} > {tol:.0e}"
    assert eh <= tol, f"ht rel-L2 {eh:.3e} > {tol:.0e}"
    return eo, eh


def run_chunk(d, q=None, k=None, v=None, h0="input", stream=None):
    q = d["q"] if q is None else q
    k = d["k"] if k is None else k
    v = d["v"] if v is None else v
    h0 = d["h0"] if isinstance(h0, str) else h0
    return kda.chunk_fwd(q, k, v, d["g"], d["beta"], d["scale"], h0=h0,
                         cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], stream=stream)


def run_conv(d, conv_state=None):
    return kda.conv_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["w_q"], d["w_k"], d["w_v"],
                        conv_state=conv_state, cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])
