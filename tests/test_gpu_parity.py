"""GPU parity: libkda (through its C ABI) against the fp64 oracle on seeded inputs.

Tolerances (relative L2 over the whole tensor, in fp64): 1e-4 for fp32 I/O and
1e-2 for bf16 I/O with fp32 gates, beta and state, on outputs and final states.
The oracle always reads back the exact bytes the GPU consumed.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from conftest import record_margin, rel_l2
from gpu_helpers import TOL_BF16, check_prefill, run_chunk, run_conv, to64, tol_for
from kimi_delta_attention_32_b200 import kda
from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_decode, make_prefill

pytestmark = pytest.mark.gpu

DEV = "cuda"


def small(name, **kw):
    return dataclasses.replace(WORKLOADS[name], **kw)


# --------------------------------------------------------------------------- #
# Decode step                                                                  #
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_recurrent_step_chain_matches_oracle(io, dk, dv):
    wl = small("decode_256x32", N=3, H=2, dk=dk, dv=dv, io=io, steps=6, seed=11)
    d = make_decode(wl, DEV)
    state = d["h0"].clone()
    S = to64(d["h0"])
    outs, refs = [], []
    for s in range(d["steps"]):
        q = torch.nn.functional.normalize(d["q_raw"][s].float(), dim=-1).to(d["q_raw"].dtype)
        k = torch.nn.functional.normalize(d["k_raw"][s].float(), dim=-1).to(d["k_raw"].dtype)
        v = d["v_raw"][s]
        g, beta = d["g"][s], d["beta"][s]
        o = kda.recurrent_step(q, k, v, g, beta, state, scale=0.8)
        cu = list(range(wl.N + 1))
        o_ref, S = oracle.kda_fwd(to64(q).reshape(wl.N, wl.H, dk), to64(k), to64(v), to64(g),
                                  to64(beta), 0.8, S, cu)
        outs.append(to64(o))
        refs.append(o_ref)
    torch.cuda.synchronize()
    tol = tol_for(io)
    assert rel_l2(np.stack(outs), np.stack(refs)) <= tol
    assert rel_l2(to64(state), S) <= tol


def _oracle_decode_chain(d, steps, scale=1.0):
    """fp64 oracle of the fused decode: per step, the prologue (conv with the carried cache,
    SiLU, L2) on the raw inputs, then one token of the recurrence. Returns (o [steps, N, H, dv],
    final state [N, H, dk, dv], final conv cache)."""
    N, H, dk, dv = d["N"], d["H"], d["dk"], d["dv"]
    cu = list(range(N + 1))
    cache = to64(d["conv_state"])
    S = to64(d["h0"])
    outs = []
    for s in range(steps):
        q, k, v, cache = oracle.prologue(to64(d["q_raw"][s]), to64(d["k_raw"][s]),
                                         to64(d["v_raw"][s]), to64(d["w_q"]), to64(d["w_k"]),
                                         to64(d["w_v"]), cache, cu, 1e-6)
        o, S = oracle.kda_fwd(q, k, v, to64(d["g"][s]), to64(d["beta"][s]), scale, S, cu)
        outs.append(o)
    return np.stack(outs), S, cache


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_conv_recurrent_step_chain_matches_oracle(io, dk, dv):
    """The fused decode (conv cache advanced in place + SiLU + L2 + state update in one kernel)
    against the fp64 oracle run on the raw inputs, over a chain of steps."""
    wl = small("decode_256x32", N=3, H=2, dk=dk, dv=dv, io=io, steps=6, seed=12)
    d = make_decode(wl, DEV)
    d["conv_state"] = torch.randn(d["conv_state"].shape, device=DEV).to(d["conv_state"].dtype)
    cache0 = d["conv_state"].clone()
    state = d["h0"].clone()
    cache = d["conv_state"].clone()
    outs = [kda.conv_recurrent_step(d["q_raw"][s], d["k_raw"][s], d["v_raw"][s], d["w_q"], d["w_k"],
                                    d["w_v"], cache, d["g"][s], d["beta"][s], state, scale=0.8)
            for s in range(d["steps"])]
    torch.cuda.synchronize()
    d["conv_state"] = cache0
    o_ref, S_ref, c_ref = _oracle_decode_chain(d, d["steps"], scale=0.8)
    tol = tol_for(io)
    assert rel_l2(to64(torch.stack(outs)), o_ref) <= tol
    assert rel_l2(to64(state), S_ref) <= tol
    assert np.array_equal(to64(cache), c_ref)             # the cache holds raw inputs: exact


def test_conv_recurrent_step_cache_equals_unfused_pair():
    """The fused kernel advances the conv cache exactly as kda_conv_fwd in decode form does."""
    wl = small("decode_256x32", N=5, H=3, steps=4, seed=13)
    d = make_decode(wl, DEV)
    c_fused, c_pair = d["conv_state"].clone(), d["conv_state"].clone()
    s_fused, s_pair = d["h0"].clone(), d["h0"].clone()
    for s in range(d["steps"]):
        x = [d[nm][s] for nm in ("q_raw", "k_raw", "v_raw")]
        kda.conv_recurrent_step(*x, d["w_q"], d["w_k"], d["w_v"], c_fused, d["g"][s], d["beta"][s],
                                s_fused)
        q, k, v = kda.conv_fwd(*[t.unsqueeze(1) for t in x], d["w_q"], d["w_k"], d["w_v"],
                               conv_state=c_pair)
        kda.recurrent_step(q[:, 0], k[:, 0], v[:, 0], d["g"][s], d["beta"][s], s_pair)
    torch.cuda.synchronize()
    torch.testing.assert_close(c_fused, c_pair, rtol=0, atol=0)
    assert rel_l2(to64(s_fused), to64(s_pair)) <= TOL_BF16


def _oracle_fused_chain(d, steps, norm, scale=1.0):
    """fp64 oracle of the whole decode step from raw projections: prologue, gate and beta from
    their logits, one token of the recurrence, then (norm) the gated RMSNorm of the output."""
    N, H, dk, dv = d["N"], d["H"], d["dk"], d["dv"]
    cu = list(range(N + 1))
    cache, S = to64(d["conv_state"]), to64(d["h0"])
    outs = []
    for s in range(steps):
        q, k, v, cache = oracle.prologue(to64(d["q_raw"][s]), to64(d["k_raw"][s]),
                                         to64(d["v_raw"][s]), to64(d["w_q"]), to64(d["w_k"]),
                                         to64(d["w_v"]), cache, cu, 1e-6)
        g = oracle.gate(to64(d["g_raw"][s]), to64(d["A_log"]), to64(d["dt_bias"]))
        beta = oracle.sigmoid(to64(d["beta_raw"][s]))
        o, S = oracle.kda_fwd(q, k, v, g, beta, scale, S, cu)
        if norm:
            o = oracle.gated_rmsnorm(o, to64(d["z"][s]), to64(d["w_norm"]), 1e-6)
        outs.append(o)
    return np.stack(outs), S, cache


def _run_fused_chain(d, steps, norm, scale=1.0):
    state, cache = d["h0"].clone(), d["conv_state"].clone()
    outs = [kda.fused_recurrent_step(d["q_raw"][s], d["k_raw"][s], d["v_raw"][s], d["g_raw"][s],
                                     d["beta_raw"][s], d["w_q"], d["w_k"], d["w_v"], cache,
                                     d["A_log"], d["dt_bias"], state,
                                     z=d["z"][s] if norm else None,
                                     w_norm=d["w_norm"] if norm else None, scale=scale)
            for s in range(steps)]
    torch.cuda.synchronize()
    return torch.stack(outs), state, cache


@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_fused_recurrent_step_chain_matches_oracle(io, dk, dv, norm):
    """The whole decode step from raw projections (conv, gate and beta from logits, state
    update, optional gated RMSNorm of the output) against the fp64 oracle's composition."""
    wl = small("decode_256x32", N=3, H=2, dk=dk, dv=dv, io=io, steps=6, seed=14)
    d = make_decode(wl, DEV)
    d["conv_state"] = torch.randn(d["conv_state"].shape, device=DEV).to(d["conv_state"].dtype)
    o, state, cache = _run_fused_chain(d, d["steps"], norm, scale=0.7)
    o_ref, S_ref, c_ref = _oracle_fused_chain(d, d["steps"], norm, scale=0.7)
    tol = tol_for(io)
    assert rel_l2(to64(o), o_ref) <= tol
    assert rel_l2(to64(state), S_ref) <= tol
    assert np.array_equal(to64(cache), c_ref)


def test_fused_recurrent_step_medium_all_pairs():
    """64 sequences x 32 heads x 64 steps of the fully fused decode step with the output norm,
    every (sequence, head) pair against the oracle (pooled and per-pair rel-L2)."""
    wl = small("decode_256x32", N=64, steps=64, seed=15)
    d = make_decode(wl, DEV)
    o, state, cache = _run_fused_chain(d, d["steps"], True)
    o_ref, S_ref, c_ref = _oracle_fused_chain(d, d["steps"], True)
    N, H = wl.N, wl.H
    po, ps = _PerUnit(N * H), _PerUnit(N * H)
    po.add(np.arange(N * H), to64(o).reshape(wl.steps, N * H, -1), o_ref.reshape(wl.steps, N * H, -1))
    ps.add(np.arange(N * H), to64(state).reshape(1, N * H, -1), S_ref.reshape(1, N * H, -1))
    assert np.array_equal(to64(cache), c_ref)
    name = "fused decode 64x32x64 (gate, norm)"
    for nm, acc in (("o", po), ("final state", ps)):
        record_margin(name, f"{nm} pooled", acc.pooled(), TOL_BF16)
        record_margin(name, f"{nm} worst pair", acc.worst(), TOL_BF16)
        assert acc.pooled() <= TOL_BF16 and acc.worst() <= TOL_BF16


# --------------------------------------------------------------------------- #
# Conv prologue                                                                #
# --------------------------------------------------------------------------- #

def _oracle_prologue(d, conv_state):
    return oracle.prologue(to64(d["q_raw"]), to64(d["k_raw"]), to64(d["v_raw"]), to64(d["w_q"]),
                           to64(d["w_k"]), to64(d["w_v"]), to64(conv_state), d["cu_host"], 1e-6)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("with_cache", [False, True])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_conv_prefill_matches_oracle(io, with_cache, dk, dv):
    lens = [1, 2, 17, 40, 0, 3, 33]
    wl = small("varlen_prologue", N=len(lens), H=3, dk=dk, dv=dv, io=io, seed=21)
    d = make_prefill(wl, DEV, lengths=lens)
    cs = None
    if with_cache:
        cs = torch.randn((len(lens), 3 * (2 * dk + dv), 3), device=DEV).to(d["q_raw"].dtype)
    cs_in = None if cs is None else cs.clone()
    q, k, v = run_conv(d, cs)
    torch.cuda.synchronize()
    qr, kr, vr, cso = _oracle_prologue(d, cs_in if cs_in is not None else
                                       torch.zeros((len(lens), 3 * (2 * dk + dv), 3)))
    tol = tol_for(io) if io == "bf16" else 1e-5
    for got, ref in ((q, qr), (k, kr), (v, vr)):
        assert rel_l2(to64(got), ref) <= tol
    if with_cache:
        # the cache holds raw inputs: it must be exact
        assert np.array_equal(to64(cs), cso.astype(np.float64))


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_step_mode_equals_sequence_conv(io):
    """Decode form (padded, T == 1): token-by-token with the cache = the whole-sequence conv."""
    T, N, H, dk, dv = 7, 5, 2, 128, 128
    wl = small("varlen_prologue", N=N, H=H, dk=dk, dv=dv, io=io, seed=22)
    d = make_prefill(wl, DEV, lengths=[T] * N)
    q_full, k_full, v_full = run_conv(d, None)
    cache = torch.zeros((N, H * (2 * dk + dv), 3), device=DEV, dtype=d["q_raw"].dtype)
    for t in range(T):
        rows = [n * T + t for n in range(N)]
        x = [d[nm][rows].reshape(N, 1, H, -1).contiguous() for nm in ("q_raw", "k_raw", "v_raw")]
        qs, ks, vs = kda.conv_fwd(*x, d["w_q"], d["w_k"], d["w_v"], conv_state=cache)
        for got, full in ((qs, q_full), (ks, k_full), (vs, v_full)):
            torch.testing.assert_close(got.reshape(N, H, -1), full[rows], rtol=0, atol=0)
    q_p = torch.empty_like(q_full)
    cache_p = torch.zeros_like(cache)
    kda.conv_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["w_q"], d["w_k"], d["w_v"],
                 conv_state=cache_p, cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], q_out=q_p)
    torch.testing.assert_close(cache, cache_p, rtol=0, atol=0)


# --------------------------------------------------------------------------- #
# Chunked prefill                                                              #
# --------------------------------------------------------------------------- #

def test_chunk_tiny_fp32():
    """B=1, H=2, T=256, dk=dv=64, fp32 I/O, chunk 64, zero initial state."""
    d = make_prefill(WORKLOADS["tiny_fp32"], DEV)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_chunk_varlen_ragged(io, dk, dv):
    lens = [1, 63, 64, 65, 0, 130, 7, 200]
    wl = small("prefill_8k", N=len(lens), H=3, dk=dk, dv=dv, io=io, h0_std=0.02, seed=31)
    d = make_prefill(wl, DEV, lengths=lens)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


@pytest.mark.parametrize("lens", [[300, 1, 64], [129, 700]])
def test_chunk_extreme_decay_takes_exact_path(lens):
    """Channels decaying by ~e^-4 per token push the half-chunk decay far past e^-80, so
    those chunks form A and P exactly on CUDA cores; the result must still match."""
    wl = small("prefill_8k", N=len(lens), H=2, io="bf16", h0_std=0.02, seed=36)
    d = make_prefill(wl, DEV, lengths=lens)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(37)
    u = torch.randn(d["g"].shape, generator=gen, device=DEV) - 4.0
    strong = torch.nn.functional.logsigmoid(u)
    d["g"][:, :, :16] = strong[:, :, :16]          # 16 of 128 channels per head
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


def test_chunk_ragged_long_and_empty_sequences_match_oracle():
    lens = [1, 63, 64, 65, 0, 130, 7, 200, 1000]
    wl = small("prefill_8k", N=len(lens), H=3, io="bf16", h0_std=0.02, seed=38)
    d = make_prefill(wl, DEV, lengths=lens)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


def _oracle_gated_prefill(d, norm, scale=1.0):
    g = oracle.gate(to64(d["g_raw"]), to64(d["A_log"]), to64(d["dt_bias"]))
    beta = oracle.sigmoid(to64(d["beta_raw"]))
    o, ht = oracle.kda_fwd(to64(d["q"]), to64(d["k"]), to64(d["v"]), g, beta, scale,
                           to64(d["h0"]), d["cu_host"])
    if norm:
        o = oracle.gated_rmsnorm(o, to64(d["z"]), to64(d["w_norm"]), 1e-6)
    return o, ht


def _run_gated(d, norm, scale=1.0):
    return kda.chunk_fwd_fused(d["q"], d["k"], d["v"], g_raw=d["g_raw"], beta_raw=d["beta_raw"],
                               A_log=d["A_log"], dt_bias=d["dt_bias"], z=d["z"] if norm else None,
                               w_norm=d["w_norm"] if norm else None, scale=scale, h0=d["h0"],
                               cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])


@pytest.mark.parametrize("norm", [False, True])
def test_chunk_gated_matches_oracle(norm):
    """Prefill with g and beta from raw logits (and the gated RMSNorm of the output) against the
    oracle's gate, sigmoid, token loop and gated RMSNorm, on ragged packed sequences."""
    lens = [1, 63, 64, 65, 0, 130, 7, 200, 700]
    wl = small("prefill_8k", N=len(lens), H=3, io="bf16", h0_std=0.02, seed=51)
    d = make_prefill(wl, DEV, lengths=lens, raw=True)
    o, ht = _run_gated(d, norm, scale=0.9)
    torch.cuda.synchronize()
    assert kda.last_device_error() == kda.KDA_OK
    o_ref, h_ref = _oracle_gated_prefill(d, norm, scale=0.9)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16
    assert rel_l2(to64(ht), h_ref) <= TOL_BF16


def test_chunk_gated_strong_gates_take_exact_path():
    """Raw gate logits near 4 on 16 channels give g near -4 per token, so every chunk fails the
    range test and forms A and P exactly (the exact path recomputes g from the raw logits)."""
    lens = [300, 129]
    wl = small("prefill_8k", N=len(lens), H=2, io="bf16", h0_std=0.02, seed=52)
    d = make_prefill(wl, DEV, lengths=lens, raw=True)
    d["g_raw"][:, :, :16] = (torch.randn_like(d["g_raw"][:, :, :16].float()) * 0.3 + 4.0).to(torch.bfloat16)
    o, ht = _run_gated(d, True)
    torch.cuda.synchronize()
    assert kda.last_device_error() == kda.KDA_OK
    o_ref, h_ref = _oracle_gated_prefill(d, True)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16
    assert rel_l2(to64(ht), h_ref) <= TOL_BF16


def test_chunk_gated_prefill_8k_full():
    """prefill_8k shape from raw gate and beta logits with the output norm: all 32 heads."""
    d = make_prefill(WORKLOADS["prefill_8k"], DEV, raw=True)
    o, ht = _run_gated(d, True)
    torch.cuda.synchronize()
    o_ref, h_ref = _oracle_gated_prefill(d, True)
    eo, eh = rel_l2(to64(o), o_ref), rel_l2(to64(ht), h_ref)
    record_margin("prefill_8k gated (gate, norm)", "o pooled", eo, TOL_BF16)
    record_margin("prefill_8k gated (gate, norm)", "ht pooled", eh, TOL_BF16)
    assert eo <= TOL_BF16 and eh <= TOL_BF16


def _oracle_conv_prefill(d, conv_state=None, gate=False, norm=False, scale=1.0):
    """fp64 oracle of the fused prefill: the prologue on the raw inputs (with the conv history),
    the gate and beta (from raw logits when gate), the token loop, the optional gated RMSNorm."""
    q, k, v, cache = oracle.prologue(to64(d["q_raw"]), to64(d["k_raw"]), to64(d["v_raw"]),
                                     to64(d["w_q"]), to64(d["w_k"]), to64(d["w_v"]),
                                     None if conv_state is None else to64(conv_state),
                                     d["cu_host"], 1e-6)
    if gate:
        g = oracle.gate(to64(d["g_raw"]), to64(d["A_log"]), to64(d["dt_bias"]))
        beta = oracle.sigmoid(to64(d["beta_raw"]))
    else:
        g, beta = to64(d["g"]), to64(d["beta"])
    o, ht = oracle.kda_fwd(q, k, v, g, beta, scale, to64(d["h0"]), d["cu_host"])
    if norm:
        o = oracle.gated_rmsnorm(o, to64(d["z"]), to64(d["w_norm"]), 1e-6)
    return o, ht, cache


def _run_conv_prefill(d, conv_state=None, gate=False, norm=False, scale=1.0):
    kw = dict(g_raw=d["g_raw"], beta_raw=d["beta_raw"], A_log=d["A_log"],
              dt_bias=d["dt_bias"]) if gate else dict(g=d["g"], beta=d["beta"])
    if norm:
        kw.update(z=d["z"], w_norm=d["w_norm"])
    return kda.chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v_raw"], w_q=d["w_q"], w_k=d["w_k"],
                               w_v=d["w_v"], conv_state=conv_state, scale=scale, h0=d["h0"],
                               cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], **kw)


@pytest.mark.parametrize("with_cache", [False, True])
def test_chunk_conv_prologue_fused_matches_oracle(with_cache):
    """Raw q, k, v through the conv prologue in the producers' load stage (3-token halo, the
    history from the conv cache or zero), on ragged packed sequences; the cache is advanced."""
    lens = [1, 2, 3, 63, 64, 65, 0, 130, 200, 700]
    wl = small("varlen_prologue", N=len(lens), H=3, seed=53)
    d = make_prefill(wl, DEV, lengths=lens)
    cs = None
    if with_cache:
        cs = torch.randn((len(lens), 3 * 384, 3), device=DEV).to(torch.bfloat16)
    cs_in = None if cs is None else cs.clone()
    o, ht = _run_conv_prefill(d, cs, scale=0.9)
    torch.cuda.synchronize()
    assert kda.last_device_error() == kda.KDA_OK
    o_ref, h_ref, c_ref = _oracle_conv_prefill(d, cs_in, scale=0.9)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16
    assert rel_l2(to64(ht), h_ref) <= TOL_BF16
    if with_cache:
        assert np.array_equal(to64(cs), c_ref)             # the cache holds raw inputs: exact


def test_chunk_fully_fused_layer_matches_oracle():
    """Conv prologue, gate and beta from raw logits, and the output norm, all in the prefill."""
    lens = [5, 64, 129, 300]
    wl = small("varlen_prologue", N=len(lens), H=2, seed=54)
    d = make_prefill(wl, DEV, lengths=lens, raw=True)
    o, ht = _run_conv_prefill(d, gate=True, norm=True)
    torch.cuda.synchronize()
    assert kda.last_device_error() == kda.KDA_OK
    o_ref, h_ref, _ = _oracle_conv_prefill(d, gate=True, norm=True)
    assert rel_l2(to64(o), o_ref) <= TOL_BF16
    assert rel_l2(to64(ht), h_ref) <= TOL_BF16


def test_varlen_prologue_fused_full():
    """varlen_prologue as its config states: raw q/k/v of 64 packed sequences through the prefill
    with the conv prologue fused in, at full size. Every head of 12 sequences (the 4 shortest,
    the 4 longest and 4 seeded others) against the oracle run on the raw inputs; pooled and
    per-unit rel-L2. (test_varlen_prologue_full checks every unit of the unfused path.)"""
    wl = WORKLOADS["varlen_prologue"]
    d = make_prefill(wl, DEV)
    o, ht = _run_conv_prefill(d)
    torch.cuda.synchronize()
    assert kda.last_device_error() == kda.KDA_OK
    cu, N, H = d["cu_host"], d["N"], d["H"]
    order = np.argsort(np.array(d["lengths"]))
    rest = [int(x) for x in order[4:-4]]
    seqs = sorted(set([int(x) for x in order[:4]] + [int(x) for x in order[-4:]] +
                      list(np.random.default_rng(wl.seed).choice(rest, 4, replace=False))))
    po, ph = _PerUnit(N * H), _PerUnit(N * H)
    for n in seqs:
        sl = slice(cu[n], cu[n + 1])
        q, k, v, _ = oracle.prologue(to64(d["q_raw"][sl]), to64(d["k_raw"][sl]), to64(d["v_raw"][sl]),
                                     to64(d["w_q"]), to64(d["w_k"]), to64(d["w_v"]), None,
                                     [0, cu[n + 1] - cu[n]], 1e-6)
        o_ref, h_ref = oracle.kda_fwd(q, k, v, to64(d["g"][sl]), to64(d["beta"][sl]), 1.0,
                                      to64(d["h0"][n:n + 1]), None)
        units = [n * H + h for h in range(H)]
        po.add(units, to64(o[sl]), o_ref)
        ph.add(units, to64(ht[n]).reshape(1, H, -1), h_ref.reshape(1, H, -1))
    name = "varlen_prologue fused (12 seq x 32 heads)"
    for nm, acc in (("o", po), ("ht", ph)):
        record_margin(name, f"{nm} pooled", acc.pooled(), TOL_BF16)
        record_margin(name, f"{nm} worst unit", acc.worst(), TOL_BF16)
        assert acc.pooled() <= TOL_BF16 and acc.worst() <= TOL_BF16


def test_chunk_padded_equals_packed():
    wl = small("prefill_8k", N=3, H=2, T=100, io="bf16", h0_std=0.02, seed=32)
    d = make_prefill(wl, DEV)
    o_packed, ht_packed = run_chunk(d)
    B, T, H = 3, 100, 2
    o_pad, ht_pad = kda.chunk_fwd(d["q"].view(B, T, H, -1), d["k"].view(B, T, H, -1),
                                  d["v"].view(B, T, H, -1), d["g"], d["beta"], h0=d["h0"])
    torch.testing.assert_close(o_pad.view_as(o_packed), o_packed, rtol=0, atol=0)
    torch.testing.assert_close(ht_pad, ht_packed, rtol=0, atol=0)


def test_chunk_split_resume_and_inplace_state():
    """run(T1) then run(T2, h0 = ht) matches run(T1 + T2); ht may alias h0."""
    wl = small("prefill_8k", N=1, H=4, T=300, io="bf16", h0_std=0.02, seed=33)
    d = make_prefill(wl, DEV)
    o_all, ht_all = run_chunk(d)
    T1 = 128
    part = lambda x, a, b: x[a:b].contiguous()     # noqa: E731
    st = d["h0"].clone()
    o1, _ = kda.chunk_fwd(part(d["q"], 0, T1), part(d["k"], 0, T1), part(d["v"], 0, T1),
                          part(d["g"], 0, T1), part(d["beta"], 0, T1), h0=st, ht=st)
    o2, _ = kda.chunk_fwd(part(d["q"], T1, 300), part(d["k"], T1, 300), part(d["v"], T1, 300),
                          part(d["g"], T1, 300), part(d["beta"], T1, 300), h0=st, ht=st)
    torch.cuda.synchronize()
    assert rel_l2(to64(torch.cat([o1, o2])), to64(o_all)) <= 1e-3
    assert rel_l2(to64(st), to64(ht_all)) <= 1e-4


def test_decode_loop_equals_prefill():
    wl = small("prefill_8k", N=2, H=2, T=70, io="f32", h0_std=0.02, seed=34)
    d = make_prefill(wl, DEV)
    o_pre, ht_pre = run_chunk(d)
    state = d["h0"].clone()
    outs = []
    for t in range(70):
        rows = [n * 70 + t for n in range(2)]
        outs.append(kda.recurrent_step(d["q"][rows], d["k"][rows], d["v"][rows], d["g"][rows],
                                       d["beta"][rows], state))
    o_dec = torch.stack(outs, 1).reshape(-1, 2, 128)
    torch.cuda.synchronize()
    assert rel_l2(to64(o_dec), to64(o_pre)) <= 1e-5
    assert rel_l2(to64(state), to64(ht_pre)) <= 1e-5


def test_chunk_prefill_8k_full():
    """B=1, H=32, T=8192, dk=dv=128, bf16 I/O, every head against the oracle."""
    d = make_prefill(WORKLOADS["prefill_8k"], DEV)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    eo, eh = check_prefill(d, d["q"], d["k"], d["v"], o, ht)
    record_margin("prefill_8k (all 32 heads)", "o pooled", eo, TOL_BF16)
    record_margin("prefill_8k (all 32 heads)", "ht pooled", eh, TOL_BF16)


class _PerUnit:
    """Accumulates squared errors per unit (sequence, head) for pooled and per-unit rel-L2."""

    def __init__(self, n_units):
        self.num = np.zeros(n_units)
        self.den = np.zeros(n_units)

    def add(self, units, got, ref):
        """got, ref: arrays shaped [rows, len(units), d]; `units` indexes the unit axis."""
        diff = (got - ref) ** 2
        self.num[units] += diff.sum(axis=(0, 2))
        self.den[units] += (ref ** 2).sum(axis=(0, 2))

    def pooled(self):
        return float(np.sqrt(self.num.sum() / self.den.sum()))

    def worst(self):
        seen = self.den > 0
        return float(np.max(np.sqrt(self.num[seen] / self.den[seen]))) if seen.any() else 0.0


def test_varlen_prologue_full():
    """64 packed sequences (lengths U[128,16384]) through conv+SiLU+L2 then chunked prefill.
    Every sequence's prologue and every (sequence, head) unit of the recurrence is checked
    against the oracle, streamed one sequence at a time; pooled and per-unit rel-L2."""
    wl = WORKLOADS["varlen_prologue"]
    d = make_prefill(wl, DEV)
    q, k, v = run_conv(d)
    o, ht = run_chunk(d, q, k, v)
    torch.cuda.synchronize()
    cu, N, H = d["cu_host"], d["N"], d["H"]
    pro = [_PerUnit(N) for _ in range(3)]
    po, ph = _PerUnit(N * H), _PerUnit(N * H)
    for n in range(N):
        sl = slice(cu[n], cu[n + 1])
        refs = oracle.prologue(to64(d["q_raw"][sl]), to64(d["k_raw"][sl]), to64(d["v_raw"][sl]),
                               to64(d["w_q"]), to64(d["w_k"]), to64(d["w_v"]), None,
                               [0, cu[n + 1] - cu[n]], 1e-6)
        for acc, got, ref in zip(pro, (q[sl], k[sl], v[sl]), refs[:3]):
            acc.add([n], to64(got).reshape(-1, 1, ref.shape[1] * ref.shape[2]),
                    ref.reshape(-1, 1, ref.shape[1] * ref.shape[2]))
        qs, ks, vs = to64(q[sl]), to64(k[sl]), to64(v[sl])
        o_ref, h_ref = oracle.kda_fwd(qs, ks, vs, to64(d["g"][sl]), to64(d["beta"][sl]), 1.0,
                                      to64(d["h0"][n:n + 1]), None)
        units = [n * H + h for h in range(H)]
        po.add(units, to64(o[sl]), o_ref)
        ph.add(units, to64(ht[n]).reshape(1, H, -1), h_ref.reshape(1, H, -1))
    name = "varlen_prologue (all 64 seq x 32 heads)"
    for nm, acc in zip("qkv", pro):
        record_margin(name, f"prologue {nm} worst sequence", acc.worst(), TOL_BF16)
        assert acc.pooled() <= TOL_BF16 and acc.worst() <= TOL_BF16
    for nm, acc in (("o", po), ("ht", ph)):
        record_margin(name, f"{nm} pooled", acc.pooled(), TOL_BF16)
        record_margin(name, f"{nm} worst unit", acc.worst(), TOL_BF16)
        assert acc.pooled() <= TOL_BF16, f"{nm} pooled rel-L2 {acc.pooled():.3e}"
        assert acc.worst() <= TOL_BF16, f"{nm} worst-unit rel-L2 {acc.worst():.3e}"


def test_long_context_skewed_gates_seeded_heads():
    """B=1, H=32, T=262144, skewed gates; the oracle checks 8 seeded heads."""
    wl = WORKLOADS["long_256k"]
    d = make_prefill(wl, DEV)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    heads = sorted(np.random.default_rng(wl.seed).choice(wl.H, 8, replace=False).tolist())
    eo, eh = check_prefill(d, d["q"], d["k"], d["v"], o, ht, pairs=[(0, h) for h in heads])
    record_margin("long_256k (8 seeded heads)", "o pooled", eo, TOL_BF16)
    record_margin("long_256k (8 seeded heads)", "ht pooled", eh, TOL_BF16)


def test_decode_full_all_pairs():
    """256 sequences x 32 heads, 1024 steps of conv (cache of width 3) + recurrent step.
    Every (sequence, head) pair is checked against the oracle over all steps: the oracle
    runs the recorded post-conv q/k/v in batches of 64 steps, carrying its fp64 states."""
    wl = WORKLOADS["decode_256x32"]
    d = make_decode(wl, DEV)
    N, H, steps, dk, dv = wl.N, wl.H, wl.steps, wl.dk, wl.dv
    state = d["h0"].clone()
    cache = d["conv_state"].clone()
    rec = {nm: torch.empty((steps, N, H, dk if nm != "v" and nm != "o" else dv),
                           dtype=torch.bfloat16, device=DEV) for nm in ("q", "k", "v", "o")}
    for s in range(steps):
        x = [d[nm][s].unsqueeze(1) for nm in ("q_raw", "k_raw", "v_raw")]
        q, k, v = kda.conv_fwd(*x, d["w_q"], d["w_k"], d["w_v"], conv_state=cache)
        q, k, v = q[:, 0], k[:, 0], v[:, 0]
        o = kda.recurrent_step(q, k, v, d["g"][s], d["beta"][s], state)
        for nm, t in (("q", q), ("k", k), ("v", v), ("o", o)):
            rec[nm][s].copy_(t)
    torch.cuda.synchronize()
    P = N * H
    S = to64(d["h0"]).reshape(P, 1, dk, dv)
    po = _PerUnit(P)
    batch = 64

    def packed(t, b0, b1):     # [steps, N, H, d] -> [P * steps_b, 1, d], pair-major
        x = t[b0:b1].permute(1, 2, 0, *range(3, t.dim())).reshape(P * (b1 - b0), 1, -1)
        return to64(x)
    for b0 in range(0, steps, batch):
        b1 = min(steps, b0 + batch)
        nb = b1 - b0
        cu = list(range(0, P * nb + 1, nb))
        beta = to64(d["beta"][b0:b1].permute(1, 2, 0).reshape(P * nb, 1))
        o_ref, S = oracle.kda_fwd(packed(rec["q"], b0, b1), packed(rec["k"], b0, b1),
                                  packed(rec["v"], b0, b1), packed(d["g"], b0, b1), beta, 1.0,
                                  S, cu)
        got = packed(rec["o"], b0, b1)
        po.add(np.arange(P), got.reshape(P, nb, dv).transpose(1, 0, 2),
               o_ref.reshape(P, nb, dv).transpose(1, 0, 2))
    ps = _PerUnit(P)
    ps.add(np.arange(P), to64(state).reshape(1, P, dk * dv), S.reshape(1, P, dk * dv))
    name = "decode_256x32 (all 8192 pairs, 1024 steps)"
    for nm, acc in (("o", po), ("final state", ps)):
        record_margin(name, f"{nm} pooled", acc.pooled(), TOL_BF16)
        record_margin(name, f"{nm} worst pair", acc.worst(), TOL_BF16)
        assert acc.pooled() <= TOL_BF16, f"{nm} pooled rel-L2 {acc.pooled():.3e}"
        assert acc.worst() <= TOL_BF16, f"{nm} worst-pair rel-L2 {acc.worst():.3e}"


def test_bounded_wait_timeout_is_reported_and_recoverable():
    """A short wait bound (~1 us) makes the prefill's cross-CTA hand-off waits give up before a
    producer has prepared a chunk: the call ends early with KDA_ERR_TIMEOUT reported by
    kda_last_device_error, its CTAs having drained their copies in flight, and the next call
    with the default bound matches the oracle."""
    wl = small("prefill_8k", N=2, H=2, T=700, io="bf16", h0_std=0.02, seed=41)
    d = make_prefill(wl, DEV)
    assert kda.last_device_error() == kda.KDA_OK
    kda.set_wait_limit(2000)
    try:
        run_chunk(d)
        status = kda.last_device_error()
    finally:
        kda.set_wait_limit(0)
    assert status == kda.KDA_ERR_TIMEOUT
    assert kda.last_device_error() == kda.KDA_OK          # read and cleared
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    assert kda.last_device_error() == kda.KDA_OK
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


def test_conv_recurrent_step_full_all_pairs():
    """decode_256x32 through the fused decode kernel: 256 sequences x 32 heads, 1024 steps, raw
    bf16 q/k/v with the width-3 conv cache carried. Every (sequence, head) pair is checked
    against the fp64 oracle (prologue on the raw inputs, then the recurrence) over all steps."""
    wl = WORKLOADS["decode_256x32"]
    d = make_decode(wl, DEV)
    N, H, steps, dk, dv = wl.N, wl.H, wl.steps, wl.dk, wl.dv
    state = d["h0"].clone()
    cache = d["conv_state"].clone()
    o_all = torch.empty((steps, N, H, dv), dtype=torch.bfloat16, device=DEV)
    for s in range(steps):
        kda.conv_recurrent_step(d["q_raw"][s], d["k_raw"][s], d["v_raw"][s], d["w_q"], d["w_k"],
                                d["w_v"], cache, d["g"][s], d["beta"][s], state, o=o_all[s])
    torch.cuda.synchronize()
    P = N * H
    cu1 = list(range(N + 1))
    ccache = to64(d["conv_state"])
    S = to64(d["h0"]).reshape(P, 1, dk, dv)
    po = _PerUnit(P)
    batch = 64
    for b0 in range(0, steps, batch):
        b1 = min(steps, b0 + batch)
        nb = b1 - b0
        qkv = []
        for s in range(b0, b1):
            q, k, v, ccache = oracle.prologue(to64(d["q_raw"][s]), to64(d["k_raw"][s]),
                                              to64(d["v_raw"][s]), to64(d["w_q"]), to64(d["w_k"]),
                                              to64(d["w_v"]), ccache, cu1, 1e-6)
            qkv.append((q, k, v))
        # [nb, N, H, d] -> [P * nb, 1, d], pair-major
        pk = [np.stack([x[i] for x in qkv]).transpose(1, 2, 0, 3).reshape(P * nb, 1, -1)
              for i in range(3)]
        g = to64(d["g"][b0:b1]).transpose(1, 2, 0, 3).reshape(P * nb, 1, dk)
        beta = to64(d["beta"][b0:b1]).transpose(1, 2, 0).reshape(P * nb, 1)
        o_ref, S = oracle.kda_fwd(pk[0], pk[1], pk[2], g, beta, 1.0, S,
                                  list(range(0, P * nb + 1, nb)))
        got = to64(o_all[b0:b1]).reshape(nb, P, dv)
        po.add(np.arange(P), got, o_ref.reshape(P, nb, dv).transpose(1, 0, 2))
    ps = _PerUnit(P)
    ps.add(np.arange(P), to64(state).reshape(1, P, dk * dv), S.reshape(1, P, dk * dv))
    assert np.array_equal(to64(cache), ccache)
    name = "decode_256x32 fused (all pairs, 1024 steps)"
    for nm, acc in (("o", po), ("final state", ps)):
        record_margin(name, f"{nm} pooled", acc.pooled(), TOL_BF16)
        record_margin(name, f"{nm} worst pair", acc.worst(), TOL_BF16)
        assert acc.pooled() <= TOL_BF16, f"{nm} pooled rel-L2 {acc.pooled():.3e}"
        assert acc.worst() <= TOL_BF16, f"{nm} worst-pair rel-L2 {acc.worst():.3e}"


def test_device_error_word_is_clear():
    d = make_prefill(small("prefill_8k", N=1, H=2, T=64, seed=35), DEV)
    run_chunk(d)
    assert kda.last_device_error() == kda.KDA_OK


@pytest.mark.parametrize("n_seq,max_len,scale", [(600, 70, 0.125), (40, 300, 2.0)])
def test_chunk_scale_and_many_sequences(n_seq, max_len, scale):
    """Output scale on the tensor-core path (applied when O leaves tensor memory), and more
    packed sequences than the kernel orders by length (it orders at most one per thread)."""
    rng = np.random.default_rng(n_seq)
    lens = [int(x) for x in rng.integers(0, max_len + 1, size=n_seq)]
    wl = small("prefill_8k", N=n_seq, H=2, io="bf16", h0_std=0.02, seed=39)
    d = make_prefill(wl, DEV, lengths=lens)
    d["scale"] = scale
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    assert kda.last_device_error() == kda.KDA_OK
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)
