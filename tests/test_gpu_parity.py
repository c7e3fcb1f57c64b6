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
from conftest import rel_l2
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
@pytest.mark.parametrize("d_head", [64, 128])
def test_chunk_varlen_ragged(io, d_head):
    lens = [1, 63, 64, 65, 0, 130, 7, 200]
    wl = small("prefill_8k", N=len(lens), H=3, dk=d_head, dv=d_head, io=io, h0_std=0.02, seed=31)
    d = make_prefill(wl, DEV, lengths=lens)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


@pytest.mark.parametrize("variant", ["cluster", "single"])
@pytest.mark.parametrize("lens", [[300, 1, 64], [129, 700]])
def test_chunk_extreme_decay_takes_exact_path(variant, lens, monkeypatch):
    """Channels decaying by ~e^-4 per token push the half-chunk decay far past e^-80, so
    those chunks form A and P exactly on CUDA cores; the result must still match."""
    monkeypatch.setenv("KDA_CHUNK_KERNEL", variant)
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


@pytest.mark.parametrize("variant", ["cluster", "single"])
def test_chunk_variants_match_oracle(variant, monkeypatch):
    monkeypatch.setenv("KDA_CHUNK_KERNEL", variant)
    lens = [1, 63, 64, 65, 0, 130, 7, 200, 1000]
    wl = small("prefill_8k", N=len(lens), H=3, io="bf16", h0_std=0.02, seed=38)
    d = make_prefill(wl, DEV, lengths=lens)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


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
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)


def test_varlen_prologue_full():
    """64 packed sequences (lengths U[128,16384]) through conv+SiLU+L2 then chunked prefill.
    The oracle checks the prologue on every token of three sequences and the recurrence
    on two heads of the shortest, a middle and the longest sequence."""
    wl = WORKLOADS["varlen_prologue"]
    d = make_prefill(wl, DEV)
    q, k, v = run_conv(d)
    o, ht = run_chunk(d, q, k, v)
    torch.cuda.synchronize()
    lens = np.array(d["lengths"])
    order = np.argsort(lens)
    seqs = [int(order[0]), int(order[len(order) // 2]), int(order[-1])]
    cu = d["cu_host"]
    for n in seqs:
        sl = slice(cu[n], cu[n + 1])
        sub = {nm: d[nm][sl] for nm in ("q_raw", "k_raw", "v_raw")}
        sub.update(w_q=d["w_q"], w_k=d["w_k"], w_v=d["w_v"], cu_host=[0, cu[n + 1] - cu[n]])
        qr, kr, vr, _ = oracle.prologue(to64(sub["q_raw"]), to64(sub["k_raw"]), to64(sub["v_raw"]),
                                        to64(d["w_q"]), to64(d["w_k"]), to64(d["w_v"]), None,
                                        sub["cu_host"], 1e-6)
        for got, ref in ((q[sl], qr), (k[sl], kr), (v[sl], vr)):
            assert rel_l2(to64(got), ref) <= TOL_BF16
    heads = [0, 31]
    check_prefill(d, q, k, v, o, ht, pairs=[(n, h) for n in seqs for h in heads])


def test_long_context_skewed_gates_seeded_heads():
    """B=1, H=32, T=262144, skewed gates; the oracle checks 4 seeded heads."""
    wl = WORKLOADS["long_256k"]
    d = make_prefill(wl, DEV)
    o, ht = run_chunk(d)
    torch.cuda.synchronize()
    heads = sorted(np.random.default_rng(wl.seed).choice(wl.H, 4, replace=False).tolist())
    check_prefill(d, d["q"], d["k"], d["v"], o, ht, pairs=[(0, h) for h in heads])


def test_decode_full_sampled_pairs():
    """256 sequences x 32 heads, 1024 steps of conv (cache of width 3) + recurrent step.
    Checked against the oracle on 8 seeded (sequence, head) pairs over all steps."""
    wl = WORKLOADS["decode_256x32"]
    d = make_decode(wl, DEV)
    N, H, steps = wl.N, wl.H, wl.steps
    rng = np.random.default_rng(wl.seed)
    pairs = [(int(rng.integers(N)), int(rng.integers(H))) for _ in range(8)]
    ns = torch.tensor([p[0] for p in pairs], device=DEV)
    hs = torch.tensor([p[1] for p in pairs], device=DEV)
    state = d["h0"].clone()
    h0_pairs = to64(d["h0"][ns, hs])
    cache = d["conv_state"].clone()
    rec = {nm: [] for nm in ("q", "k", "v", "o")}
    for s in range(steps):
        x = [d[nm][s].unsqueeze(1) for nm in ("q_raw", "k_raw", "v_raw")]
        q, k, v = kda.conv_fwd(*x, d["w_q"], d["w_k"], d["w_v"], conv_state=cache)
        q, k, v = q[:, 0], k[:, 0], v[:, 0]
        o = kda.recurrent_step(q, k, v, d["g"][s], d["beta"][s], state)
        for nm, t in (("q", q), ("k", k), ("v", v), ("o", o)):
            rec[nm].append(t[ns, hs])
    torch.cuda.synchronize()
    rec = {nm: to64(torch.stack(ts)) for nm, ts in rec.items()}     # [steps, 8, d]
    g = to64(d["g"][:, ns, hs])
    beta = to64(d["beta"][:, ns, hs])
    o_ref, S_ref = oracle.kda_fwd(rec["q"], rec["k"], rec["v"], g, beta, 1.0,
                                  h0_pairs[None], None)
    assert rel_l2(rec["o"], o_ref) <= TOL_BF16
    assert rel_l2(to64(state[ns, hs]), S_ref[0]) <= TOL_BF16


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
