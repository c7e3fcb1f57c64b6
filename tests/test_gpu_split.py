"""GPU parity of the split (context-parallel) prefill against the fp64 oracle: the end states
and transitions of stretches (kda_chunk_states), their join (kda_state_scan), and the prefill
that runs every sequence as stretches side by side (kda_chunk_fwd_split).

The transition of a stretch is the oracle's product of the per-token linear maps
(I - beta k k^T) diag(exp g); its end state from h0 is the oracle's final state. The split
prefill must match the oracle run over whole sequences within the bf16 bar (1e-2 rel-L2),
pooled and per (sequence, head).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from conftest import record_margin, rel_l2
from gpu_helpers import TOL_BF16, to64
from kimi_delta_attention_32_b200 import kda
from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(lens, H, seed, h0_std=0.02):
    wl = dataclasses.replace(WORKLOADS["prefill_8k"], N=len(lens), H=H, h0_std=h0_std, seed=seed)
    return make_prefill(wl, DEV, lengths=lens)


def _per_unit_worst(x, ref):
    """Largest rel-L2 over the leading (sequence, head) axes of [N, H, ...] arrays."""
    worst = 0.0
    for n in range(ref.shape[0]):
        for h in range(ref.shape[1]):
            if np.linalg.norm(ref[n, h]) > 0:
                worst = max(worst, rel_l2(x[n, h], ref[n, h]))
    return worst


def _per_unit_worst_o(o, ref, cu, H):
    worst = 0.0
    for n in range(len(cu) - 1):
        if cu[n + 1] == cu[n]:
            continue
        for h in range(H):
            worst = max(worst, rel_l2(o[cu[n]:cu[n + 1], h], ref[cu[n]:cu[n + 1], h]))
    return worst


def test_chunk_states_match_oracle():
    lens = [1, 63, 64, 65, 0, 130, 700]
    d = _inputs(lens, 3, 51)
    ht, m, o, w = kda.chunk_states(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.5, h0=d["h0"],
                                   cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], output=True,
                                   carried_queries=True)
    torch.cuda.synchronize()
    q64, k64, g64, b64 = to64(d["q"]), to64(d["k"]), to64(d["g"]), to64(d["beta"])
    o_ref, ht_ref = oracle.kda_fwd(q64, k64, to64(d["v"]), g64, b64, 0.5, to64(d["h0"]),
                                   d["cu_host"])
    m_ref = oracle.transition(k64, g64, b64, d["cu_host"])
    # w_t = scale M_t^T q_t: the output of the run with v = 0 started from the identity
    eye = np.broadcast_to(np.eye(128), (len(lens), 3, 128, 128))
    w_ref, _ = oracle.kda_fwd(q64, k64, np.zeros_like(q64), g64, b64, 0.5, eye, d["cu_host"])
    ht, m, o, w = to64(ht), to64(m), to64(o), to64(w)
    eh, em = _per_unit_worst(ht, ht_ref), _per_unit_worst(m, m_ref)
    eo = _per_unit_worst_o(o, o_ref, d["cu_host"], 3)
    ew = _per_unit_worst_o(w, w_ref, d["cu_host"], 3)
    label = "chunk_states (7 ragged seqs x 3 heads)"
    record_margin(label, "end state, worst unit", eh, TOL_BF16)
    record_margin(label, "output, worst unit", eo, TOL_BF16)
    record_margin(label, "transition, worst unit", em, TOL_BF16)
    record_margin(label, "carried queries, worst unit", ew, TOL_BF16)
    assert max(eh, em, eo, ew) <= TOL_BF16
    # an empty sequence: the identity, and the state it was given
    assert np.array_equal(m[4], np.broadcast_to(np.eye(128), (3, 128, 128)))
    assert np.array_equal(ht[4], to64(d["h0"][4]))


def test_chunk_states_end_state_only_equals_prefill_state():
    """Without transitions the launch forms the end states and outputs kda_chunk_fwd forms
    (same arithmetic)."""
    d = _inputs([500, 1, 129], 2, 52)
    ht, m, o, _ = kda.chunk_states(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                                   cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"],
                                   transition=False, output=True)
    o_ref, ht_ref = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 1.0, h0=d["h0"],
                                  cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])
    torch.cuda.synchronize()
    assert m is None
    assert rel_l2(to64(ht), to64(ht_ref)) <= 1e-6
    assert rel_l2(to64(o), to64(o_ref)) <= 1e-6


@pytest.mark.parametrize("dk,strides", [(128, "seq_major"), (128, "seg_major"), (64, "seq_major")])
def test_state_scan_matches_host_join(dk, strides):
    N, P, H, dv = 3, 4, 2, 128
    rng = np.random.default_rng(53)
    m = 0.6 * np.eye(dk) + rng.normal(0.0, 0.05, (N * P, H, dk, dk))
    z = rng.normal(0.0, 1.0, (N * P, H, dk, dv))
    h0 = rng.normal(0.0, 1.0, (N, H, dk, dv))
    sn, sp = (P, 1) if strides == "seq_major" else (1, N)
    t = lambda a: torch.tensor(a, dtype=torch.float32, device=DEV)
    hs, ht = kda.state_scan(t(m), t(z), t(h0), N=N, P=P, seq_stride=sn, seg_stride=sp)
    torch.cuda.synchronize()
    m32, z32 = to64(t(m)), to64(t(z))
    hs_ref = np.zeros_like(z)
    ht_ref = np.zeros_like(h0)
    for n in range(N):
        cur = to64(t(h0[n]))
        for p in range(P):
            j = n * sn + p * sp
            hs_ref[j] = cur
            cur = np.einsum("hij,hjc->hic", m32[j], cur) + z32[j]
        ht_ref[n] = cur
    assert rel_l2(to64(hs), hs_ref) < 1e-5
    assert rel_l2(to64(ht), ht_ref) < 1e-5


def _check_split(d, o, ht, label):
    o_ref, ht_ref = oracle.kda_fwd(to64(d["q"]), to64(d["k"]), to64(d["v"]), to64(d["g"]),
                                   to64(d["beta"]), d["scale"], to64(d["h0"]), d["cu_host"])
    o, ht = to64(o), to64(ht)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ht))
    eo, eh = rel_l2(o, o_ref), rel_l2(ht, ht_ref)
    wo = _per_unit_worst_o(o, o_ref, d["cu_host"], d["H"])
    wh = _per_unit_worst(ht, ht_ref)
    record_margin(label, "o pooled", eo, TOL_BF16)
    record_margin(label, "o worst unit", wo, TOL_BF16)
    record_margin(label, "ht worst unit", wh, TOL_BF16)
    assert max(eo, eh, wo, wh) <= TOL_BF16


@pytest.mark.parametrize("lens,n_split", [([1000], 4), ([300, 1, 64, 0, 777], 3), ([130], 7),
                                          ([8192], 0)])
def test_chunk_fwd_split_matches_oracle(lens, n_split):
    """Stretches of whole chunks with a ragged last one; sequences shorter than the stretch
    count (empty stretches), an empty sequence, and the automatic choice."""
    d = _inputs(lens, 2, 54)
    P, _ = kda.chunk_fwd_split_plan(d["q"], d["v"], d["cu_seqlens"], d["cu_host"], n_split)
    assert P == n_split or (n_split == 0 and P > 1)     # 2 heads leave the GPU idle: split
    o, ht = kda.chunk_fwd_split(d["q"], d["k"], d["v"], d["g"], d["beta"], 1.0, h0=d["h0"],
                                cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], n_split=n_split)
    torch.cuda.synchronize()
    _check_split(d, o, ht, f"chunk_fwd_split {lens} x 2 heads, {P} stretches")


def test_chunk_fwd_split_padded_scaled_and_one_stretch():
    """A padded batch with an output scale; n_split = 1 is kda_chunk_fwd bit for bit."""
    wl = dataclasses.replace(WORKLOADS["prefill_8k"], N=2, H=2, T=900, h0_std=0.02, seed=55)
    d = make_prefill(wl, DEV)
    q, k, v = (d[x].view(2, 900, 2, 128) for x in ("q", "k", "v"))
    g, beta = d["g"].view(2, 900, 2, 128), d["beta"].view(2, 900, 2)
    o, ht = kda.chunk_fwd_split(q, k, v, g, beta, 0.5, h0=d["h0"], n_split=5)
    o1, ht1 = kda.chunk_fwd_split(q, k, v, g, beta, 0.5, h0=d["h0"], n_split=1)
    o_ref, ht_ref = kda.chunk_fwd(q, k, v, g, beta, 0.5, h0=d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o_ref) and torch.equal(ht1, ht_ref)
    d["scale"] = 0.5
    _check_split(d, o.view(1800, 2, 128), ht, "chunk_fwd_split padded 2x900 x 2 heads, 5 stretches")


def test_long_256k_tp4_split_full():
    """B=1, H=8, T=262144 with skewed gates, split automatically; the oracle checks every head."""
    wl = WORKLOADS["long_256k_tp4"]
    d = make_prefill(wl, DEV)
    P, _ = kda.chunk_fwd_split_plan(d["q"], d["v"], d["cu_seqlens"], d["cu_host"], 0)
    assert P > 1
    o, ht = kda.chunk_fwd_split(d["q"], d["k"], d["v"], d["g"], d["beta"], 1.0,
                                cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])
    torch.cuda.synchronize()
    _check_split(d, o, ht, f"long_256k_tp4 (all 8 heads, {P} stretches)")


def test_output_correct_matches_host_product():
    """o[t] += h[n]^T w[t] per sequence, against an fp64 product of the same bf16 inputs. h is
    taken as two bf16 halves (16 mantissa bits: each product within 2^-16 of exact), and the
    sum is rounded once to bf16, so every element lies within
    2^-8 |ref| + 2^-14 sum_i |w_i h_ij| of the exact value (each term with a 2x-4x margin)."""
    lens = [1, 700, 0, 64, 1500]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    H = 3
    gen = torch.Generator(device=DEV)
    gen.manual_seed(56)
    w = torch.randn((cu[-1], H, 128), generator=gen, device=DEV).bfloat16()
    o = torch.randn((cu[-1], H, 128), generator=gen, device=DEV).bfloat16()
    h = torch.randn((len(lens), H, 128, 128), generator=gen, device=DEV) * 0.1
    ref = to64(o).copy()
    mag = np.zeros_like(ref)
    w64, h64 = to64(w), to64(h)
    for n in range(len(lens)):
        ref[cu[n]:cu[n + 1]] += np.einsum("thi,hic->thc", w64[cu[n]:cu[n + 1]], h64[n])
        mag[cu[n]:cu[n + 1]] = np.einsum("thi,hic->thc", np.abs(w64[cu[n]:cu[n + 1]]), np.abs(h64[n]))
    cu_t = torch.tensor(cu, dtype=torch.int32, device=DEV)
    kda.output_correct(w, h, o, cu_t, cu)
    torch.cuda.synchronize()
    excess = np.abs(to64(o) - ref) / (2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * mag)
    assert np.max(excess) <= 1.0, f"error {np.max(excess):.2f}x its bound"
    assert rel_l2(to64(o), ref) <= 2e-3


def test_cross_rank_steps_through_the_abi():
    """The cross-rank context-parallel steps on one GPU: two ranks' stretches (cut anywhere,
    not at chunk bounds, one of them empty for a sequence) run through kda_chunk_states,
    are stacked in the all-gather's order, joined by kda_state_scan with the rank-major index,
    and corrected by kda_output_correct; the assembled outputs and final states must match the
    whole-sequence oracle."""
    lens = [700, 130, 95]
    cuts = [300, 130, 1]                    # rank 0 takes the first cut tokens of each sequence
    d = _inputs(lens, 2, 57)
    cu = d["cu_host"]
    parts = []
    for r in range(2):
        idx = torch.cat([torch.arange(cu[n] + (0 if r == 0 else cuts[n]),
                                      cu[n] + (cuts[n] if r == 0 else lens[n]))
                         for n in range(len(lens))]).to(DEV)
        cu_r = [0]
        for n in range(len(lens)):
            cu_r.append(cu_r[-1] + (cuts[n] if r == 0 else lens[n] - cuts[n]))
        sl = {x: d[x].index_select(0, idx).contiguous() for x in ("q", "k", "v", "g", "beta")}
        cu_t = torch.tensor(cu_r, dtype=torch.int32, device=DEV)
        z, m, o, w = kda.chunk_states(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], 1.0,
                                      cu_seqlens=cu_t, cu_host=cu_r, output=True,
                                      carried_queries=True)
        parts.append((idx, cu_t, cu_r, z, m, o, w))
    N = len(lens)
    h_start, ht = kda.state_scan(torch.cat([p[4] for p in parts]), torch.cat([p[3] for p in parts]),
                                 d["h0"], N=N, P=2, seq_stride=1, seg_stride=N)
    o_full = torch.empty_like(d["v"])
    for r, (idx, cu_t, cu_r, z, m, o, w) in enumerate(parts):
        kda.output_correct(w, h_start[r * N:(r + 1) * N].contiguous(), o, cu_t, cu_r)
        o_full.index_copy_(0, idx, o)
    torch.cuda.synchronize()
    _check_split(d, o_full, ht, "cross-rank steps, 2 ranks x 3 seqs x 2 heads")


def test_chunk_fwd_cp_one_rank():
    """cp.chunk_fwd_cp through its libkda steps and an NCCL group of one rank."""
    import os
    import socket
    import torch.distributed as dist
    from kimi_delta_attention_32_b200 import cp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        d = _inputs([500, 64, 3], 2, 58)
        o, ht = cp.chunk_fwd_cp(d["q"], d["k"], d["v"], d["g"], d["beta"], 1.0, h0=d["h0"],
                                cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    _check_split(d, o, ht, "cp.chunk_fwd_cp, 1 rank x 3 seqs x 2 heads")
