"""Seeded synthetic inputs for the KDA workloads.

This module only draws random numbers with fixed seeds and arranges them in the
library's layouts. It holds none of the method's arithmetic, so both the CUDA
path's tests/benchmarks and the CPU oracle can consume what it makes.

Distributions (one reading of each workload, see the design notes):
  q, k   ~ N(0, 1), then divided by their per-head-vector L2 norm (in fp64) and
           rounded to the I/O dtype, unless the workload feeds raw inputs
           through the conv prologue;
  v      ~ N(0, 1);
  beta   = sigmoid(N(0, 1))                      (fp32, in (0, 1));
  g      = -softplus(-u) = log(sigmoid(u)),  u ~ N(4, 1)   (fp32, per key channel,
           so exp(g) is mostly in 0.9 .. 1.0);  the long-context workload skews
           13 of 128 channels per head to u ~ N(-1, 0.5) clamped <= -0.05
           (exp(g) < 0.5);
  h0     = 0, or N(0, 0.02) fp32 where the workload says so;
  conv weights ~ N(0, 0.5) fp32, shape [H*d, 4].
Raw projections for the fully fused entry points (their own generator, seed + 100, so the
fields above keep their values): gate logits g_raw = -u, u ~ N(4, 1), with A_log ~ N(0, 0.1)
per head and dt_bias ~ N(0, 0.1) per key channel (so -exp(A_log) softplus(g_raw + dt_bias)
follows the g recipe above); beta logits ~ N(0, 1); output-norm gate z ~ N(0, 1) and weight
w_norm ~ N(1, 0.1) [dv].
N(m, s) means mean m and standard deviation s.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    N: int                      # sequences
    H: int
    T: int                      # tokens per sequence (padded layouts), 0 if varlen
    dk: int
    dv: int
    chunk: int = 64
    io: str = "bf16"            # "f32" or "bf16" for q/k/v/o
    prologue: bool = False      # raw q/k/v pass through conv + SiLU + L2 norm
    h0_std: float = 0.0         # 0 -> zero initial state
    varlen: tuple = ()          # (min_len, max_len) uniform lengths
    skew_channels: int = 0      # channels per head with strong decay
    steps: int = 0              # decode steps (decode workload only)
    seed: int = 0
    notes: str = field(default="", compare=False)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", N=1, H=2, T=256, dk=64, dv=64, io="f32", seed=1000,
                          notes="B=1,H=2,T=256,dk=dv=64, fp32 I/O, zero h0"),
    "prefill_8k": Workload("prefill_8k", N=1, H=32, T=8192, dk=128, dv=128, io="bf16",
                           seed=1001, notes="B=1,H=32,T=8192,dk=dv=128, bf16 I/O, zero h0"),
    "varlen_prologue": Workload("varlen_prologue", N=64, H=32, T=0, dk=128, dv=128, io="bf16",
                                prologue=True, h0_std=0.02, varlen=(128, 16384), seed=1002,
                                notes="64 packed sequences, lengths U[128,16384], raw q/k/v "
                                      "through conv(k=4)+SiLU+L2, h0 ~ N(0,0.02)"),
    "decode_256x32": Workload("decode_256x32", N=256, H=32, T=1, dk=128, dv=128, io="bf16",
                              prologue=True, h0_std=0.02, steps=1024, seed=1003,
                              notes="256 sequences x 32 heads, fp32 state, 1024 decode steps "
                                    "with a width-3 conv cache"),
    "long_256k": Workload("long_256k", N=1, H=32, T=262144, dk=128, dv=128, io="bf16",
                          skew_channels=13, seed=1004,
                          notes="B=1,H=32,T=262144, 13/128 channels per head with exp(g)<0.5"),
    # one of four tensor-parallel GPUs (the 4-GPU serving set-up of the model card) holds 8 of
    # the 32 heads: too few (sequence, head) pairs to fill the GPU, the case the split prefill
    # serves
    "long_256k_tp4": Workload("long_256k_tp4", N=1, H=8, T=262144, dk=128, dv=128, io="bf16",
                              skew_channels=13, seed=1005,
                              notes="B=1,H=8,T=262144 (32 heads over 4 tensor-parallel GPUs), "
                                    "13/128 channels per head with exp(g)<0.5"),
}


def io_dtype(io: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[io]


def _gen(device, seed: int) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return gen


def varlen_lengths(wl: Workload) -> list[int]:
    """Seeded sequence lengths, uniform integers in [min_len, max_len] (CPU generator)."""
    lo, hi = wl.varlen
    gen = _gen("cpu", wl.seed + 7)
    return torch.randint(lo, hi + 1, (wl.N,), generator=gen).tolist()


def cu_seqlens_of(lengths: list[int]) -> list[int]:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return cu


def _randn(shape, gen, device, mean=0.0, std=1.0, dtype=torch.float32):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x.to(dtype)


def _unit_rows(shape, gen, device, dtype, block_rows=1 << 16):
    """N(0,1) vectors along the last axis divided by their L2 norm (in fp64), then rounded."""
    out = torch.empty(shape, device=device, dtype=dtype)
    flat = out.view(-1, shape[-1])
    for r0 in range(0, flat.shape[0], block_rows):
        r1 = min(flat.shape[0], r0 + block_rows)
        x = torch.randn((r1 - r0, shape[-1]), generator=gen, device=device,
                        dtype=torch.float32).double()
        x = x / x.norm(dim=-1, keepdim=True)
        flat[r0:r1] = x.to(dtype)
    return out


def _log_decay(shape, gen, device, skew_channels=0, head_axis=-2):
    """g = log(sigmoid(u)) = -softplus(-u) in fp32, u ~ N(4, 1); optional skewed channels."""
    u = _randn(shape, gen, device, mean=4.0, std=1.0)
    if skew_channels:
        H, dk = shape[head_axis], shape[-1]
        sel = torch.zeros((H, dk), dtype=torch.bool)
        cpu_gen = _gen("cpu", 424242)
        for h in range(H):
            sel[h, torch.randperm(dk, generator=cpu_gen)[:skew_channels]] = True
        sel = sel.to(device)
        strong = _randn(shape, gen, device, mean=-1.0, std=0.5).clamp_(max=-0.05)
        u = torch.where(sel, strong, u)
    return -F.softplus(-u)


def make_prefill(wl: Workload, device="cpu", T: int | None = None, lengths=None,
                 raw: bool = False) -> dict:
    """Inputs of one prefill call (padded as one packed batch when varlen is empty).

    Returns a dict with q, k, v (io dtype), g, beta (fp32), h0 (fp32 or None),
    cu_seqlens (int32 tensor on device), cu_host (list), and for prologue workloads
    q_raw/k_raw/v_raw and w_q/w_k/w_v instead of q/k/v being normalised. raw=True adds the raw
    projections of the fused entry points (g_raw, beta_raw, A_log, dt_bias, z, w_norm).
    """
    gen = _gen(device, wl.seed)
    dt = io_dtype(wl.io)
    if lengths is not None:
        lengths = list(lengths)
    elif wl.varlen:
        lengths = varlen_lengths(wl)
    else:
        lengths = [T if T is not None else wl.T] * wl.N
    cu = cu_seqlens_of(lengths)
    T_tot, H, dk, dv = cu[-1], wl.H, wl.dk, wl.dv
    d = {"cu_host": cu, "lengths": lengths, "N": len(lengths), "H": H, "dk": dk, "dv": dv,
         "T_tot": T_tot, "io": wl.io, "scale": 1.0, "chunk": wl.chunk}
    d["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    if wl.prologue:
        d["q_raw"] = _randn((T_tot, H, dk), gen, device, dtype=dt)
        d["k_raw"] = _randn((T_tot, H, dk), gen, device, dtype=dt)
        d["v_raw"] = _randn((T_tot, H, dv), gen, device, dtype=dt)
        d["w_q"] = _randn((H * dk, 4), gen, device, std=0.5)
        d["w_k"] = _randn((H * dk, 4), gen, device, std=0.5)
        d["w_v"] = _randn((H * dv, 4), gen, device, std=0.5)
    else:
        d["q"] = _unit_rows((T_tot, H, dk), gen, device, dt)
        d["k"] = _unit_rows((T_tot, H, dk), gen, device, dt)
        d["v"] = _randn((T_tot, H, dv), gen, device, dtype=dt)
    d["beta"] = torch.sigmoid(_randn((T_tot, H), gen, device))
    d["g"] = _log_decay((T_tot, H, dk), gen, device, wl.skew_channels)
    d["h0"] = (_randn((len(lengths), H, dk, dv), gen, device, std=wl.h0_std)
               if wl.h0_std > 0 else None)
    if raw:
        d.update(_raw_projections((T_tot, H), H, dk, dv, dt, device, wl.seed))
    return d


def make_decode(wl: Workload, device="cpu", N: int | None = None, steps: int | None = None) -> dict:
    """Inputs of a decode run: initial state, conv weights, and per-step raw q/k/v, g, beta."""
    gen = _gen(device, wl.seed)
    N = N if N is not None else wl.N
    steps = steps if steps is not None else wl.steps
    H, dk, dv = wl.H, wl.dk, wl.dv
    dt = io_dtype(wl.io)
    d = {"N": N, "H": H, "dk": dk, "dv": dv, "steps": steps, "io": wl.io, "scale": 1.0}
    d["h0"] = _randn((N, H, dk, dv), gen, device, std=wl.h0_std)
    d["w_q"] = _randn((H * dk, 4), gen, device, std=0.5)
    d["w_k"] = _randn((H * dk, 4), gen, device, std=0.5)
    d["w_v"] = _randn((H * dv, 4), gen, device, std=0.5)
    d["conv_state"] = torch.zeros((N, H * (2 * dk + dv), 3), dtype=dt, device=device)
    d["q_raw"] = _randn((steps, N, H, dk), gen, device, dtype=dt)
    d["k_raw"] = _randn((steps, N, H, dk), gen, device, dtype=dt)
    d["v_raw"] = _randn((steps, N, H, dv), gen, device, dtype=dt)
    d["beta"] = torch.sigmoid(_randn((steps, N, H), gen, device))
    d["g"] = _log_decay((steps, N, H, dk), gen, device)
    d.update(_raw_projections((steps, N, H), H, dk, dv, dt, device, wl.seed))
    return d


def _raw_projections(lead, H, dk, dv, dt, device, seed) -> dict:
    """Raw gate and beta logits, A_log, dt_bias, and the output norm's gate and weight."""
    gen = _gen(device, seed + 100)
    return {"g_raw": _randn((*lead, dk), gen, device, mean=-4.0, dtype=dt),
            "beta_raw": _randn(lead, gen, device, dtype=dt),
            "A_log": _randn((H,), gen, device, std=0.1),
            "dt_bias": _randn((H * dk,), gen, device, std=0.1),
            "z": _randn((*lead, dv), gen, device, dtype=dt),
            "w_norm": _randn((dv,), gen, device, mean=1.0, std=0.1)}
