#!/usr/bin/env python3
"""Benchmark of libkda's KDA hot path on B200; prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload prefill_8k|varlen_prologue|long_256k|long_256k_tp4|decode_256x32|conv_8k]
                  [--no-rows]

Headline (default workload prefill_8k: B=1, H=32, T=8192, dk=dv=128, bf16 I/O, fp32
gates/beta/state, chunk 64): prefill tokens/s of kda_chunk_fwd with inputs resident in
HBM, timed per step with CUDA events on the launching stream, L2 flushed between steps.
`e2e` is the same metric through the C ABI with pinned HOST buffers (host->device copy of
the step's inputs and device->host copy of o and the final state inside the timed region).
`rows` adds every other config of the path measured in the same run: the conv prologue and
the packed 64-sequence prefill with its prologue, the 262,144-token prefill, and the decode
step (alone and with its conv step) on 256 x 32 states.
Under torchrun (N > 1) every rank runs its own replica (weak scaling, no collective on
the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (H=32,d=128) & decode GB/s; % of roofline on 1×B200"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic per launch of each workload's dominant kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum; profiles/ holds the summaries and commands).
# It is reported only while that kernel's sources hash to what was profiled.
MEASURED_TRAFFIC = {
    "prefill_8k": (("chunk_tcx.cu", "tc.cuh", "common.cuh", "tma_host.h"),
                   "fb083c4b23146025607119dc4bd5b0292d087831482b6dbf0e1565890c8cc62b", 392144640),
    "conv_8k": (("conv.cu", "common.cuh"),
                "28908a4c60fb3f184b90005e406d903129202d5acbbcbca4cb52243982fcf542", 365856512),
    "decode_256x32": (("recurrent_step.cu", "common.cuh"),
                      "a963466ab8982d94dcf368779351935ba00f725c3c02a9b04e8dababc04db62e", 1028144128),
}


# One description per workload, printed by both arms in config.workload.
WL_DESC = {
    "prefill_8k": "prefill_8k: B=1,H=32,T=8192,dk=dv=128,bf16 q/k/v/o,fp32 g/beta/state,chunk 64,"
                  "zero h0,final state returned",
    "long_256k": "long_256k: B=1,H=32,T=262144,dk=dv=128,bf16 q/k/v/o,fp32 g/beta/state,chunk 64,"
                 "13/128 channels per head with exp(g)<0.5,final state returned",
    "long_256k_tp4": "long_256k_tp4: B=1,H=8,T=262144,dk=dv=128,bf16 q/k/v/o,fp32 g/beta/state,"
                     "chunk 64,13/128 channels per head with exp(g)<0.5,final state returned,"
                     "split prefill",
}


def measured_traffic(workload):
    import hashlib
    entry = MEASURED_TRAFFIC.get(workload)
    if entry is None:
        return None
    files, digest, nbytes = entry
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "kimi_delta_attention_32_b200", "csrc")
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return nbytes if h.hexdigest() == digest else None


def max_over_ranks(dist, torch, value, device, world):
    """The largest `value` over all ranks (every rank gets it); `value` itself when world == 1.
    Timings of a multi-GPU run are the slowest rank's."""
    if world <= 1:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# Algorithmic bytes per token*head of the prefill (d = 128, bf16 q/k/v/o, fp32 g, beta):
# q, k, v in (3 * 256) + o out (256) + g (512) + beta (4) = 1540; plus h0/ht once per state.
def prefill_bytes(T_tot, H, dk, dv, N, io_bytes=2, h0=False, ht=True):
    per_tok = H * ((2 * dk + 2 * dv) * io_bytes + 4 * dk + 4)
    state = N * H * dk * dv * 4
    return T_tot * per_tok + state * (int(h0) + int(ht))


def prefill_flops(T_tot, H, dk, dv, C=64):
    # 6 dk dv (Qhat S, W S, Ktilde^T Ut) + C (3 dk + 2 dv) (A, P, W, U, intra-chunk O) + C^2/3
    return T_tot * H * (6 * dk * dv + C * (3 * dk + 2 * dv) + C * C / 3)


def decode_bytes(N, H, dk, dv, io_bytes=2):
    return N * H * (2 * dk * dv * 4 + (2 * dk + 2 * dv) * io_bytes + 4 * dk + 4)


def conv_bytes(T_tot, H, dk, dv, io_bytes=2):
    return T_tot * H * (2 * dk + dv) * io_bytes * 2


class ClockSampler:
    """Samples SM clocks and throttle reasons of this process's GPU during a region."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9 or (self.uuid and self.uuid not in parts[0]):
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- #
# CPU oracle arm                                                               #
# --------------------------------------------------------------------------- #

def oracle_prefill_rate(min_seconds=10.0, max_reps=50):
    """Times the fp64 oracle on the prefill_8k workload (all 32 heads x 8192 tokens) on the
    host cores; repeats whole passes until min_seconds. Returns (tokens/s, cores, sample)."""
    import oracle
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill
    d = make_prefill(WORKLOADS["prefill_8k"], "cpu")
    f64 = lambda t: t.double().numpy()       # noqa: E731
    args = [f64(d[n]) for n in ("q", "k", "v", "g", "beta")]
    cores = os.cpu_count() or 1
    oracle.load()
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.kda_fwd(*args, 1.0, None, d["cu_host"], nthreads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            break
    tokens = reps * d["T_tot"]
    sample = (f"{reps} full pass(es) of prefill_8k (B=1,H=32,T=8192,dk=dv=128) through the "
              f"fp64 token-by-token oracle, parallel over heads on {cores} threads, {el:.1f} s")
    return tokens / el, cores, sample, el / reps


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rate, cores, sample, sec_per_pass = None, None, None, None
    import oracle
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill
    d = make_prefill(WORKLOADS["prefill_8k"], "cpu")
    f64 = lambda t: t.double().numpy()       # noqa: E731
    a = [f64(d[n]) for n in ("q", "k", "v", "g", "beta")]
    cores = os.cpu_count() or 1
    oracle.load()
    for _ in range(args.warmup):
        oracle.kda_fwd(*a, 1.0, None, d["cu_host"], nthreads=cores)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.kda_fwd(*a, 1.0, None, d["cu_host"], nthreads=cores)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    rate = args.steps * d["T_tot"] / total
    sample = (f"each step: one full pass of prefill_8k (B=1,H=32,T=8192,dk=dv=128) through the "
              f"fp64 token-by-token oracle on {cores} host threads")
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WL_DESC["prefill_8k"], "parallelism": "1 GPU" if args.gpus <= 1
                       else f"replicas x{args.gpus} (rank 0 times the oracle)"},
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- #
# GPU arm                                                                      #
# --------------------------------------------------------------------------- #

def _events_time(torch, fn, steps, warmup, flush=None, stream=None):
    """Per-step device time (ms) with CUDA events on `stream`; `flush` runs between steps,
    outside the timed events."""
    stream = stream or torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush()
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    from kimi_delta_attention_32_b200 import kda
    status = kda.last_device_error()
    if status != kda.KDA_OK:         # a bounded wait gave up: the timing is not a valid number
        raise RuntimeError(f"device error word set during the timed steps (status {status})")
    return [a.elapsed_time(b) for a, b in ev]


def run_ours(args):
    import torch
    import torch.distributed as dist

    from kimi_delta_attention_32_b200 import kda
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_decode, make_prefill

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (libkda has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    kda.load_library()
    peaks, peaks_src = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])

    l2_flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def flush():
        l2_flush.fill_(1)

    wl = WORKLOADS.get(args.workload, WORKLOADS["prefill_8k"])
    stream = torch.cuda.current_stream()
    launches_per_step = 1
    rows = {}

    if args.workload == "conv_8k":
        # conv prologue alone on prefill_8k-shaped raw inputs (B=1, H=32, T=8192, d=128, bf16)
        import dataclasses
        cw = dataclasses.replace(WORKLOADS["varlen_prologue"], N=1, varlen=(), T=8192, h0_std=0.0)
        d = make_prefill(cw, dev)
        qo, ko, vo = (torch.empty_like(d[n]) for n in ("q_raw", "k_raw", "v_raw"))

        def step():
            kda.conv_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["w_q"], d["w_k"], d["w_v"], qo, ko,
                         vo, cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], stream=stream)
        units = d["T_tot"]
        algo_bytes = conv_bytes(d["T_tot"], d["H"], d["dk"], d["dv"])
        wl_desc = "conv_8k: conv+SiLU+L2 prologue on B=1,H=32,T=8192,dk=dv=128 raw bf16 q/k/v"
        flops = 0
        dtype = "bf16-io/f32"
        args.no_e2e = True
    elif args.workload == "decode_256x32":
        d = make_decode(wl, dev, steps=max(1, args.steps + args.warmup))
        state = d["h0"].clone()
        N, H, dk, dv = d["N"], d["H"], d["dk"], d["dv"]
        qn = torch.nn.functional.normalize(d["q_raw"].float(), dim=-1).to(d["q_raw"].dtype)
        kn = torch.nn.functional.normalize(d["k_raw"].float(), dim=-1).to(d["k_raw"].dtype)
        it = iter(range(10 ** 9))

        def step():
            s = next(it) % d["steps"]
            kda.recurrent_step(qn[s], kn[s], d["v_raw"][s], d["g"][s], d["beta"][s], state,
                               stream=stream)
        units = N        # tokens per step (one per sequence), over H heads
        algo_bytes = decode_bytes(N, H, dk, dv)
        wl_desc = (f"decode_256x32: N={N} sequences x H={H}, fp32 state {dk}x{dv}, bf16 q/k/v/o, "
                   "one token per sequence per step")
        flops = N * H * 7 * dk * dv
        dtype = "f32"
    else:
        d = make_prefill(wl, dev)
        T_tot, N, H, dk, dv = d["T_tot"], d["N"], d["H"], d["dk"], d["dv"]
        if wl.prologue:
            q, k, v = kda.conv_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["w_q"], d["w_k"],
                                   d["w_v"], cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])
        else:
            q, k, v = d["q"], d["k"], d["v"]
        o = torch.empty_like(v)
        ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
        ws_bytes = kda.chunk_fwd_workspace_size(N, T_tot, H, dk, dv,
                                                io=kda.KDA_IO_F32 if wl.io == "f32" else kda.KDA_IO_BF16)
        ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev) if ws_bytes else None

        def prefill(qq, kk, vv, gg, bb):
            kda.chunk_fwd(qq, kk, vv, gg, bb, 1.0, h0=d["h0"], ht=ht, o=o,
                          cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], workspace=ws,
                          stream=stream)
        if args.workload == "long_256k_tp4":
            # too few (sequence, head) pairs to fill the GPU: the split prefill (stretch bounds,
            # stretches from a zero state with their transitions, the join, the correction)
            P, need = kda.chunk_fwd_split_plan(q, v, d["cu_seqlens"], d["cu_host"], 0)
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
            launches_per_step = 4 if P > 1 else 1

            def prefill(qq, kk, vv, gg, bb):
                kda.chunk_fwd_split(qq, kk, vv, gg, bb, 1.0, h0=d["h0"], ht=ht, o=o,
                                    cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], n_split=P,
                                    workspace=ws, stream=stream)

        def step():
            prefill(q, k, v, d["g"], d["beta"])
        units = T_tot
        algo_bytes = prefill_bytes(T_tot, H, dk, dv, N, h0=d["h0"] is not None)
        wl_desc = dict(WL_DESC, varlen_prologue=f"varlen_prologue: 64 packed sequences "
                       f"U[128,16384] (T_tot={T_tot}),H=32,dk=dv=128,bf16,h0~N(0,0.02) "
                       "(timed: chunked prefill on the prologue's outputs)").get(args.workload,
                                                                                 args.workload)
        flops = prefill_flops(T_tot, H, dk, dv)
        dtype = "f32" if wl.io == "f32" else "bf16-io/f32"

    uuid = ""
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(uuid) as clk:
        times = _events_time(torch, step, args.steps, 0, flush=flush, stream=stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(dist, torch, sum(times), dev, world)
    ms_step = ms_total / args.steps
    value = units * world * args.steps / (ms_total / 1e3)
    achieved = algo_bytes / (statistics.mean(times) / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": measured_traffic(args.workload),
                "algorithmic_bytes_per_launch": algo_bytes,
                "peak_source": f"{peaks_src} hbm_gbs",
                "flop_term_frac": (flops / (statistics.mean(times) / 1e3) / 1e12)
                / float(peaks["bf16_tflops"])}

    # ---------------- e2e through the C ABI with pinned host buffers ----------------
    e2e = None
    if args.workload != "decode_256x32" and not args.no_e2e:
        names = ["q", "k", "v", "g", "beta"]
        host = {}
        srcs = {"q": q, "k": k, "v": v, "g": d["g"], "beta": d["beta"]}
        for nm in names:
            host[nm] = torch.empty(srcs[nm].shape, dtype=srcs[nm].dtype, pin_memory=True)
            host[nm].copy_(srcs[nm])
        dbuf = {nm: torch.empty_like(srcs[nm]) for nm in names}
        o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        ht_host = torch.empty(ht.shape, dtype=ht.dtype, pin_memory=True)
        h2d = sum(host[nm].numel() * host[nm].element_size() for nm in names)
        d2h = o_host.numel() * o_host.element_size() + ht_host.numel() * ht_host.element_size()

        def e2e_step():
            for nm in names:
                dbuf[nm].copy_(host[nm], non_blocking=True)
            prefill(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"])
            o_host.copy_(o, non_blocking=True)
            ht_host.copy_(ht, non_blocking=True)
        et = _events_time(torch, e2e_step, max(2, args.steps // 2), 2, stream=stream)
        ems = max_over_ranks(dist, torch, sum(et), dev, world)
        e2e = {"value": units * world * len(et) / (ems / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / len(et)}

    # ---------------- other rows of the path, same run (one GPU: they characterise the
    # kernels, and under torchrun they would hold every GPU for minutes between collectives) ----
    if not args.no_rows and args.workload == "prefill_8k" and world == 1:
        rows = measure_rows(torch, kda, dev, flush, hbm_peak, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, cores, sample, _ = oracle_prefill_rate() if args.workload == "prefill_8k" else \
            (None, None, None, None)
        if rate is not None:
            cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                   "sample": sample}
            r1, s1 = oracle_one_core_rate()
            cpu["one_core"] = {"value": r1, "unit": "tokens/s", "cores": 1, "sample": s1}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic (seeded, device-generated)",
            "config": {"workload": wl_desc, "parallelism": f"replicas x{world}" if world > 1
                       else "1 GPU", "l2": "flushed (256 MiB write) between timed steps"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(), "rows": rows}
    print(json.dumps(line), flush=True)
    return 0


def _prefill_row(torch, kda, dev, flush, hbm_peak, stream, name, with_prologue=False, steps=5):
    """One prefill workload timed as in the headline: chunk pass alone, and for the packed
    workload also conv prologue + chunk pass (the config as stated)."""
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill
    wl = WORKLOADS[name]
    d = make_prefill(wl, dev)
    T_tot, N, H, dk, dv = d["T_tot"], d["N"], d["H"], d["dk"], d["dv"]
    o = torch.empty((T_tot, H, dv), dtype=torch.bfloat16, device=dev)
    ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    ws = torch.empty(kda.chunk_fwd_workspace_size(N, T_tot, H, dk, dv), dtype=torch.uint8,
                     device=dev)
    if with_prologue:
        q, k, v = (torch.empty_like(d[n]) for n in ("q_raw", "k_raw", "v_raw"))
    else:
        q, k, v = d["q"], d["k"], d["v"]

    def conv():
        kda.conv_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["w_q"], d["w_k"], d["w_v"], q, k, v,
                     cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], stream=stream)

    def chunk():
        kda.chunk_fwd(q, k, v, d["g"], d["beta"], 1.0, h0=d["h0"], ht=ht, o=o,
                      cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], workspace=ws, stream=stream)

    if with_prologue:
        conv()
    algo = prefill_bytes(T_tot, H, dk, dv, N, h0=d["h0"] is not None)
    ms = statistics.mean(_events_time(torch, chunk, steps, 2, flush=flush, stream=stream))
    row = {"workload": WL_DESC.get(name, f"{name}: {N} packed sequences (T_tot={T_tot}),H={H},"
                                          f"dk=dv={dk},bf16,h0~N(0,0.02)"),
           "chunk_ms": ms, "chunk_tokens/s": T_tot / ms * 1e3,
           "algorithmic_bytes": algo, "chunk_frac_hbm": algo / ms / 1e6 / hbm_peak}
    if with_prologue:
        def both():
            conv()
            chunk()
        ms2 = statistics.mean(_events_time(torch, both, steps, 2, flush=flush, stream=stream))

        def fused():
            kda.chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v_raw"], d["g"], d["beta"], w_q=d["w_q"],
                                w_k=d["w_k"], w_v=d["w_v"], h0=d["h0"], ht=ht, o=o,
                                cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], workspace=ws,
                                stream=stream)
        ms3 = statistics.mean(_events_time(torch, fused, steps, 2, flush=flush, stream=stream))
        # the config's own bytes: raw q/k/v in instead of the normalised ones (same size); the
        # headline of the row is the prefill with the prologue fused in, as the config states
        row.update({"conv_then_chunk_ms": ms2, "fused_ms": ms3, "tokens/s": T_tot / ms3 * 1e3,
                    "frac_hbm": algo / ms3 / 1e6 / hbm_peak,
                    "conv_then_chunk_frac_hbm": algo / ms2 / 1e6 / hbm_peak})
    else:
        row.update({"tokens/s": T_tot / ms * 1e3, "frac_hbm": algo / ms / 1e6 / hbm_peak})
    return row


def _gated_row(torch, kda, dev, flush, hbm_peak, stream, steps=5):
    """prefill_8k's shape with the gate and beta from raw bf16 logits and the gated RMSNorm of
    the output fused in: bytes per token*head are q, k, v, o (4 * 256) + raw gate logits (256) +
    raw beta (2) + the norm's gate z (256)."""
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill
    d = make_prefill(WORKLOADS["prefill_8k"], dev, raw=True)
    T_tot, N, H, dk, dv = d["T_tot"], d["N"], d["H"], d["dk"], d["dv"]
    o = torch.empty_like(d["v"])
    ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    ws = torch.empty(kda.chunk_fwd_workspace_size(N, T_tot, H, dk, dv), dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_fwd_fused(d["q"], d["k"], d["v"], g_raw=d["g_raw"], beta_raw=d["beta_raw"],
                            A_log=d["A_log"], dt_bias=d["dt_bias"], z=d["z"], w_norm=d["w_norm"],
                            ht=ht, o=o, workspace=ws, stream=stream)
    ms = statistics.mean(_events_time(torch, step, steps, 2, flush=flush, stream=stream))
    algo = T_tot * H * (4 * 256 + 256 + 2 + 256) + N * H * dk * dv * 4
    return {"workload": "prefill_8k shape, gate and beta from raw bf16 logits, gated RMSNorm output",
            "ms": ms, "tokens/s": T_tot / ms * 1e3, "algorithmic_bytes": algo,
            "frac_hbm": algo / ms / 1e6 / hbm_peak}


def _split_row(torch, kda, dev, flush, hbm_peak, stream, steps=3):
    """long_256k_tp4 (8 heads of one of four tensor-parallel GPUs, 262144 tokens): the prefill
    as one cluster per (sequence, head), and split into stretches that run side by side (the
    count chosen by the library). Same algorithmic bytes for both."""
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill
    wl = WORKLOADS["long_256k_tp4"]
    d = make_prefill(wl, dev)
    T_tot, N, H, dk, dv = d["T_tot"], d["N"], d["H"], d["dk"], d["dv"]
    o = torch.empty_like(d["v"])
    ht = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    P, need = kda.chunk_fwd_split_plan(d["q"], d["v"], d["cu_seqlens"], d["cu_host"], 0)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def run(n_split):
        return lambda: kda.chunk_fwd_split(d["q"], d["k"], d["v"], d["g"], d["beta"], 1.0, ht=ht,
                                           o=o, cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"],
                                           n_split=n_split, workspace=ws, stream=stream)
    ms1 = statistics.mean(_events_time(torch, run(1), steps, 2, flush=flush, stream=stream))
    msP = statistics.mean(_events_time(torch, run(P), steps, 2, flush=flush, stream=stream))
    algo = prefill_bytes(T_tot, H, dk, dv, N, h0=False)
    return {"workload": "long_256k_tp4: B=1,H=8,T=262144,dk=dv=128,bf16,skewed gates",
            "stretches": P, "one_cluster_per_head_ms": ms1, "split_ms": msP,
            "tokens/s": T_tot / msP * 1e3, "algorithmic_bytes": algo,
            "frac_hbm": algo / msP / 1e6 / hbm_peak,
            "one_cluster_per_head_frac_hbm": algo / ms1 / 1e6 / hbm_peak}


def measure_rows(torch, kda, dev, flush, hbm_peak, stream):
    """Every other config of the path, measured in the same run: the conv prologue and the
    packed prefill with its prologue (64 sequences), the long-context prefill, and the decode
    step alone and paired with its conv step (256 x 32 states)."""
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_decode, make_prefill
    out = {}
    wl = WORKLOADS["varlen_prologue"]
    d = make_prefill(wl, dev)
    qo, ko, vo = (torch.empty_like(d[n]) for n in ("q_raw", "k_raw", "v_raw"))

    def conv():
        kda.conv_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["w_q"], d["w_k"], d["w_v"], qo, ko, vo,
                     cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"], stream=stream)
    t = _events_time(torch, conv, 5, 2, flush=flush, stream=stream)
    b = conv_bytes(d["T_tot"], d["H"], d["dk"], d["dv"])
    ms = statistics.mean(t)
    out["a1_conv_prologue"] = {"workload": f"varlen_prologue raw q/k/v (T_tot={d['T_tot']},H=32,"
                                           "d=128,bf16)", "ms": ms, "GB/s": b / ms / 1e6,
                               "frac_hbm": b / ms / 1e6 / hbm_peak,
                               "tokens/s": d["T_tot"] / ms * 1e3}
    del d, qo, ko, vo
    torch.cuda.empty_cache()

    out["varlen_prologue"] = _prefill_row(torch, kda, dev, flush, hbm_peak, stream,
                                          "varlen_prologue", with_prologue=True, steps=3)
    torch.cuda.empty_cache()
    out["long_256k"] = _prefill_row(torch, kda, dev, flush, hbm_peak, stream, "long_256k", steps=3)
    torch.cuda.empty_cache()
    out["prefill_8k_gated_norm"] = _gated_row(torch, kda, dev, flush, hbm_peak, stream)
    torch.cuda.empty_cache()
    out["long_256k_tp4_split"] = _split_row(torch, kda, dev, flush, hbm_peak, stream)
    torch.cuda.empty_cache()

    wl = WORKLOADS["decode_256x32"]
    steps = 16
    dd = make_decode(wl, dev, steps=steps)
    qn = torch.nn.functional.normalize(dd["q_raw"].float(), dim=-1).to(dd["q_raw"].dtype)
    kn = torch.nn.functional.normalize(dd["k_raw"].float(), dim=-1).to(dd["k_raw"].dtype)
    state = dd["h0"].clone()
    cache = dd["conv_state"].clone()
    it = iter(range(10 ** 9))

    def dec():
        s = next(it) % steps
        kda.recurrent_step(qn[s], kn[s], dd["v_raw"][s], dd["g"][s], dd["beta"][s], state,
                           stream=stream)
    t = _events_time(torch, dec, 20, 3, flush=flush, stream=stream)
    b = decode_bytes(wl.N, wl.H, wl.dk, wl.dv)
    ms = statistics.mean(t)
    it2 = iter(range(10 ** 9))
    bufs = [torch.empty_like(dd[n][0]).unsqueeze(1) for n in ("q_raw", "k_raw", "v_raw")]

    def pair():
        s = next(it2) % steps
        x = [dd[n][s].unsqueeze(1) for n in ("q_raw", "k_raw", "v_raw")]
        qq, kk, vv = kda.conv_fwd(*x, dd["w_q"], dd["w_k"], dd["w_v"], *bufs, conv_state=cache,
                                  stream=stream)
        kda.recurrent_step(qq[:, 0], kk[:, 0], vv[:, 0], dd["g"][s], dd["beta"][s], state,
                           stream=stream)
    tp = statistics.mean(_events_time(torch, pair, 20, 3, flush=flush, stream=stream))
    it3 = iter(range(10 ** 9))

    def fused():
        s = next(it3) % steps
        kda.conv_recurrent_step(dd["q_raw"][s], dd["k_raw"][s], dd["v_raw"][s], dd["w_q"],
                                dd["w_k"], dd["w_v"], cache, dd["g"][s], dd["beta"][s], state,
                                stream=stream)
    tf = statistics.mean(_events_time(torch, fused, 20, 3, flush=flush, stream=stream))
    # the pair's own bytes: the step's, with raw q/k/v in place of the normalised ones, plus
    # the width-3 conv cache read and written
    cache_rw = 2 * wl.N * wl.H * (2 * wl.dk + wl.dv) * 3 * 2
    out["a5_decode_step"] = {"workload": "decode_256x32: 256 seq x 32 heads, fp32 128x128 state",
                             "ms": ms, "GB/s": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm_peak,
                             "tokens/s": wl.N / ms * 1e3,
                             "conv_plus_step_ms": tp,
                             "conv_plus_step_GB/s": (b + cache_rw) / tp / 1e6,
                             "conv_plus_step_frac_hbm": (b + cache_rw) / tp / 1e6 / hbm_peak,
                             "fused_conv_step_ms": tf,
                             "fused_conv_step_GB/s": (b + cache_rw) / tf / 1e6,
                             "fused_conv_step_frac_hbm": (b + cache_rw) / tf / 1e6 / hbm_peak}
    return out


def oracle_one_core_rate(heads=4):
    """The fp64 oracle on ONE host thread over a bounded sample of prefill_8k (the first
    `heads` heads, all 8192 tokens). Returns (tokens/s normalised to H=32, sample)."""
    import oracle
    from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill
    d = make_prefill(WORKLOADS["prefill_8k"], "cpu")
    f64 = lambda t: t[:, :heads].double().numpy()       # noqa: E731
    args = [f64(d[n]) for n in ("q", "k", "v", "g", "beta")]
    oracle.load()
    t0 = time.perf_counter()
    oracle.kda_fwd(*args, 1.0, None, d["cu_host"], nthreads=1)
    el = time.perf_counter() - t0
    rate = d["T_tot"] * heads / el / d["H"]
    return rate, (f"heads 0..{heads - 1} of prefill_8k (8192 tokens each) on 1 host thread, "
                  f"{el:.1f} s, scaled to H={d['H']}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_8k",
                    choices=["prefill_8k", "varlen_prologue", "long_256k", "decode_256x32",
                             "conv_8k", "long_256k_tp4"])
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
