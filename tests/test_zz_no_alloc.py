"""kda_chunk_fwd_noalloc: the chunked prefill for callers that cannot allocate device memory
(a runtime whose pool already holds the free memory, a plug-in given only tensor pointers, or
a path that cannot take cudaMalloc's implicit synchronisation). It uses the library's own
device array as scratch instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on different inputs, and checks each
result against kda_chunk_fwd (the entry point with a caller workspace) within the bf16
parity tolerance, and against the oracle. It also checks that neither call allocates. The file
is collected last, so a run that stops at the first failure has run every other test first.
"""
from __future__ import annotations

import ctypes
import dataclasses

import pytest
import torch

from conftest import rel_l2
from gpu_helpers import TOL_BF16, check_prefill, to64
from kimi_delta_attention_32_b200 import kda
from kimi_delta_attention_32_b200.workloads import WORKLOADS, make_prefill

FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: checks fail first


def _noalloc(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, scale=1.0, h0=None, ht=None, o=FAKE,
             cu=None, cuh=None, B=1, T=64, N=1, H=2, dk=128, dv=128, chunk=64, io=1, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd_noalloc(a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"],
                                     a["h0"], a["ht"], a["o"], a["cu"], a["cuh"], a["B"], a["T"],
                                     a["N"], a["H"], a["dk"], a["dv"], a["chunk"], a["io"],
                                     a["stream"])


def test_noalloc_entry_is_exported_and_checks_arguments():
    lib = kda.load_library()
    assert hasattr(lib, "kda_chunk_fwd_noalloc")
    assert _noalloc(lib, chunk=0) == kda.KDA_ERR_INVALID_ARG
    assert _noalloc(lib, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _noalloc(lib, H=0) == kda.KDA_ERR_INVALID_ARG
    assert _noalloc(lib, dk=96, dv=96) == kda.KDA_ERR_UNSUPPORTED


def _free_bytes():
    free, _ = torch.cuda.mem_get_info()
    return free


@pytest.mark.gpu
def test_noalloc_two_calls_match_workspace_call_and_oracle():
    cases = [([1, 63, 64, 65, 0, 130, 7, 200], 77), ([1000, 3], 78)]
    inputs = []
    for lens, seed in cases:
        wl = dataclasses.replace(WORKLOADS["prefill_8k"], N=len(lens), H=3, h0_std=0.02, seed=seed)
        d = make_prefill(wl, "cuda", lengths=lens)
        args = (d["q"], d["k"], d["v"], d["g"], d["beta"], 1.0)
        kw = dict(h0=d["h0"], cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])
        o_ref, ht_ref = kda.chunk_fwd(*args, **kw)            # caller-workspace entry point
        inputs.append((d, args, kw, o_ref, ht_ref, torch.empty_like(o_ref),
                       torch.empty_like(ht_ref)))
    torch.cuda.synchronize()
    for i, (d, args, kw, o_ref, ht_ref, o, ht) in enumerate(inputs):   # two calls in a row
        before, free_before = torch.cuda.memory_allocated(), _free_bytes()
        kda.chunk_fwd_noalloc(*args, o=o, ht=ht, **kw)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before        # nothing allocated by the call
        if i > 0:
            # the first call on a device may be the one that makes CUDA load the library's
            # module, which reserves the static array; later calls leave device memory alone
            assert _free_bytes() >= free_before
        assert kda.last_device_error() == kda.KDA_OK
        eo, eh = rel_l2(to64(o), to64(o_ref)), rel_l2(to64(ht), to64(ht_ref))
        print(f"noalloc vs kda_chunk_fwd: o {eo:.2e}, ht {eh:.2e}")
        assert eo <= TOL_BF16 and eh <= TOL_BF16
        assert torch.equal(o, o_ref) and torch.equal(ht, ht_ref)   # same kernels, same inputs
        check_prefill(d, d["q"], d["k"], d["v"], o, ht)
