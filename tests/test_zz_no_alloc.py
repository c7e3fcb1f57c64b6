"""kda_chunk_fwd_noalloc: the chunked prefill with the library's own device array as its
workspace, so that the call allocates nothing. It must give exactly kda_chunk_fwd's results
(same kernels, same inputs), which the oracle checks in turn. Collected last."""
from __future__ import annotations

import ctypes
import dataclasses

import pytest
import torch

from gpu_helpers import check_prefill
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
    assert _noalloc(lib, dk=96, dv=96) == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("lens", [[1, 63, 64, 65, 0, 130, 7, 200], [1000, 3]])
def test_noalloc_matches_workspace_call_and_oracle(lens):
    wl = dataclasses.replace(WORKLOADS["prefill_8k"], N=len(lens), H=3, h0_std=0.02, seed=77)
    d = make_prefill(wl, "cuda", lengths=lens)
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"], 1.0)
    kw = dict(h0=d["h0"], cu_seqlens=d["cu_seqlens"], cu_host=d["cu_host"])
    o_ref, ht_ref = kda.chunk_fwd(*args, **kw)
    o = torch.empty_like(o_ref)
    ht = torch.empty_like(ht_ref)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    kda.chunk_fwd_noalloc(*args, o=o, ht=ht, **kw)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before          # nothing allocated by the call
    assert kda.last_device_error() == kda.KDA_OK
    assert torch.equal(o, o_ref) and torch.equal(ht, ht_ref)
    check_prefill(d, d["q"], d["k"], d["v"], o, ht)
