"""CPU tests of the C ABI: the library loads, exports every function kda.h declares,
and rejects bad arguments on the host before anything is launched."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from kimi_delta_attention_32_b200 import build as kbuild
from kimi_delta_attention_32_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "kda.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(kda.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libkda.so does not export {name}"


def test_status_strings(lib):
    for s in range(6):
        assert lib.kda_status_string(s)
    assert lib.kda_status_string(99) == b"unknown status"
    assert lib.kda_version() >= 100


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: checks fail first
MIS = ctypes.c_void_p(0x10004)           # misaligned


def _chunk(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, scale=1.0, h0=None, ht=None, o=FAKE,
             cu=None, cuh=None, B=1, T=64, N=1, H=2, dk=128, dv=128, chunk=64, io=1, ws=None,
             wsb=0, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"], a["h0"],
                             a["ht"], a["o"], a["cu"], a["cuh"], a["B"], a["T"], a["N"], a["H"],
                             a["dk"], a["dv"], a["chunk"], a["io"], a["ws"], a["wsb"],
                             a["stream"])


def _cu_host(vals):
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return arr, ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(o=None), kda.KDA_ERR_INVALID_ARG),
    (dict(k=MIS), kda.KDA_ERR_INVALID_ARG),
    (dict(h0=MIS), kda.KDA_ERR_INVALID_ARG),
    (dict(chunk=0), kda.KDA_ERR_INVALID_ARG),
    (dict(chunk=-64), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=0), kda.KDA_ERR_INVALID_ARG),
    (dict(B=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(io=7), kda.KDA_ERR_INVALID_ARG),
    (dict(chunk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(dk=96, dv=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dk=128, dv=32), kda.KDA_ERR_UNSUPPORTED),
])
def test_chunk_fwd_rejects(lib, kw, status):
    assert _chunk(lib, **kw) == status


def test_chunk_fwd_rejects_bad_cu_seqlens(lib):
    keep, cuh = _cu_host([0, 5, 3])                      # not monotone
    assert _chunk(lib, cu=FAKE, cuh=cuh, N=2) == kda.KDA_ERR_INVALID_ARG
    keep, cuh = _cu_host([1, 5, 9])                      # does not start at 0
    assert _chunk(lib, cu=FAKE, cuh=cuh, N=2) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, cu=FAKE, cuh=None, N=2) == kda.KDA_ERR_INVALID_ARG   # host copy missing
    keep, cuh = _cu_host([0, 5, 9])
    assert _chunk(lib, cu=None, cuh=cuh, N=2) == kda.KDA_ERR_INVALID_ARG    # device copy missing
    del keep


def _conv(lib, **kw):
    a = dict(x=FAKE, w=FAKE, y=FAKE, cs=None, cu=None, cuh=None, B=2, T=16, N=2, H=2, dk=128,
             dv=128, K=4, eps=1e-6, io=1)
    a.update(kw)
    return lib.kda_conv_fwd(a["x"], a["x"], a["x"], a["w"], a["w"], a["w"], a["y"], a["y"],
                            a["y"], a["cs"], a["cu"], a["cuh"], a["B"], a["T"], a["N"], a["H"],
                            a["dk"], a["dv"], a["K"], a["eps"], a["io"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(K=1), kda.KDA_ERR_INVALID_ARG),           # conv kernel must be >= 2
    (dict(K=0), kda.KDA_ERR_INVALID_ARG),
    (dict(x=None), kda.KDA_ERR_INVALID_ARG),
    (dict(w=MIS), kda.KDA_ERR_INVALID_ARG),
    (dict(cs=MIS), kda.KDA_ERR_INVALID_ARG),
    (dict(eps=-1.0), kda.KDA_ERR_INVALID_ARG),
    (dict(H=-2), kda.KDA_ERR_INVALID_ARG),
    (dict(K=3), kda.KDA_ERR_UNSUPPORTED),
    (dict(K=2), kda.KDA_ERR_UNSUPPORTED),
    (dict(dk=32), kda.KDA_ERR_UNSUPPORTED),
])
def test_conv_fwd_rejects(lib, kw, status):
    assert _conv(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(state=None), kda.KDA_ERR_INVALID_ARG),
    (dict(q=MIS), kda.KDA_ERR_INVALID_ARG),
    (dict(N=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dv=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=256), kda.KDA_ERR_UNSUPPORTED),
])
def test_recurrent_step_rejects(lib, kw, status):
    a = dict(q=FAKE, state=FAKE, N=4, H=2, dk=128, dv=128)
    a.update(kw)
    st = lib.kda_recurrent_step(a["q"], FAKE, FAKE, FAKE, FAKE, 1.0, a["state"], FAKE, a["N"],
                                a["H"], a["dk"], a["dv"], 1, None)
    assert st == status


def test_workspace_query(lib):
    out = ctypes.c_size_t(123)
    # bf16, dk = dv = 128, chunk 64: the tensor-core pipeline's fixed hand-off rings
    assert lib.kda_chunk_fwd_workspace_size(1, 8192, 32, 128, 128, 64, 1, ctypes.byref(out)) == 0
    ring = out.value
    assert ring > 0 and ring % 16 == 0
    assert lib.kda_chunk_fwd_workspace_size(64, 527241, 32, 128, 128, 64, 1, ctypes.byref(out)) == 0
    assert out.value == ring                              # independent of the batch
    for dk, io in ((128, 0), (64, 1), (64, 0)):           # fp32 I/O and d = 64 need none
        assert lib.kda_chunk_fwd_workspace_size(1, 8192, 32, dk, dk, 64, io, ctypes.byref(out)) == 0
        assert out.value == 0
    assert lib.kda_chunk_fwd_workspace_size(1, 8192, 32, 128, 128, 0, 1, ctypes.byref(out)) == \
        kda.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_workspace_size(1, 8192, 32, 128, 128, 64, 1, None) == \
        kda.KDA_ERR_INVALID_ARG


def test_wait_limit_checks_its_argument(lib):
    assert lib.kda_set_wait_limit(-1) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_set_wait_limit(123456) == kda.KDA_OK
    assert lib.kda_set_wait_limit(0) == kda.KDA_OK


def test_chunk_fwd_checks_workspace(lib):
    out = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(1, 64, 2, 128, 128, 64, 1, ctypes.byref(out)) == 0
    need = out.value
    assert _chunk(lib) == kda.KDA_ERR_WORKSPACE                          # missing
    assert _chunk(lib, ws=MIS, wsb=need) == kda.KDA_ERR_WORKSPACE         # misaligned
    assert _chunk(lib, ws=FAKE, wsb=need - 16) == kda.KDA_ERR_WORKSPACE   # too small


def _fused_step(lib, **kw):
    a = dict(qr=FAKE, kr=FAKE, vr=FAKE, gr=FAKE, br=FAKE, wq=FAKE, wk=FAKE, wv=FAKE, cs=FAKE,
             A=FAKE, dt=FAKE, z=None, wn=None, neps=1e-6, scale=1.0, state=FAKE, o=FAKE, N=2,
             H=2, dk=128, dv=128, K=4, eps=1e-6, io=1, stream=None)
    a.update(kw)
    return lib.kda_fused_recurrent_step(a["qr"], a["kr"], a["vr"], a["gr"], a["br"], a["wq"],
                                        a["wk"], a["wv"], a["cs"], a["A"], a["dt"], a["z"],
                                        a["wn"], a["neps"], a["scale"], a["state"], a["o"], a["N"],
                                        a["H"], a["dk"], a["dv"], a["K"], a["eps"], a["io"],
                                        a["stream"])


def _conv_step(lib, **kw):
    a = dict(qr=FAKE, kr=FAKE, vr=FAKE, wq=FAKE, wk=FAKE, wv=FAKE, cs=FAKE, g=FAKE, b=FAKE,
             scale=1.0, state=FAKE, o=FAKE, N=2, H=2, dk=128, dv=128, K=4, eps=1e-6, io=1,
             stream=None)
    a.update(kw)
    return lib.kda_conv_recurrent_step(a["qr"], a["kr"], a["vr"], a["wq"], a["wk"], a["wv"],
                                       a["cs"], a["g"], a["b"], a["scale"], a["state"], a["o"],
                                       a["N"], a["H"], a["dk"], a["dv"], a["K"], a["eps"],
                                       a["io"], a["stream"])


def test_fused_decode_entry_points_check_arguments(lib):
    for fn in (_fused_step, _conv_step):
        assert fn(lib, cs=None) == kda.KDA_ERR_INVALID_ARG          # the conv history is required
        assert fn(lib, qr=MIS) == kda.KDA_ERR_INVALID_ARG
        assert fn(lib, K=1) == kda.KDA_ERR_INVALID_ARG
        assert fn(lib, K=3) == kda.KDA_ERR_UNSUPPORTED
        assert fn(lib, dk=96) == kda.KDA_ERR_UNSUPPORTED
        assert fn(lib, eps=-1.0) == kda.KDA_ERR_INVALID_ARG
        assert fn(lib, H=0) == kda.KDA_ERR_INVALID_ARG
        assert fn(lib, io=7) == kda.KDA_ERR_INVALID_ARG
    assert _fused_step(lib, A=None) == kda.KDA_ERR_INVALID_ARG
    assert _fused_step(lib, dt=None) == kda.KDA_ERR_INVALID_ARG
    assert _fused_step(lib, z=FAKE) == kda.KDA_ERR_INVALID_ARG       # a norm gate without weight
    assert _fused_step(lib, br=ctypes.c_void_p(0x10001)) == kda.KDA_ERR_INVALID_ARG


def _fused(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, wq=None, wk=None, wv=None, cs=None, l2=1e-6, g=FAKE, b=FAKE,
             gr=None, br=None, A=None, dt=None, z=None, wn=None, neps=1e-6, scale=1.0, h0=None,
             ht=None, o=FAKE, cu=None, cuh=None, B=1, T=64, N=1, H=2, dk=128, dv=128, K=4,
             chunk=64, io=1, ws=FAKE, wsb=1 << 30, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd_fused(a["q"], a["k"], a["v"], a["wq"], a["wk"], a["wv"], a["cs"],
                                   a["l2"], a["g"], a["b"], a["gr"], a["br"], a["A"], a["dt"],
                                   a["z"], a["wn"], a["neps"], a["scale"], a["h0"], a["ht"],
                                   a["o"], a["cu"], a["cuh"], a["B"], a["T"], a["N"], a["H"],
                                   a["dk"], a["dv"], a["K"], a["chunk"], a["io"], a["ws"], a["wsb"],
                                   a["stream"])


def test_fused_prefill_checks_arguments(lib):
    gate = dict(gr=FAKE, br=FAKE, A=FAKE, dt=FAKE, g=None, b=None)
    conv = dict(wq=FAKE, wk=FAKE, wv=FAKE)
    assert _fused(lib, g=None) == kda.KDA_ERR_INVALID_ARG            # neither g nor raw logits
    assert _fused(lib, **dict(gate, A=None)) == kda.KDA_ERR_INVALID_ARG
    assert _fused(lib, **dict(gate, dt=None)) == kda.KDA_ERR_INVALID_ARG
    assert _fused(lib, **dict(gate, br=ctypes.c_void_p(0x10001))) == kda.KDA_ERR_INVALID_ARG
    assert _fused(lib, wq=FAKE) == kda.KDA_ERR_INVALID_ARG           # conv weights all or none
    assert _fused(lib, cs=FAKE) == kda.KDA_ERR_INVALID_ARG           # a history without the conv
    assert _fused(lib, **dict(conv, l2=-1.0)) == kda.KDA_ERR_INVALID_ARG
    assert _fused(lib, **dict(conv, K=3)) == kda.KDA_ERR_UNSUPPORTED
    assert _fused(lib, z=FAKE) == kda.KDA_ERR_INVALID_ARG            # a norm gate without weight
    assert _fused(lib, chunk=0) == kda.KDA_ERR_INVALID_ARG
    assert _fused(lib, io=0) == kda.KDA_ERR_UNSUPPORTED               # tensor-core path only
    assert _fused(lib, dk=64, dv=64) == kda.KDA_ERR_UNSUPPORTED
    assert _fused(lib, ws=None) == kda.KDA_ERR_WORKSPACE


def test_split_workspace_query(lib):
    P, out = ctypes.c_int(0), ctypes.c_size_t(0)
    ring = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(1, 8192, 4, 128, 128, 64, 1, ctypes.byref(ring)) == 0
    sizes = []
    for n_split in (1, 2, 8):
        assert lib.kda_chunk_fwd_split_workspace_size(None, 1, 8192, 0, 4, 128, 128, 64, 1, n_split,
                                                      ctypes.byref(P), ctypes.byref(out)) == 0
        assert P.value == n_split
        sizes.append(out.value)
    assert sizes[0] == ring.value                       # one stretch: kda_chunk_fwd's rings
    # rings + stretch bounds + (transition, end state, entering state) per stretch and head
    # + the carried-back queries (bf16, one row per token and head)
    per = 4 * 128 * 128 * 3
    wq = 8192 * 4 * 128 * 2
    assert sizes[1] >= ring.value + 2 * 4 * per + wq and sizes[2] >= ring.value + 8 * 4 * per + wq
    assert sizes[2] - sizes[1] < 6 * 4 * per + 1024
    keep, cuh = _cu_host([0, 100, 100, 5000])
    assert lib.kda_chunk_fwd_split_workspace_size(cuh, 0, 0, 3, 4, 128, 128, 64, 1, 3,
                                                  ctypes.byref(P), ctypes.byref(out)) == 0
    assert P.value == 3 and out.value >= ring.value + 9 * 4 * per
    bad = _cu_host([0, 100, 50])
    assert lib.kda_chunk_fwd_split_workspace_size(bad[1], 0, 0, 2, 4, 128, 128, 64, 1, 2,
                                                  ctypes.byref(P), ctypes.byref(out)) == \
        kda.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_split_workspace_size(None, 1, 8192, 0, 4, 128, 128, 64, 1, -1,
                                                  ctypes.byref(P), ctypes.byref(out)) == \
        kda.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_split_workspace_size(None, 1, 8192, 0, 4, 128, 128, 64, 0, 2,
                                                  ctypes.byref(P), ctypes.byref(out)) == \
        kda.KDA_ERR_UNSUPPORTED                          # fp32 I/O has no split path
    assert lib.kda_chunk_fwd_split_workspace_size(None, 1, 8192, 0, 4, 128, 128, 64, 1, 2, None,
                                                  ctypes.byref(out)) == kda.KDA_ERR_INVALID_ARG
    del keep


def _states(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, scale=1.0, h0=None, ht=FAKE, o=None, m=FAKE,
             w=None, cu=None, cuh=None, B=1, T=64, N=1, H=2, dk=128, dv=128, chunk=64, io=1,
             ws=FAKE, wsb=1 << 40, stream=None)
    a.update(kw)
    return lib.kda_chunk_states(a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"], a["h0"],
                                a["ht"], a["o"], a["m"], a["w"], a["cu"], a["cuh"], a["B"], a["T"],
                                a["N"], a["H"], a["dk"], a["dv"], a["chunk"], a["io"], a["ws"],
                                a["wsb"], a["stream"])


def test_chunk_states_checks_arguments(lib):
    assert _states(lib, ht=None, m=None) == kda.KDA_ERR_INVALID_ARG     # nothing to form
    assert _states(lib, o=MIS) == kda.KDA_ERR_INVALID_ARG
    assert _states(lib, w=MIS) == kda.KDA_ERR_INVALID_ARG
    assert _states(lib, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _states(lib, m=MIS) == kda.KDA_ERR_INVALID_ARG
    assert _states(lib, beta=None) == kda.KDA_ERR_INVALID_ARG
    assert _states(lib, io=0) == kda.KDA_ERR_UNSUPPORTED                 # tensor-core path only
    assert _states(lib, dk=64, dv=64) == kda.KDA_ERR_UNSUPPORTED
    assert _states(lib, ws=None) == kda.KDA_ERR_WORKSPACE
    assert _states(lib, wsb=16) == kda.KDA_ERR_WORKSPACE


def test_state_scan_checks_arguments(lib):
    def scan(**kw):
        a = dict(m=FAKE, z=FAKE, h0=None, hs=FAKE, ht=None, N=2, P=3, H=2, dk=128, dv=128, sn=3,
                 sp=1)
        a.update(kw)
        return lib.kda_state_scan(a["m"], a["z"], a["h0"], a["hs"], a["ht"], a["N"], a["P"], a["H"],
                                  a["dk"], a["dv"], a["sn"], a["sp"], None)
    assert scan(P=0) == kda.KDA_ERR_INVALID_ARG
    assert scan(m=None) == kda.KDA_ERR_INVALID_ARG
    assert scan(z=MIS) == kda.KDA_ERR_INVALID_ARG
    assert scan(sn=-1) == kda.KDA_ERR_INVALID_ARG
    assert scan(H=0) == kda.KDA_ERR_INVALID_ARG
    assert scan(dk=96) == kda.KDA_ERR_UNSUPPORTED


def test_chunk_fwd_split_checks_arguments(lib):
    def split(**kw):
        a = dict(o=FAKE, q=FAKE, n=2, io=1, ws=FAKE, wsb=16, chunk=64)
        a.update(kw)
        return lib.kda_chunk_fwd_split(a["q"], FAKE, FAKE, FAKE, FAKE, 1.0, None, None, a["o"], None,
                                       None, 1, 8192, 0, 4, 128, 128, a["chunk"], a["io"], a["n"],
                                       a["ws"], a["wsb"], None)
    assert split(o=None) == kda.KDA_ERR_INVALID_ARG
    assert split(q=MIS) == kda.KDA_ERR_INVALID_ARG
    assert split(n=-2) == kda.KDA_ERR_INVALID_ARG
    assert split(io=0) == kda.KDA_ERR_UNSUPPORTED
    assert split(chunk=32) == kda.KDA_ERR_UNSUPPORTED
    assert split() == kda.KDA_ERR_WORKSPACE                            # 16 bytes is too small
    assert split(ws=None, wsb=1 << 40) == kda.KDA_ERR_WORKSPACE


def test_output_correct_checks_arguments(lib):
    keep, cuh = _cu_host([0, 10, 30])

    def corr(**kw):
        a = dict(w=FAKE, h=FAKE, o=FAKE, cu=FAKE, cuh=cuh, N=2, H=2, dk=128, dv=128, io=1)
        a.update(kw)
        return lib.kda_output_correct(a["w"], a["h"], a["o"], a["cu"], a["cuh"], 0, 0, a["N"],
                                      a["H"], a["dk"], a["dv"], a["io"], None)
    assert corr(w=None) == kda.KDA_ERR_INVALID_ARG
    assert corr(h=MIS) == kda.KDA_ERR_INVALID_ARG
    assert corr(cuh=None) == kda.KDA_ERR_INVALID_ARG                     # host copy missing
    assert corr(H=0) == kda.KDA_ERR_INVALID_ARG
    assert corr(io=0) == kda.KDA_ERR_UNSUPPORTED
    assert corr(dk=64) == kda.KDA_ERR_UNSUPPORTED
    assert corr(cu=None, cuh=None) == kda.KDA_ERR_UNSUPPORTED            # padded: not supported
    del keep


def _plan(lib, cuh=None, B=1, T=8192, N=0, H=32, n_split=0, clusters=33):
    P, out = ctypes.c_int(0), ctypes.c_size_t(0)
    st = lib.kda_chunk_fwd_split_plan(cuh, B, T, N, H, 128, 128, 64, 1, n_split, clusters,
                                      ctypes.byref(P), ctypes.byref(out))
    return st, P.value, out.value


def test_split_plan_choices(lib):
    """The split's cost model on a B200 (33 resident 4-SM clusters), host-only: the benchmark's
    workloads with 32 heads keep one stretch; the 8 heads of one of four tensor-parallel GPUs
    over 262144 tokens split in two (measured 4.7 ms against 8.4 ms unsplit); 4 heads split in
    four; a GPU that 8 heads already fill does not split."""
    assert _plan(lib, T=8192, H=32)[:2] == (kda.KDA_OK, 1)              # prefill_8k
    assert _plan(lib, T=262144, H=32)[:2] == (kda.KDA_OK, 1)            # long_256k
    assert _plan(lib, T=262144, H=8)[:2] == (kda.KDA_OK, 2)             # long_256k_tp4
    assert _plan(lib, T=262144, H=4)[:2] == (kda.KDA_OK, 4)
    assert _plan(lib, T=262144, H=8, clusters=8)[:2] == (kda.KDA_OK, 1)
    assert _plan(lib, T=256, H=2)[:2] == (kda.KDA_OK, 1)                # too short to pay
    lens = [128 + (97 * i) % 16257 for i in range(64)]                   # a varlen batch
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    keep, cuh = _cu_host(cu)
    assert _plan(lib, cuh=cuh, B=0, T=0, N=64, H=32)[:2] == (kda.KDA_OK, 1)
    del keep
    # the same sizes as the device query reports for a given count
    st, P, nbytes = _plan(lib, T=262144, H=8)
    st2, P2, nbytes2 = _plan(lib, T=262144, H=8, n_split=2, clusters=0)   # count unused
    assert (st2, P2, nbytes2) == (st, P, nbytes)
    assert _plan(lib, clusters=0)[0] == kda.KDA_ERR_INVALID_ARG          # n_split 0 needs a count
    assert _plan(lib, clusters=-3)[0] == kda.KDA_ERR_INVALID_ARG
