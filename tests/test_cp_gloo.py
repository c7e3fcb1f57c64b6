"""The context-parallel prefill's orchestration (kimi_delta_attention_32_b200.cp) on CPU: ranks
as gloo processes, each holding one stretch of every sequence, with the steps run by fp64
stand-ins written from the oracle (the stretch from a zero state with its transition and
carried-back queries, the join, the output correction).
The assembled outputs and final states must equal the oracle run over whole sequences: this
checks which stretch each rank forms, the order of the all-gather, the join's indexing and the
output correction's entering states.
The libkda steps themselves are checked against the oracle on the GPU."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from kimi_delta_attention_32_b200 import cp

LENS = [40, 17, 0, 9]          # tokens per sequence (one empty)
H, DK, DV = 2, 5, 4


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(61)
    T = sum(LENS)
    q = rng.standard_normal((T, H, DK))
    k = rng.standard_normal((T, H, DK))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, DV))
    g = np.log(1.0 / (1.0 + np.exp(-rng.normal(3.0, 1.0, (T, H, DK)))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    h0 = rng.normal(0.0, 0.5, (len(LENS), H, DK, DV))
    return q, k, v, g, beta, h0


def _cuts(world):
    """Token bounds of each rank's stretch of each sequence: uneven, some empty."""
    cuts = []
    for n, L in enumerate(LENS):
        c = sorted(np.random.default_rng(70 + n).integers(0, L + 1, world - 1).tolist())
        cuts.append([0, *c, L])
    return cuts


class _OracleOps:
    """fp64 stand-ins for the libkda steps (test infrastructure only)."""

    def chunk_states(self, q, k, v, g, beta, scale, cu_seqlens, cu_host):
        a = [x.numpy() for x in (q, k, v, g, beta)]
        o, z = oracle.kda_fwd(*a, scale, None, cu_host, nthreads=1)
        m = oracle.transition(a[1], a[3], a[4], cu_host, nthreads=1)
        # the queries carried back to each stretch's start: the output of the run with v = 0
        # started from the identity
        eye = np.broadcast_to(np.eye(DK), (len(cu_host) - 1, H, DK, DK))
        w, _ = oracle.kda_fwd(a[0], a[1], np.zeros_like(a[0]), a[3], a[4], scale, eye, cu_host,
                              nthreads=1)
        return (torch.from_numpy(z), torch.from_numpy(m), torch.from_numpy(o),
                torch.from_numpy(w))

    def state_scan(self, m, z, h0, N, P, seq_stride, seg_stride):
        m, z = m.numpy(), z.numpy()
        hs = np.zeros_like(z)
        ht = np.zeros((N, *z.shape[1:]))
        for n in range(N):
            cur = np.zeros(z.shape[1:]) if h0 is None else h0[n].numpy()
            for p in range(P):
                j = n * seq_stride + p * seg_stride
                hs[j] = cur
                cur = np.einsum("hij,hjc->hic", m[j], cur) + z[j]
            ht[n] = cur
        return torch.from_numpy(hs), torch.from_numpy(ht)

    def output_correct(self, w, h, o, cu_seqlens, cu_host):
        w, h, o = w.numpy(), h.numpy(), o.numpy().copy()
        for n in range(len(cu_host) - 1):
            sl = slice(cu_host[n], cu_host[n + 1])
            o[sl] += np.einsum("thi,hic->thc", w[sl], h[n])
        return torch.from_numpy(o)


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, g, beta, h0 = _inputs()
        cuts = _cuts(world)
        cu = np.concatenate([[0], np.cumsum(LENS)])
        idx = np.concatenate([np.arange(cu[n] + cuts[n][rank], cu[n] + cuts[n][rank + 1])
                              for n in range(len(LENS))]).astype(np.int64)
        cu_r = [0]
        for n in range(len(LENS)):
            cu_r.append(cu_r[-1] + cuts[n][rank + 1] - cuts[n][rank])
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x[idx]))
        o, ht = cp.chunk_fwd_cp(t(q), t(k), t(v), t(g), t(beta), 0.75, torch.from_numpy(h0),
                                cu_seqlens=None, cu_host=cu_r, ops=_OracleOps())
        out[rank] = (idx.tolist(), o.numpy().tolist(), ht.numpy().tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_prefill_equals_whole_sequences(world):
    q, k, v, g, beta, h0 = _inputs()
    cu = np.concatenate([[0], np.cumsum(LENS)])
    o_ref, ht_ref = oracle.kda_fwd(q, k, v, g, beta, 0.75, h0, cu)
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    o = np.full_like(o_ref, np.nan)
    for r in range(world):
        idx, o_r, ht_r = res[r]
        o[np.asarray(idx, dtype=np.int64)] = np.asarray(o_r).reshape(-1, H, DV)
        np.testing.assert_allclose(np.asarray(ht_r), ht_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
