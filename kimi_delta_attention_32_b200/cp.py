"""Context-parallel prefill over ranks: every rank holds one stretch of each sequence.

The KDA recurrence (sarnas.ru, "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base ...",
section "Что именно изменилось"; m.lqnn.cn/news/205170, section "KDA 与 Gated Attention ...")
maps the state affinely at every token, so the stretch on rank r, started from S, ends in
M_r S + Z_r and emits o_t(from zero) + S^T w_t, with w_t = scale M_t^T q_t. The model is
trained at contexts up to 256K tokens (sarnas.ru, section "Как проходило обучение"); a context
too long for one GPU's time budget is cut along time:

1. each rank runs its stretches from a zero state: outputs, end states Z_r, transitions M_r
   and carried-back queries w (kda_chunk_states, one launch);
2. the ranks all-gather (M_r, Z_r): 64 KiB each per (sequence, head) and rank for d = 128;
3. each rank joins the stretches before its own (kda_state_scan):
   H_0 = h0, H_{p+1} = M_p H_p + Z_p;
4. each rank adds its entering state's share to its outputs, o_t += H_r^T w_t
   (kda_output_correct, a dense product on the tensor cores).

Rank r's tensors are its own tokens of every sequence, in packed layout with cu_seqlens /
cu_host (a sequence may have no tokens on a rank). Every rank gets the final states ht (after
the last rank's stretch). The exchange is the only collective, and every rank takes it once
per call, in the same order.

The ops argument exists for the host-side tests, which run the steps on CPU stand-ins; by
default every step is a libkda call on the current CUDA stream (and fails loudly without the
library).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class _LibkdaOps:
    """The steps as libkda calls."""

    def __init__(self):
        from . import kda
        self.kda = kda

    def chunk_states(self, q, k, v, g, beta, scale, cu_seqlens, cu_host):
        z, m, o, w = self.kda.chunk_states(q, k, v, g, beta, scale, h0=None, cu_seqlens=cu_seqlens,
                                           cu_host=cu_host, output=True, carried_queries=True)
        return z, m, o, w

    def state_scan(self, m, z, h0, N, P, seq_stride, seg_stride):
        return self.kda.state_scan(m, z, h0, N=N, P=P, seq_stride=seq_stride,
                                   seg_stride=seg_stride)

    def output_correct(self, w, h, o, cu_seqlens, cu_host):
        return self.kda.output_correct(w, h, o, cu_seqlens, cu_host)


def chunk_fwd_cp(q, k, v, g, beta, scale=1.0, h0=None, cu_seqlens=None, cu_host=None,
                 group=None, ops=None):
    """Prefill of this rank's stretch of every sequence. q, k, g: [T_r, H, dk] packed with
    cu_seqlens (device) and cu_host (list); v: [T_r, H, dv]; h0: [N, H, dk, dv] or None, the
    same on every rank. Returns (o of this rank's tokens, ht [N, H, dk, dv])."""
    ops = ops if ops is not None else _LibkdaOps()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    z, m, o, w = ops.chunk_states(q, k, v, g, beta, scale, cu_seqlens, cu_host)
    N = z.shape[0]
    zs = [torch.empty_like(z) for _ in range(world)]
    ms = [torch.empty_like(m) for _ in range(world)]
    dist.all_gather(zs, z.contiguous(), group=group)
    dist.all_gather(ms, m.contiguous(), group=group)
    # stretch p of sequence n is index p * N + n of the gathered stacks
    h_start, ht = ops.state_scan(torch.cat(ms), torch.cat(zs), h0, N, world, 1, N)
    o = ops.output_correct(w, h_start[rank * N:(rank + 1) * N].contiguous(), o, cu_seqlens,
                           cu_host)
    return o, ht
