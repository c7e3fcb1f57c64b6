"""Test-only fp64 chunked (WY / UT) form of the KDA recurrence.

This is NOT the oracle. It restates the token recurrence (per-row decay, read-out,
correction scaled by beta, output from the updated state -- the sarnas.ru
article, section "Что именно изменилось", and m.lqnn.cn/news/205170, section
"KDA 与 Gated Attention：每 4 层只留 1 层全注意力") chunk by chunk, in the
algebra the CUDA prefill kernels use, so the tests can show on the CPU that the
algebra reproduces the token-by-token oracle before any kernel is trusted.

Per chunk of L tokens with state S (dk x dv) at its start, gamma_r = sum_{s<=r} g_s
(per key channel, within the chunk):
  A[r,i] = sum_c k[r,c] k[i,c] exp(gamma[r,c] - gamma[i,c])       (i < r)
  P[r,i] = sum_c q[r,c] k[i,c] exp(gamma[r,c] - gamma[i,c])       (i <= r)
  T      = (I + diag(beta) A)^-1                                  (unit lower triangular)
  W      = T diag(beta) (k * exp(gamma)),   U = T diag(beta) v
  Ut     = U - W S                         (row r equals beta_r * u_r)
  O      = scale * ((q * exp(gamma)) S + P Ut)
  S'     = diag(exp(gamma_last)) S + (k * exp(gamma_last - gamma))^T Ut
A and P are built in 16-token sub-blocks: an off-diagonal block (rows in sub-block R,
columns in an earlier sub-block I) uses the cumulative decay at the last token of I as
its reference point, so both factors exp(gamma_r - gamma_ref) and exp(gamma_ref - gamma_i)
are <= 1; a diagonal block forms exp(gamma_r - gamma_i) as a running product of exp(g).
"""
from __future__ import annotations

import numpy as np


def _chunk_AP(q, k, g, sub=16):
    L, dk = k.shape
    gam = np.cumsum(g, axis=0)
    A = np.zeros((L, L))
    P = np.zeros((L, L))
    a = np.exp(g)
    nsub = (L + sub - 1) // sub
    for Rb in range(nsub):
        r0, r1 = Rb * sub, min(L, (Rb + 1) * sub)
        for Ib in range(Rb):
            i0, i1 = Ib * sub, (Ib + 1) * sub
            ref = gam[i1 - 1]
            left_k = k[r0:r1] * np.exp(gam[r0:r1] - ref)
            left_q = q[r0:r1] * np.exp(gam[r0:r1] - ref)
            right = k[i0:i1] * np.exp(ref - gam[i0:i1])
            A[r0:r1, i0:i1] = left_k @ right.T
            P[r0:r1, i0:i1] = left_q @ right.T
        # diagonal block: D[r, i, :] = prod_{s=i+1..r} exp(g_s)
        for i in range(r0, r1):
            D = np.ones(dk)
            for r in range(i, r1):
                if r > i:
                    D = D * a[r]
                    A[r, i] = np.sum(k[r] * k[i] * D)
                P[r, i] = np.sum(q[r] * k[i] * D)
    return A, P, gam


def _unit_lower_inverse(M):
    """(I + M)^-1 for strictly lower triangular M by forward substitution."""
    L = M.shape[0]
    T = np.zeros((L, L))
    for r in range(L):
        T[r, r] = 1.0
        for i in range(r):
            T[r, i] = -np.dot(M[r, i:r], T[i:r, i])
    return T


def chunk_fwd(q, k, v, g, beta, scale=1.0, h0=None, cu_seqlens=None, chunk=64, sub=16):
    """Same signature and results (to rounding) as the oracle's kda_fwd."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T_tot, H, dk = q.shape
    dv = v.shape[2]
    cu = [0, T_tot] if cu_seqlens is None else [int(x) for x in cu_seqlens]
    N = len(cu) - 1
    o = np.zeros((T_tot, H, dv))
    ht = np.zeros((N, H, dk, dv))
    for n in range(N):
        for h in range(H):
            S = np.zeros((dk, dv)) if h0 is None else np.array(h0[n, h], dtype=np.float64)
            for c0 in range(cu[n], cu[n + 1], chunk):
                c1 = min(cu[n + 1], c0 + chunk)
                qc, kc, vc, gc, bc = (x[c0:c1, h] for x in (q, k, v, g, beta))
                A, P, gam = _chunk_AP(qc, kc, gc, sub)
                T = _unit_lower_inverse(bc[:, None] * A)
                W = T @ (bc[:, None] * (kc * np.exp(gam)))
                U = T @ (bc[:, None] * vc)
                Ut = U - W @ S
                o[c0:c1, h] = scale * ((qc * np.exp(gam)) @ S + P @ Ut)
                last = gam[-1]
                S = np.exp(last)[:, None] * S + (kc * np.exp(last - gam)).T @ Ut
            ht[n, h] = S
    return o, ht


def split_chunk_fwd(q, k, v, g, beta, scale=1.0, h0=None, chunk=64, half_range=80.0,
                    rounding=None):
    """The state-transition split that the bf16 prefill kernel computes, for one sequence.

    Per chunk, with gamma the within-chunk cumulative log-decay, gamma_C its last row and
    gamma_ref = gamma at the chunk middle (or 0 when some channel decays by more than
    `half_range` in either half of the chunk, the kernel's range test):
      Lk = k e^{gamma-gamma_ref}, Lq = q e^{gamma-gamma_ref}, R = k e^{gamma_ref-gamma},
      Rh = k e^{gamma_C-gamma};  A = strict lower part of Lk R^T, P = lower part of Lq R^T
      (formed exactly from e^{gamma_r-gamma_i} when the range test fails);
      T' = (I + diag(beta) A)^-1 diag(beta);  Yh^T = Rh^T T',  Wh^T = P T';
      Sm = S^T diag(e^{gamma_ref}),  X = Sm Lk^T,  U = V^T - X;
      S'^T = S^T diag(e^{gamma_C}) + U Yh,  O^T = scale (Sm Lq^T + U Wh).
    `rounding`, if given, is applied where the kernel rounds to bf16 (every tensor-core
    operand). Returns (o [T, H, dv], ht [1, H, dk, dv], number of chunks that failed the
    range test).
    """
    rnd = rounding or (lambda x: x)
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    o = np.zeros((T, H, dv))
    ht = np.zeros((1, H, dk, dv))
    nbad = 0
    for h in range(H):
        S = np.zeros((dk, dv)) if h0 is None else np.array(h0[0, h], dtype=np.float64)
        for c0 in range(0, T, chunk):
            L = min(chunk, T - c0)

            def pad(x, width):
                out = np.zeros((chunk, width))
                out[:L] = x[c0:c0 + L, h]
                return out

            qc, kc, vc, gc = pad(q, dk), pad(k, dk), pad(v, dv), pad(g, dk)
            bc = np.zeros(chunk)
            bc[:L] = beta[c0:c0 + L, h]
            gam = np.cumsum(gc, axis=0)
            g_half, g_last = gam[chunk // 2 - 1], gam[chunk - 1]
            bad = bool(np.any(g_half < -half_range) or np.any(g_last - g_half < -half_range))
            nbad += bad
            g_ref = np.zeros(dk) if bad else g_half
            Lk = rnd(kc * np.exp(gam - g_ref))
            Lq = rnd(qc * np.exp(gam - g_ref))
            Rh = rnd(kc * np.exp(g_last - gam))
            if bad:
                E = np.exp(gam[:, None, :] - gam[None, :, :])
                A = np.einsum('rc,ic,ric->ri', kc, kc, E)
                P = np.einsum('rc,ic,ric->ri', qc, kc, E)
            else:
                R = rnd(kc * np.exp(g_ref - gam))
                A = Lk @ R.T
                P = Lq @ R.T
            A = np.tril(A, -1)
            P = rnd(np.tril(P))
            Tp = rnd(np.linalg.inv(np.eye(chunk) + bc[:, None] * A) * bc[None, :])
            Yt = rnd(Rh.T @ Tp)                      # Yh^T [dk, chunk]
            Wt = rnd(P @ Tp)                         # Wh^T [chunk, chunk]
            Sm = rnd(S.T * np.exp(g_ref)[None, :])   # [dv, dk]
            U = rnd(vc.T - Sm @ Lk.T)                # [dv, chunk]
            Ot = scale * (Sm @ Lq.T + U @ Wt.T)      # [dv, chunk]
            o[c0:c0 + L, h] = Ot.T[:L]
            S = (S.T * np.exp(g_last)[None, :] + U @ Yt.T).T
        ht[0, h] = S
    return o, ht, nbad
