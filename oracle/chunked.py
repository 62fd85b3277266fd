"""Chunked UT/WY formulation of the KDA forward, numpy fp64 -- TEST INFRASTRUCTURE ONLY.

An independent second formulation of the recurrence in ``kda_oracle.c``.  It is
exact algebra (the same result up to rounding order), reached by unrolling the
token recurrence inside a chunk of C tokens.  With Gamma_r the inclusive
in-chunk cumulative sum of the log decay g (per key channel), rows r, i of
the chunk, S the state entering the chunk:

  A_kk[r,i] = beta_r sum_c k^_rc k^_ic exp(Gamma_rc - Gamma_ic)        (i < r)
  A_qk[r,i] =        sum_c q^_rc k^_ic exp(Gamma_rc - Gamma_ic)        (i <= r)
  T  = (I + A_kk)^-1                        (the UT transform)
  W  = T diag(beta) (K^ * exp(Gamma)),  U = T diag(beta) V        (WY factors)
  U~ = U - W S                              (the chunk's corrected values)
  O  = (Q^ * exp(Gamma)) S + A_qk U~
  S <- Diag(exp(Gamma_last)) S + (K^ * exp(Gamma_last - Gamma))^T U~

Chunks start at each document start, so the last chunk of a document may be
short.  Used only by the tests, to check the recurrence oracle against a
different algorithm (and so to confirm the algebra the CUDA kernels follow).
"""
from __future__ import annotations

import numpy as np


def kda_fwd_chunked(q, k, v, g, beta, cu_seqlens, chunk: int = 64, scale: float | None = None,
                    eps: float = 1e-6, heads=None):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    T, H, K = q.shape
    V = v.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    out = np.full((T, H, V), np.nan)
    heads = range(H) if heads is None else heads
    cu = [int(x) for x in cu_seqlens]
    for d in range(len(cu) - 1):
        for h in heads:
            S = np.zeros((K, V))
            for s0 in range(cu[d], cu[d + 1], chunk):
                s1 = min(s0 + chunk, cu[d + 1])
                L = s1 - s0
                qc, kc, vc = q[s0:s1, h], k[s0:s1, h], v[s0:s1, h]
                qn = qc / np.sqrt((qc * qc).sum(1, keepdims=True) + eps)
                kn = kc / np.sqrt((kc * kc).sum(1, keepdims=True) + eps)
                b = beta[s0:s1, h]
                G = np.cumsum(g[s0:s1, h], axis=0)
                diff = G[:, None, :] - G[None, :, :]          # [r, i, c]
                lower = np.tril(np.ones((L, L), dtype=bool), -1)
                lower_eq = np.tril(np.ones((L, L), dtype=bool), 0)
                dec = np.exp(np.where(lower_eq[:, :, None], diff, 0.0))
                Akk = b[:, None] * np.einsum("rc,ic,ric->ri", kn, kn, dec)
                Akk = np.where(lower, Akk, 0.0)
                Aqk = np.where(lower_eq, np.einsum("rc,ic,ric->ri", qn, kn, dec), 0.0)
                Tm = np.linalg.inv(np.eye(L) + Akk)
                W = Tm @ (b[:, None] * kn * np.exp(G))
                U = Tm @ (b[:, None] * vc)
                Ut = U - W @ S
                O = (qn * np.exp(G)) @ S + Aqk @ Ut
                out[s0:s1, h] = scale * O
                S = np.exp(G[-1])[:, None] * S + (kn * np.exp(G[-1][None, :] - G)).T @ Ut
    return out
