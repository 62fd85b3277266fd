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


def kda_bwd_chunked(q, k, v, g, beta, dout, cu_seqlens, chunk: int = 64, scale: float | None = None,
                    eps: float = 1e-6, heads=None):
    """Chunked reverse-mode formulation of the KDA backward, numpy fp64 -- TEST INFRASTRUCTURE ONLY.

    The derivative of the chunked forward above, taken step by step.  A forward sweep keeps the
    state S entering every chunk; a reverse sweep carries dS, the gradient of the state leaving
    the chunk, and per chunk (dO = scale dout, QG = Q^ e^Gamma, Kd = K^ e^{Gamma_last - Gamma},
    D = e^{Gamma_last}):

      dU~ = A_qk^T dO + Kd dS                   dS_in = QG^T dO + D dS - W^T dU~
      dQG = dO S^T     dA_qk = lower(dO U~^T)   dKd = U~ dS^T   dGamma_last += D (S . dS)
      dW  = -dU~ S^T   dU = dU~                 dT = dW (beta KG)^T + dU (beta V)^T
      dA_kk = strict_lower(-T^T dT T^T)         (T = (I + A_kk)^-1)

    and then the chain rule through beta, the pairwise decays exp(Gamma_r - Gamma_i), the
    factors exp(Gamma) of KG, QG and Kd, the in-chunk cumsum (dg = reverse cumsum of dGamma) and
    the l2 norms.  Tests compare it with the token-recurrence backward ``oracle.kda_bwd``.
    Returns dq, dk, dv, dg, dbeta as in ``oracle.kda_bwd``.
    """
    q, k, v, g, beta, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta, dout))
    T, H, K = q.shape
    V = v.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    res = {n: np.full(s, np.nan) for n, s in (("dq", (T, H, K)), ("dk", (T, H, K)), ("dv", (T, H, V)),
                                               ("dg", (T, H, K)), ("dbeta", (T, H)))}
    heads = range(H) if heads is None else heads
    cu = [int(x) for x in cu_seqlens]
    for d in range(len(cu) - 1):
        for h in heads:
            starts = list(range(cu[d], cu[d + 1], chunk))
            S = np.zeros((K, V))
            S_in = []
            cache = []
            for s0 in starts:
                s1 = min(s0 + chunk, cu[d + 1])
                L = s1 - s0
                qc, kc, vc = q[s0:s1, h], k[s0:s1, h], v[s0:s1, h]
                rq = 1.0 / np.sqrt((qc * qc).sum(1, keepdims=True) + eps)
                rk = 1.0 / np.sqrt((kc * kc).sum(1, keepdims=True) + eps)
                qn, kn = qc * rq, kc * rk
                b = beta[s0:s1, h]
                G = np.cumsum(g[s0:s1, h], axis=0)
                lower = np.tril(np.ones((L, L), dtype=bool), -1)
                lower_eq = np.tril(np.ones((L, L), dtype=bool), 0)
                dec = np.where(lower_eq[:, :, None], np.exp(np.where(lower_eq[:, :, None],
                                                                     G[:, None, :] - G[None, :, :], 0.0)), 0.0)
                Ahat = np.einsum("rc,ic,ric->ri", kn, kn, dec)
                Akk = np.where(lower, b[:, None] * Ahat, 0.0)
                Aqk = np.einsum("rc,ic,ric->ri", qn, kn, dec)          # zero above the diagonal via dec
                Tm = np.linalg.inv(np.eye(L) + Akk)
                KG = kn * np.exp(G)
                W = Tm @ (b[:, None] * KG)
                U = Tm @ (b[:, None] * vc)
                Ut = U - W @ S
                S_in.append(S)
                cache.append((s0, s1, qn, kn, rq, rk, vc, b, G, dec, Ahat, Aqk, Tm, KG, W, Ut, lower))
                S = np.exp(G[-1])[:, None] * S + (kn * np.exp(G[-1][None, :] - G)).T @ Ut
            dS = np.zeros((K, V))
            for n in range(len(starts) - 1, -1, -1):
                s0, s1, qn, kn, rq, rk, vc, b, G, dec, Ahat, Aqk, Tm, KG, W, Ut, lower = cache[n]
                S = S_in[n]
                dO = scale * dout[s0:s1, h]
                eG = np.exp(G)
                QG = qn * eG
                Dl = np.exp(G[-1])
                Kd = kn * np.exp(G[-1][None, :] - G)
                dUt = Aqk.T @ dO + Kd @ dS
                dS_in = QG.T @ dO + Dl[:, None] * dS - W.T @ dUt
                dQG = dO @ S.T
                dAqk = np.tril(dO @ Ut.T)
                dKd = Ut @ dS.T
                dGl = Dl * (S * dS).sum(1)
                dW = -dUt @ S.T
                dU = dUt
                Bk, Bv = b[:, None] * KG, b[:, None] * vc
                dT = dW @ Bk.T + dU @ Bv.T
                dBk, dBv = Tm.T @ dW, Tm.T @ dU
                dvc = b[:, None] * dBv
                db = (dBv * vc).sum(1) + (dBk * KG).sum(1)
                dKG = b[:, None] * dBk
                dAkk = np.where(lower, -(Tm.T @ dT @ Tm.T), 0.0)
                db += (dAkk * Ahat).sum(1)
                dAh = b[:, None] * dAkk
                dkn = np.einsum("ri,ic,ric->rc", dAh, kn, dec) + np.einsum("ri,rc,ric->ic", dAh, kn, dec)
                dqn = np.einsum("ri,ic,ric->rc", dAqk, kn, dec)
                dkn += np.einsum("ri,rc,ric->ic", dAqk, qn, dec)
                ddec = (dAh[:, :, None] * kn[:, None, :] * kn[None, :, :]
                        + dAqk[:, :, None] * qn[:, None, :] * kn[None, :, :]) * dec
                dG = ddec.sum(1) - ddec.sum(0)
                dkn += dKG * eG
                dG += dKG * KG
                dqn += dQG * eG
                dG += dQG * QG
                dkn += dKd * np.exp(G[-1][None, :] - G)
                dG -= dKd * Kd
                dGl += (dKd * Kd).sum(0)
                dG[-1] += dGl
                dg = np.cumsum(dG[::-1], axis=0)[::-1]
                res["dq"][s0:s1, h] = rq * (dqn - qn * (qn * dqn).sum(1, keepdims=True))
                res["dk"][s0:s1, h] = rk * (dkn - kn * (kn * dkn).sum(1, keepdims=True))
                res["dv"][s0:s1, h] = dvc
                res["dg"][s0:s1, h] = dg
                res["dbeta"][s0:s1, h] = db
                dS = dS_in
    return res
