"""Independent re-derivations of the KDA core, used only to pin the oracle.

Each is a different algebraic form of the same recurrence, written separately from
oracle/kda_recurrence.c, so that a dropped term, a wrong sign or a transposed operand
in one of them shows up as a disagreement:

  * brute_force: the state as an explicit sum of products of D x D transition matrices,
        S_t = A_t S_{t-1} + B_t,  A_t = (I - beta_t k_t k_t^T) diag(exp g_t),  B_t = beta_t k_t v_t^T;
  * chunked_wy:  the chunked form (chunks of C tokens): in-chunk cumulative log-decay
        Gamma, the unit-lower-triangular system (I + L) U = diag(beta)(V - (K*e^Gamma) S0)
        solved by a triangular inverse (the WY/UT representation), inter-chunk read-out
        O = (Q*e^Gamma) S0 + M U and the chunk-end state update.
"""
from __future__ import annotations

import numpy as np


def brute_force(q, k, v, g, beta, s0, scale=1.0):
    """One head: q, k, v, g [T, D]; beta [T]; s0 [D, D]. Returns (o [T, D], S_T)."""
    T, D = q.shape
    I = np.eye(D)
    A = [(I - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) for t in range(T)]
    B = [beta[t] * np.outer(k[t], v[t]) for t in range(T)]
    o = np.zeros((T, D))
    S_t = s0
    for t in range(T):
        # S_t = sum_{j<=t} (A_t ... A_{j+1}) B_j + (A_t ... A_0) S0
        S = np.zeros((D, D))
        P = np.eye(D)
        for j in range(t, -1, -1):
            S = S + P @ B[j]
            P = P @ A[j]
        S_t = S + P @ s0
        o[t] = scale * (S_t.T @ q[t])
    return o, S_t


def chunked_wy(q, k, v, g, beta, s0, scale=1.0, C=64):
    """One head, chunked WY/UT form. Shapes as brute_force. Returns (o, S_T)."""
    T, D = q.shape
    S = np.array(s0, dtype=np.float64, copy=True)
    o = np.zeros((T, D))
    for n0 in range(0, T, C):
        sl = slice(n0, min(n0 + C, T))
        Q, K, V, G, b = q[sl], k[sl], v[sl], g[sl], beta[sl]
        n = Q.shape[0]
        Gam = np.cumsum(G, axis=0)                      # inclusive, per channel
        diff = Gam[:, None, :] - Gam[None, :, :]        # Gamma_i - Gamma_j
        lower = np.tril(np.ones((n, n), dtype=bool))
        E = np.where(lower[:, :, None], np.exp(np.where(lower[:, :, None], diff, 0.0)), 0.0)
        KK = np.einsum("ic,jc,ijc->ij", K, K, E)
        L = np.tril(b[:, None] * KK, -1)
        M = np.einsum("ic,jc,ijc->ij", Q, K, E)         # includes the diagonal
        A = np.exp(Gam)
        Tinv = np.linalg.inv(np.eye(n) + L)
        W = Tinv @ (b[:, None] * K * A)
        Ut = Tinv @ (b[:, None] * V)
        U = Ut - W @ S
        o[sl] = scale * ((Q * A) @ S + M @ U)
        S = np.exp(Gam[-1])[:, None] * S + (K * np.exp(Gam[-1][None, :] - Gam)).T @ U
    return o, S


def _chunk_terms(Q, K, V, G, b):
    """The per-chunk WY/UT quantities of chunked_wy: A = e^Gamma, a = e^{Gamma_C}, K-bar =
    K o e^{Gamma_C - Gamma}, M, W, U~ (the state-independent part of a chunk)."""
    n = Q.shape[0]
    Gam = np.cumsum(G, axis=0)
    diff = Gam[:, None, :] - Gam[None, :, :]
    lower = np.tril(np.ones((n, n), dtype=bool))
    E = np.where(lower[:, :, None], np.exp(np.where(lower[:, :, None], diff, 0.0)), 0.0)
    L = np.tril(b[:, None] * np.einsum("ic,jc,ijc->ij", K, K, E), -1)
    M = np.einsum("ic,jc,ijc->ij", Q, K, E)
    A = np.exp(Gam)
    Tinv = np.linalg.inv(np.eye(n) + L)
    return dict(QA=Q * A, a=np.exp(Gam[-1]), Kbar=K * np.exp(Gam[-1][None, :] - Gam), M=M,
                W=Tinv @ (b[:, None] * K * A), Ut=Tinv @ (b[:, None] * V))


def chunked_lookahead(q, k, v, g, beta, s0, scale=1.0, C=64):
    """One head, the chunked form with the inter-chunk chain carried by U instead of S:
        U_{c+1} = U~_{c+1} - W_{c+1} (a_c o S_c) - Z_{c+1} U_c,   Z_{c+1} = W_{c+1} K-bar_c^T,
    where the state update S_{c+1} = a_c o S_c + K-bar_c^T U_c and the product W_{c+1}(a_c o S_c)
    both use S_c, one step behind the chain (a state pass built this way has one dependent
    product and one epilogue per chunk on its critical path). Shapes as brute_force."""
    T, D = q.shape
    ch = [_chunk_terms(q[n0:n0 + C], k[n0:n0 + C], v[n0:n0 + C], g[n0:n0 + C], beta[n0:n0 + C])
          for n0 in range(0, T, C)]
    S = np.array(s0, dtype=np.float64, copy=True)
    o = np.zeros((T, D))
    U = ch[0]["Ut"] - ch[0]["W"] @ S
    for c, t in enumerate(ch):
        n0 = c * C
        o[n0:n0 + t["M"].shape[0]] = scale * (t["QA"] @ S + t["M"] @ U)
        aS = t["a"][:, None] * S
        if c + 1 < len(ch):
            nx = ch[c + 1]
            Z = nx["W"] @ t["Kbar"].T
            U_next = nx["Ut"] - nx["W"] @ aS - Z @ U
        S = aS + t["Kbar"].T @ U
        if c + 1 < len(ch):
            U = U_next
    return o, S

