"""fp64 chunkwise (WY / UT) form of the gated delta rule -- TEST INFRASTRUCTURE.

A second CPU path, written from the chunk equations of "Reading notes: Kimi
Delta Attention" (mzeromiko), section 4 "Forward pass" (the matrix form of
S_[t]^C and O_[t], the U_[t] / W_[t] solve and the matrix A~_[t]), in the
d_v x d_k orientation.  It exists only to pin the recurrence in
``gdr_oracle.c`` (the two must agree for every chunk size); it is not the
parity reference of the CUDA library and the CUDA library does not use it.

Per chunk (rows r = 1..C of the chunk, G_r = sum_{j<=r} log alpha_j per key
channel, gamma_r = exp(G_r), Gamma stacks the gamma_r as rows):
    K<- = K * Gamma,  K-> = K / Gamma,  Q<- = Q * Gamma
    A~  = (I + Diag(beta) (K<- K->^T * M_{-1}))^{-1}        (M_{-1}: strictly lower)
    W   = A~ Diag(beta) K<-,     U = A~ Diag(beta) V
    S_next = S Diag(gamma_C) + (U^T - S W^T) K-> Diag(gamma_C)
    O   = Q<- S^T + (Q<- K->^T * M)(U - W S^T)                (M: lower incl. diagonal)
No rescaling is done: fp64 holds gamma down to exp(-5*C) for the chunk sizes
the pins use.  A last partial chunk simply has fewer rows.
"""
from __future__ import annotations

import numpy as np


def chunk_forward(q, k, v, g, beta, S0=None, C: int = 64, gate: str = "per_channel", clamp: bool = True):
    """q,k [T,dk]; v [T,dv]; g [T,dk] or [T]; beta [T]; S0 [dv,dk]. One head, fp64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    if gate == "per_channel":
        logalpha = np.maximum(g, -5.0) if clamp else g.copy()
    else:
        logalpha = np.repeat(g[:, None], dk, axis=1)
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, np.float64)
    O = np.zeros((T, dv))
    for s in range(0, T, C):
        e = min(T, s + C)
        n = e - s
        Q, K, V, b = q[s:e], k[s:e], v[s:e], beta[s:e]
        G = np.cumsum(logalpha[s:e], axis=0)          # [n, dk]
        Gam = np.exp(G)
        Kl = K * Gam                                  # K<-
        Kr = K / Gam                                  # K->
        Ql = Q * Gam                                  # Q<-
        strict = np.tril(np.ones((n, n)), -1)
        lower = np.tril(np.ones((n, n)), 0)
        Atil = np.linalg.inv(np.eye(n) + np.diag(b) @ ((Kl @ Kr.T) * strict))
        W = Atil @ np.diag(b) @ Kl
        U = Atil @ np.diag(b) @ V
        Vnew = U - W @ S.T                            # pseudo-value
        O[s:e] = Ql @ S.T + ((Ql @ Kr.T) * lower) @ Vnew
        gC = Gam[-1]
        S = S * gC[None, :] + (Vnew.T @ Kr) * gC[None, :]
    return O, S


def chunk_forward_gdr2(q, k, v, g, b, w, S0=None, C: int = 64, gate: str = "per_channel", clamp: bool = True):
    """Gated Delta Rule-2 in chunk form, one head, fp64: the equations of
    "Token Mixer I", section "Gated DeltaNet-2", subsection "Chunkwise parallel
    training", in the d_v x d_k orientation.  Per chunk, with the state
    normalised by the cumulative decay (S_r = S^_r Diag(gamma_r)):
        E- = B * K * Gamma (erase-side keys),  K-> = K / Gamma,  Z = W * V
        T  = StrictTril(E- K->^T),  A = (I + T)^{-1}   (forward substitution)
        Y  = A E-  (erase side),    U = A Z  (write side)
        Delta  = U - Y S^T
        S_next = S Diag(gamma_C) + Delta^T K_tail,   K_tail_r = k_r * gamma_C / gamma_r
        O      = Q_gamma S^T + (Q_gamma K->^T * M) Delta   (M: lower incl. diagonal)
    b, q, k [T,dk]; w, v [T,dv]; g [T,dk] or [T]; S0 [dv,dk]."""
    q, k, v, g, b, w = (np.asarray(x, np.float64) for x in (q, k, v, g, b, w))
    T, dk = q.shape
    dv = v.shape[1]
    if gate == "per_channel":
        logalpha = np.maximum(g, -5.0) if clamp else g.copy()
    else:
        logalpha = np.repeat(g[:, None], dk, axis=1)
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, np.float64)
    O = np.zeros((T, dv))
    for s in range(0, T, C):
        e = min(T, s + C)
        n = e - s
        G = np.cumsum(logalpha[s:e], axis=0)
        Gam = np.exp(G)
        Ebar = b[s:e] * k[s:e] * Gam
        Kbar = k[s:e] / Gam
        Z = w[s:e] * v[s:e]
        Tm = np.tril(Ebar @ Kbar.T, -1)
        # A = (I + T)^{-1}: forward substitution, column by column
        A = np.zeros((n, n))
        for j in range(n):
            x = np.zeros(n)
            x[j] = 1.0
            for r in range(j + 1, n):
                x[r] = -Tm[r, j:r] @ x[j:r]
            A[:, j] = x
        Y = A @ Ebar
        U = A @ Z
        Delta = U - Y @ S.T
        Qg = q[s:e] * Gam
        O[s:e] = Qg @ S.T + ((Qg @ Kbar.T) * np.tril(np.ones((n, n)))) @ Delta
        Ktail = k[s:e] * (Gam[-1][None, :] / Gam)
        S = S * Gam[-1][None, :] + Delta.T @ Ktail
    return O, S
