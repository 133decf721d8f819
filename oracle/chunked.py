"""Chunked (WY-form) gated delta rule for one head, float64 numpy.

Test infrastructure only (see the package docstring).

The chunkwise-parallel form of DeltaNet / Gated DeltaNet (Yang et al., "Parallelizing
Linear Transformers with the Delta Rule over Sequence Length", 2024, and "Gated Delta
Networks", 2024), restated for S in R^{dv x dk}. Within a chunk of C tokens with
incoming state S0, let Gamma_r = sum_{s<=r} log a_s and gamma_r = e^{Gamma_r}. With
delta_r = b_r (v_r - a_r S_{r-1} k_r) the recurrence unrolls to

    S_r = gamma_r S0 + sum_{i<=r} e^{Gamma_r - Gamma_i} delta_i k_i^T,

and stacking the delta_r as rows of Delta gives the unit-lower-triangular system

    (I + A) Delta = diag(b) V - diag(b gamma) K S0^T,
    A_ri = b_r e^{Gamma_r - Gamma_i} (k_r . k_i)  for i < r,  0 otherwise.

Outputs and carried state:

    O   = diag(gamma) Q S0^T + (Q K^T (.) M) Delta,   M_ri = e^{Gamma_r - Gamma_i}, i <= r
    S_C = gamma_C S0 + Delta^T diag(e^{Gamma_C - Gamma}) K.

Only differences Gamma_r - Gamma_i with i <= r are exponentiated, so no factor exceeds 1.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

__all__ = ["deltanet_chunked", "deltanet_recurrent"]


def deltanet_recurrent(S0, Q, K, V, a, b):
    """Reference loop: S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t.

    Q, K: [T, dk]; V: [T, dv]; a, b: [T]. Returns (O [T, dv], S_T).
    """
    S = np.array(S0, dtype=np.float64, copy=True)
    O = np.empty((Q.shape[0], V.shape[1]))
    for t in range(Q.shape[0]):
        S = a[t] * S - b[t] * np.outer(a[t] * S @ K[t], K[t]) + b[t] * np.outer(V[t], K[t])
        O[t] = S @ Q[t]
    return O, S


def _one_chunk(S0, Q, K, V, a, b):
    C = Q.shape[0]
    G = np.cumsum(np.log(a))                       # Gamma_r, r = 1..C
    gam = np.exp(G)
    diff = G[:, None] - G[None, :]                 # Gamma_r - Gamma_i
    lower = np.tril(np.ones((C, C), dtype=bool))
    M = np.where(lower, np.exp(np.where(lower, diff, 0.0)), 0.0)
    strict = np.tril(np.ones((C, C), dtype=bool), k=-1)
    A = np.where(strict, b[:, None] * M * (K @ K.T), 0.0)
    rhs = b[:, None] * V - (b * gam)[:, None] * (K @ S0.T)
    Delta = solve_triangular(np.eye(C) + A, rhs, lower=True, unit_diagonal=True)
    O = gam[:, None] * (Q @ S0.T) + ((Q @ K.T) * M) @ Delta
    w = np.exp(G[-1] - G)                          # e^{Gamma_C - Gamma_i}
    S_C = gam[-1] * S0 + Delta.T @ (w[:, None] * K)
    return O, S_C


def deltanet_chunked(S0, Q, K, V, a, b, chunk: int):
    """WY-form evaluation over chunks of ``chunk`` tokens (the last may be short).

    Same arguments and results as ``deltanet_recurrent``.
    """
    T = Q.shape[0]
    S = np.array(S0, dtype=np.float64, copy=True)
    O = np.empty((T, V.shape[1]))
    for s in range(0, T, chunk):
        e = min(T, s + chunk)
        O[s:e], S = _one_chunk(S, Q[s:e], K[s:e], V[s:e], a[s:e], b[s:e])
    return O, S
