"""Brute-force fp64 evaluation of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Independent of the C oracle: every token's transition matrix is formed as an
explicit d_k x d_k matrix and the state at step t is expanded as

    S_t = (A_t ... A_1) S_0 + sum_{i<=t} (A_t ... A_{i+1}) beta_i k_i v_i^T

with A_i = Diag(a_i)(I - beta_i k_i k_i^T) for the operator order of the KDA
row of the table "Everything, in one table" (thethings.ai, "The argument, in
one page"), A_i = (I - beta_i k_i k_i^T) Diag(a_i) for the other order, and
A_i = Diag(a_i) when the erase term is removed (the "Linear attention" row,
gated).  Every product is recomputed from scratch for each t, so the cost is
O(T^2 d^3): tiny T only.
"""
from __future__ import annotations

import numpy as np


def _transition(k, beta, a, order, rule):
    d_k = k.shape[0]
    D = np.diag(a)
    if rule == "linear":
        return D
    E = np.eye(d_k) - beta * np.outer(k, k)
    if order == "erase_then_decay":
        return D @ E
    if order == "decay_then_erase":
        return E @ D
    raise ValueError(order)


def transition_products(q, k, v, g, beta, s0=None, *, order="erase_then_decay",
                        rule="delta"):
    """One chain: q, k [T, d_k]; v [T, d_v]; g [T, d_k] or [T]; beta [T];
    s0 [d_k, d_v] or None.  Returns (o [T, d_v], S_T [d_k, d_v])."""
    q, k, v, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, beta))
    g = np.asarray(g, dtype=np.float64)
    T, d_k = k.shape
    d_v = v.shape[1]
    if g.ndim == 1:
        g = np.repeat(g[:, None], d_k, axis=1)
    S0 = np.zeros((d_k, d_v)) if s0 is None else np.asarray(s0, dtype=np.float64)
    A = [_transition(k[i], beta[i], np.exp(g[i]), order, rule) for i in range(T)]
    W = [beta[i] * np.outer(k[i], v[i]) for i in range(T)]
    o = np.zeros((T, d_v))
    St = S0
    for t in range(T):
        P = np.eye(d_k)
        for i in range(t, -1, -1):          # P = A_t ... A_0 (0-based)
            P = P @ A[i]
        St = P @ S0
        for i in range(t + 1):
            Pi = np.eye(d_k)
            for j in range(t, i, -1):       # A_t ... A_{i+1}
                Pi = Pi @ A[j]
            St = St + Pi @ W[i]
        o[t] = St.T @ q[t]
    return o, St
