"""Brute-force explicit-product evaluation of the KDA recurrence — TEST INFRASTRUCTURE ONLY.

For one (sequence, head) unit with already-transformed inputs, every per-token transition is
formed as an explicit K x K matrix

    M_u = (I - beta_u khat_u khat_u^T) Diag(alpha_u)

and the state after token t is evaluated from prefix products,

    S_t = (M_t ... M_1) S_0 + sum_{s <= t} (M_t ... M_{s+1}) beta_s khat_s v_s^T,
    o_t = scale * S_t^T qhat_t,

which is the closed form of the recurrence S_t = M_t S_{t-1} + beta_t khat_t v_t^T that the
Kimi Delta Attention operator (FlashKDA `fwd`, fla `chunk_kda`) computes.  It is O(T^2 K^3) and
meant for T <= 8; it shares no evaluation order with the C oracle, which updates S in place.
"""
from __future__ import annotations

import numpy as np


def explicit_products(qhat, khat, v, log_alpha, beta, scale, S0=None):
    """qhat, khat, log_alpha: [T, K]; v: [T, V]; beta: [T]; S0: [K, V] or None.
    Returns (o [T, V], S_T [K, V]) in fp64."""
    qhat, khat, v, log_alpha = (np.asarray(x, dtype=np.float64) for x in (qhat, khat, v, log_alpha))
    beta = np.asarray(beta, dtype=np.float64)
    T, K = khat.shape
    V = v.shape[1]
    S0 = np.zeros((K, V)) if S0 is None else np.asarray(S0, dtype=np.float64)
    eye = np.eye(K)
    M = [(eye - beta[u] * np.outer(khat[u], khat[u])) @ np.diag(np.exp(log_alpha[u]))
         for u in range(T)]

    def prefix(t, s):
        """M_t M_{t-1} ... M_{s+1} (0-based token indices; identity when s == t)."""
        P = eye.copy()
        for u in range(s + 1, t + 1):
            P = M[u] @ P
        return P

    o = np.zeros((T, V))
    S_t = S0
    for t in range(T):
        S_t = prefix(t, -1) @ S0
        for s in range(t + 1):
            S_t = S_t + prefix(t, s) @ (beta[s] * np.outer(khat[s], v[s]))
        o[t] = scale * (S_t.T @ qhat[t])
    return o, S_t
