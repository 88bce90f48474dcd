"""The chunked (WY / UT) form of the KDA recurrence — TEST INFRASTRUCTURE ONLY.

This restates, for one (sequence, head) unit, the chunk-parallel algorithm that fla's
`chunk_kda` names: the recurrence is cut into chunks of C tokens; inside a chunk the per-token
delta corrections are solved for at once through a unit lower-triangular system, and only the
state crosses chunk boundaries.  It is used to pin the algebra the GPU kernel relies on against
the token recurrence, and to check that the exponent referencing keeps every intermediate
finite in float32.

Derivation (per chunk, rows r = 1..C, S0 the state entering the chunk):
  Gamma_r   = sum_{s <= r} log alpha_s                  (per channel, inclusive)
  delta_r   = beta_r (v_r - S_{r-1}^T Diag(alpha_r) k_r)
  S_r       = Diag(e^{Gamma_r}) S0 + sum_{s <= r} Diag(e^{Gamma_r - Gamma_s}) k_s delta_s^T
  (I + A) Delta = diag(beta) (V - (K * e^Gamma) S0),  A_rs = beta_r sum_c k_rc k_sc e^{Gamma_rc - Gamma_sc}  (s < r)
  T = (I + A)^{-1},  W = T diag(beta) (K * e^Gamma),  U = T diag(beta) V,  Delta = U - W S0
  O   = scale [ (Q * e^Gamma) S0 + tril_incl((Q * e^Gamma)(K * e^{-Gamma})^T) Delta ]
  S_C = Diag(e^{Gamma_C}) S0 + (K * e^{Gamma_C - Gamma})^T Delta

Exponent referencing (``blocked=True``): e^{+-Gamma} over a 64-token chunk can reach e^{320},
beyond float32.  The chunk is cut into sub-blocks of ``block`` rows.  For rows r of sub-block I,
the pair products with columns s <= end(I) use the reference m_{I-1} (Gamma at the last row of
the previous sub-block, 0 for the first):
    left  = k_r e^{Gamma_r - m_{I-1}}   in [e^{-5*block}, 1]
    right = k_s e^{m_{I-1} - Gamma_s}   <= 1 for s before sub-block I, <= e^{5*block} inside it
so no factor overflows for |log alpha| <= 5 and block <= 16, and a factor underflows only where
the exact product is below float32's range anyway.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def chunk_intermediates(qhat, khat, v, log_alpha, beta, scale, C, blocked=False, block=16,
                        dtype=np.float64):
    """Per-chunk quantities for one unit: a list of dicts with Gamma, A, P, T, W, U, Qt, Kt, gC.

    qhat, khat, log_alpha: [L, K]; v: [L, V]; beta: [L].  Rows past the end of the last (partial)
    chunk are simply absent (the chunk is shorter).
    """
    f = lambda x: np.asarray(x, dtype=dtype)
    qhat, khat, v, log_alpha, beta = map(f, (qhat, khat, v, log_alpha, beta))
    L = khat.shape[0]
    out = []
    for c0 in range(0, L, C):
        c1 = min(c0 + C, L)
        n = c1 - c0
        q, k, vv, la, b = qhat[c0:c1], khat[c0:c1], v[c0:c1], log_alpha[c0:c1], beta[c0:c1]
        G = np.cumsum(la, axis=0, dtype=dtype)
        if not blocked:
            KG = k * np.exp(G)
            KGinv = k * np.exp(-G)
            A = np.tril(b[:, None] * (KG @ KGinv.T), -1)
            P = np.tril((q * np.exp(G)) @ KGinv.T) * dtype(scale)
        else:
            A = np.zeros((n, n), dtype=dtype)
            P = np.zeros((n, n), dtype=dtype)
            for i0 in range(0, n, block):
                i1 = min(i0 + block, n)
                ref = G[i0 - 1] if i0 > 0 else np.zeros(G.shape[1], dtype=dtype)
                left_k = k[i0:i1] * np.exp(G[i0:i1] - ref)
                left_q = q[i0:i1] * np.exp(G[i0:i1] - ref)
                right = k[:i1] * np.exp(ref - G[:i1])
                Ak = left_k @ right.T
                Aq = left_q @ right.T
                rows = np.arange(i0, i1)[:, None]
                cols = np.arange(i1)[None, :]
                A[i0:i1, :i1] = np.where(cols < rows, b[i0:i1, None] * Ak, 0)
                P[i0:i1, :i1] = np.where(cols <= rows, Aq * dtype(scale), 0)
        I = np.eye(n, dtype=dtype)
        T = solve_triangular(I + A, I, lower=True, unit_diagonal=True)
        KG = k * np.exp(G)
        W = T @ (b[:, None] * KG)
        U = T @ (b[:, None] * vv)
        Qt = q * np.exp(G) * dtype(scale)
        Kt = k * np.exp(G[-1][None, :] - G)
        out.append(dict(Gamma=G, A=A, P=P, T=T, W=W, U=U, Qt=Qt, Kt=Kt, gC=np.exp(G[-1])))
    return out


def chunked_forward(qhat, khat, v, log_alpha, beta, scale, S0=None, C=64, blocked=False,
                    block=16, dtype=np.float64):
    """O [L, V] and S_final [K, V] of one unit by the chunked form."""
    K = np.asarray(khat).shape[1]
    V = np.asarray(v).shape[1]
    S = np.zeros((K, V), dtype=dtype) if S0 is None else np.asarray(S0, dtype=dtype).copy()
    outs = []
    for ch in chunk_intermediates(qhat, khat, v, log_alpha, beta, scale, C, blocked, block, dtype):
        Delta = ch["U"] - ch["W"] @ S
        outs.append(ch["Qt"] @ S + ch["P"] @ Delta)
        S = ch["gC"][:, None] * S + ch["Kt"].T @ Delta
    O = np.concatenate(outs, axis=0) if outs else np.zeros((0, V), dtype=dtype)
    return O, S
