"""Pins for the oracle's recurrence, written against a generic single-unit core.

A core is ``core(qhat[T,K], khat[T,K], v[T,V], log_alpha[T,K], beta[T], scale, S0[K,V])`` and
returns ``(o[T,V], S_T[K,V])``.  Each pin raises AssertionError when the core disagrees with a
fact fixed independently of it: brute-force explicit products, or a closed form of a special
case of the recurrence.  ``tests/test_oracle_pins.py`` runs every pin on the C oracle, and runs
them on deliberately broken numpy cores to show that each plausible mistake trips a pin.
"""
from __future__ import annotations

import numpy as np

from oracle.brute import explicit_products


def _unit(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def _close(a, b, rtol, what):
    a = np.asarray(a)
    b = np.asarray(b)
    err = np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)
    assert np.all(np.isfinite(a)) and err <= rtol, f"{what}: rel err {err:.3e} > {rtol:.1e}"


def pin_brute_force(core, seed=0):
    """Random inputs, T <= 8: the core equals the explicit-product closed form."""
    rng = np.random.default_rng(seed)
    for (T, K, V) in [(1, 8, 6), (5, 16, 12), (8, 12, 16), (4, 128, 128)]:
        qh, kh = _unit(rng, T, K), _unit(rng, T, K)
        v = rng.standard_normal((T, V))
        la = -rng.uniform(0.0, 2.0, (T, K))
        beta = rng.uniform(0.05, 0.95, T)
        S0 = rng.standard_normal((K, V)) * 0.3
        scale = 0.37
        o, S = core(qh, kh, v, la, beta, scale, S0)
        o_ref, S_ref = explicit_products(qh, kh, v, la, beta, scale, S0)
        _close(o, o_ref, 1e-11, f"o (T={T},K={K},V={V})")
        _close(S, S_ref, 1e-11, f"S (T={T},K={K},V={V})")


def pin_identity(core, seed=1):
    """beta = 0 and alpha = 1: the state never changes and o_t = scale * S0^T qhat_t."""
    rng = np.random.default_rng(seed)
    T, K, V = 40, 16, 8
    qh, kh = _unit(rng, T, K), _unit(rng, T, K)
    v = rng.standard_normal((T, V))
    S0 = rng.standard_normal((K, V))
    o, S = core(qh, kh, v, np.zeros((T, K)), np.zeros(T), 0.5, S0)
    assert np.array_equal(S, S0), "state changed with beta=0, alpha=1"
    _close(o, 0.5 * qh @ S0, 1e-14, "o with beta=0, alpha=1")


def pin_pure_decay(core, seed=2):
    """beta = 0: S_t = Diag(exp(Gamma_t)) S0 with Gamma_t the cumulative log-decay."""
    rng = np.random.default_rng(seed)
    T, K, V = 70, 16, 8
    qh, kh = _unit(rng, T, K), _unit(rng, T, K)
    v = rng.standard_normal((T, V))
    la = -rng.uniform(0.0, 0.2, (T, K))
    S0 = rng.standard_normal((K, V))
    o, S = core(qh, kh, v, la, np.zeros(T), 1.3, S0)
    G = np.cumsum(la, axis=0)
    _close(S, np.exp(G[-1])[:, None] * S0, 1e-12, "final state under pure decay")
    o_ref = np.stack([1.3 * (np.exp(G[t])[:, None] * S0).T @ qh[t] for t in range(T)])
    _close(o, o_ref, 1e-12, "o under pure decay")


def pin_delta_rule_interpolates(core, seed=3):
    """alpha = 1, beta = 1, unit keys: after token t the state maps khat_t to v_t exactly."""
    rng = np.random.default_rng(seed)
    T, K, V = 12, 16, 8
    kh = _unit(rng, T, K)
    v = rng.standard_normal((T, V))
    S0 = rng.standard_normal((K, V))
    for t in range(1, T + 1):
        o, S = core(kh[:t], kh[:t], v[:t], np.zeros((t, K)), np.ones(t), 1.0, S0)
        _close(S.T @ kh[t - 1], v[t - 1], 1e-12, f"S_t^T k_t at t={t}")
        _close(o[t - 1], v[t - 1], 1e-12, f"o_t with q=k at t={t}")


def pin_collinear(core, seed=4):
    """q = k = one fixed direction, channel-uniform decay a, zero S0: S_t = k y_t^T with the
    scalar-gain recursion y_t = a (1 - beta) y_{t-1} + beta v_t, and o_t = scale * y_t."""
    rng = np.random.default_rng(seed)
    T, K, V = 300, 32, 8
    u = _unit(rng, 1, K)[0]
    v = np.tile(rng.standard_normal((16, V)), (T // 16 + 1, 1))[:T]
    la_scalar = -0.01
    beta = 0.999
    o, S = core(np.tile(u, (T, 1)), np.tile(u, (T, 1)), v, np.full((T, K), la_scalar),
                np.full(T, beta), 0.25, None)
    y = np.zeros(V)
    a = np.exp(la_scalar)
    ys = []
    for t in range(T):
        y = a * (1.0 - beta) * y + beta * v[t]
        ys.append(y.copy())
    _close(o, 0.25 * np.array(ys), 1e-11, "o on collinear keys")
    _close(S, np.outer(u, y), 1e-11, "final state on collinear keys")


def pin_orthogonal_keys(core, seed=5):
    """alpha = 1 and one-hot keys: only the selected row of S moves, towards v."""
    rng = np.random.default_rng(seed)
    T, K, V = 30, 8, 5
    idx = rng.integers(0, K, T)
    kh = np.eye(K)[idx]
    v = rng.standard_normal((T, V))
    beta = rng.uniform(0.1, 0.9, T)
    S0 = rng.standard_normal((K, V))
    o, S = core(kh, kh, v, np.zeros((T, K)), beta, 1.0, S0)
    R = S0.copy()
    for t in range(T):
        j = idx[t]
        R[j] = (1 - beta[t]) * R[j] + beta[t] * v[t]
        _close(o[t], R[j], 1e-12, f"o_t at t={t}")
    _close(S, R, 1e-12, "state with one-hot keys")


def pin_linearity(core, seed=6):
    """For fixed q, k, alpha, beta the map (V, S0) -> (O, S_T) is linear."""
    rng = np.random.default_rng(seed)
    T, K, V = 33, 16, 8
    qh, kh = _unit(rng, T, K), _unit(rng, T, K)
    la = -rng.uniform(0, 0.5, (T, K))
    beta = rng.uniform(0.1, 0.9, T)
    v1, v2 = rng.standard_normal((2, T, V))
    s1, s2 = rng.standard_normal((2, K, V))
    a, b = 0.7, -1.9
    o1, S1 = core(qh, kh, v1, la, beta, 0.5, s1)
    o2, S2 = core(qh, kh, v2, la, beta, 0.5, s2)
    o3, S3 = core(qh, kh, a * v1 + b * v2, la, beta, 0.5, a * s1 + b * s2)
    _close(o3, a * o1 + b * o2, 1e-12, "linearity of O")
    _close(S3, a * S1 + b * S2, 1e-12, "linearity of S")


def pin_split_resume(core, seed=7):
    """Running [0, t1), then [t1, T) from the carried state, equals the unsplit run."""
    rng = np.random.default_rng(seed)
    T, K, V = 50, 16, 8
    qh, kh = _unit(rng, T, K), _unit(rng, T, K)
    v = rng.standard_normal((T, V))
    la = -rng.uniform(0, 0.5, (T, K))
    beta = rng.uniform(0.1, 0.9, T)
    S0 = rng.standard_normal((K, V))
    o, S = core(qh, kh, v, la, beta, 0.5, S0)
    for t1 in (1, 16, 17, 49):
        oa, Sa = core(qh[:t1], kh[:t1], v[:t1], la[:t1], beta[:t1], 0.5, S0)
        ob, Sb = core(qh[t1:], kh[t1:], v[t1:], la[t1:], beta[t1:], 0.5, Sa)
        _close(np.concatenate([oa, ob]), o, 1e-13, f"split at {t1}: o")
        _close(Sb, S, 1e-13, f"split at {t1}: S")


ALL_PINS = [pin_brute_force, pin_identity, pin_pure_decay, pin_delta_rule_interpolates,
            pin_collinear, pin_orthogonal_keys, pin_linearity, pin_split_resume]
