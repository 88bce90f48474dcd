"""Pins of the oracle's backward pass (oracle.kda_bwd), independent of the adjoint's own code:

- the fp64-input forward it differentiates (oracle.kda_fwd_f64) equals the pinned bf16-input
  forward (oracle.kda_fwd) on bf16-representable inputs;
- central finite differences of that forward, along random directions of every input (q, k, v, g,
  beta, A_log, dt_bias, the initial state), equal the adjoint's inner products with the same
  directions (the loss is sum(d_out * o) + sum(d_final * S_final));
- closed form: with beta = 0 and alpha = 1 the state never moves, so the gradient of the initial
  state is d_final + scale sum_t qhat_t d_out_t^T and v, g, A_log and dt_bias get no gradient.
"""
import numpy as np
import pytest
import torch

import kda_inputs
import oracle


def _problem(lens, H, seed, lb=-5.0, state_std=0.3):
    x = kda_inputs.make_random("bwd", lens, H, seed=seed, state_std=state_std, lower_bound=lb)
    rng = np.random.default_rng(seed)
    d_out = rng.standard_normal(x.v.shape)
    d_final = rng.standard_normal((len(lens), H, 128, 128)) * 0.5
    return x, d_out, d_final


def _loss(x, vals, d_out, d_final):
    o, s = oracle.kda_fwd_f64(vals["q"], vals["k"], vals["v"], vals["g"], vals["beta"], x.scale, vals["A_log"],
                              vals["dt_bias"], x.lower_bound, initial_state=vals["s0"], cu_seqlens=x.cu_seqlens)
    return float(np.sum(d_out * o) + np.sum(d_final * s))


def _vals(x):
    f = lambda t: t.double().numpy().copy()
    return dict(q=f(x.q), k=f(x.k), v=f(x.v), g=f(x.g), beta=f(x.beta), A_log=f(x.A_log), dt_bias=f(x.dt_bias),
                s0=f(x.initial_state))


def test_fwd_f64_equals_bf16_forward():
    x = kda_inputs.make_random("t", [5, 70, 0, 33], 3, seed=101, state_std=0.2)
    o1, s1 = oracle.fwd_inputs(x)
    v = _vals(x)
    o2, s2 = oracle.kda_fwd_f64(v["q"], v["k"], v["v"], v["g"], v["beta"], x.scale, v["A_log"], v["dt_bias"],
                                x.lower_bound, initial_state=v["s0"], cu_seqlens=x.cu_seqlens)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2, s1, rtol=0, atol=1e-12)


@pytest.mark.parametrize("lb", [-5.0, -1.0])
def test_adjoint_matches_finite_differences(lb):
    x, d_out, d_final = _problem([4, 6], 2, seed=102, lb=lb)
    vals = _vals(x)
    g = oracle.kda_bwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, d_out,
                       initial_state=x.initial_state, d_final=d_final, cu_seqlens=x.cu_seqlens)
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "A_log": "dA_log",
             "dt_bias": "ddt_bias", "s0": "d_initial"}
    rng = np.random.default_rng(7)
    for name, gname in names.items():
        u = rng.standard_normal(vals[name].shape)
        h = 1e-6 * max(1.0, float(np.abs(vals[name]).max()))
        plus = {n: (a + h * u if n == name else a) for n, a in vals.items()}
        minus = {n: (a - h * u if n == name else a) for n, a in vals.items()}
        fd = (_loss(x, plus, d_out, d_final) - _loss(x, minus, d_out, d_final)) / (2 * h)
        ad = float(np.sum(g[gname] * u))
        assert abs(fd - ad) <= 1e-6 * max(1.0, abs(ad)), f"{name}: finite differences {fd:.10e}, adjoint {ad:.10e}"


def test_adjoint_closed_form_frozen_state():
    x, d_out, d_final = _problem([7, 3], 2, seed=103, lb=0.0)
    x.beta.fill_(-float("inf"))  # beta = sigmoid(-inf) = 0; lower_bound 0 gives alpha = 1
    g = oracle.kda_bwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, d_out,
                       initial_state=x.initial_state, d_final=d_final, cu_seqlens=x.cu_seqlens)
    qh, _, _, _ = oracle.prologue(x.q, x.k, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound)
    cu = x.cu_seqlens.tolist()
    for n in range(2):
        want = d_final[n] + x.scale * np.einsum("thk,thv->hkv", qh[0, cu[n]:cu[n + 1]], d_out[0, cu[n]:cu[n + 1]])
        np.testing.assert_allclose(g["d_initial"][n], want, rtol=1e-12, atol=1e-12)
    for name in ("dv", "dg", "dA_log", "ddt_bias"):
        assert np.all(g[name] == 0), name


def test_gate_parameter_gradients_follow_from_dg():
    """The gate is log alpha = lb sigmoid(e^A_log (g + dt_bias)): its derivatives in A_log and in
    dt_bias are those in g times (g + dt_bias) and times 1, so dA_log[h] = sum_{t,c} dg (g + dt_bias)
    and ddt_bias[h, c] = sum_t dg (the chain rule, independent of the adjoint's code)."""
    x, d_out, d_final = _problem([9, 40, 17], 3, seed=104)
    x.A_log.copy_(torch.tensor([-0.7, 0.0, 0.9]))
    g = oracle.kda_bwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, d_out,
                       initial_state=x.initial_state, d_final=d_final, cu_seqlens=x.cu_seqlens)
    H = x.num_heads
    dg = g["dg"].reshape(-1, H, 128)
    gate = x.g.double().numpy().reshape(-1, H, 128) + x.dt_bias.double().numpy()[None]
    np.testing.assert_allclose(g["dA_log"], (dg * gate).sum(axis=(0, 2)), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(g["ddt_bias"], dg.sum(axis=0), rtol=1e-10, atol=1e-14)
