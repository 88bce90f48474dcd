"""Pins of the CPU oracle against facts fixed independently of it (CPU only).

The pages print no worked numeric example for KDA, so the oracle is pinned by brute force,
closed forms of special cases, invariants of the recurrence, and library routines for the
elementwise transforms.  A final group plants plausible mistakes in a numpy copy of the core
and checks that some pin catches each one.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from oracle.chunked import chunked_forward, chunk_intermediates
import pins
import kda_inputs


def c_core(qh, kh, v, la, beta, scale, S0):
    """The C oracle's recurrence for one unit (adds and drops the head axis)."""
    o, S = oracle.core(qh[:, None, :], kh[:, None, :], v[:, None, :], la[:, None, :],
                       np.asarray(beta)[:, None], scale,
                       None if S0 is None else np.asarray(S0)[None, None])
    return o[:, 0, :], S[0, 0]


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_c_oracle_core_pins(pin):
    pin(c_core)


# --------------------------------------------------------------------------- planted mistakes

def numpy_core(mistake=None):
    def core(qh, kh, v, la, beta, scale, S0):
        T, K = kh.shape
        V = v.shape[1]
        S = np.zeros((K, V)) if S0 is None else np.array(S0, dtype=np.float64)
        o = np.zeros((T, V))
        for t in range(T):
            a = np.exp(la[t])
            if mistake != "no_decay" and mistake != "decay_after":
                S = a[:, None] * S
            pred = S.T @ kh[t]
            if mistake == "pred_before_decay":
                pred = (S / a[:, None]).T @ kh[t]
            d = (v[t] - pred) if mistake == "no_beta" else beta[t] * (v[t] - pred)
            S_prev = S
            S = S - np.outer(kh[t], d) if mistake == "sign" else S + np.outer(kh[t], d)
            if mistake == "decay_after":
                S = a[:, None] * S
            if mistake == "wrong_key":
                S = S_prev + np.outer(kh[max(t - 1, 0)], d)
            Sr = S_prev if mistake == "output_pre_update" else S
            o[t] = scale * (Sr @ qh[t] if mistake == "transpose" else Sr.T @ qh[t])
            if mistake == "scale_in_state":
                S = S * (1.0 + 0.0 * scale) if scale == 1.0 else S * scale
        return o, S
    return core


def test_numpy_core_passes_pins():
    for pin in pins.ALL_PINS:
        pin(numpy_core(None))


@pytest.mark.parametrize("mistake", ["no_decay", "decay_after", "pred_before_decay", "no_beta",
                                     "sign", "wrong_key", "output_pre_update", "transpose",
                                     "scale_in_state"])
def test_planted_mistake_is_caught(mistake):
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(numpy_core(mistake))
        except (AssertionError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mistake {mistake!r}"


# --------------------------------------------------------------------------- prologue pins

def _bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def test_l2norm_matches_library_norm_and_zero_vector():
    g = torch.Generator().manual_seed(0)
    q = (torch.randn(3, 5, 2, 128, generator=g)).to(torch.bfloat16)
    q[0, 0, 0] = 0.0
    z = torch.zeros_like(q)
    qh, kh, _, _ = oracle.prologue(q, q, z, torch.zeros(3, 5, 2, dtype=torch.bfloat16),
                                   torch.zeros(2), torch.zeros(2, 128), -5.0)
    qf = q.double().numpy()
    n = np.linalg.norm(qf, axis=-1, keepdims=True)
    mask = n[..., 0] > 0
    # eps = 1e-6 against |q|^2 ~ 128 moves the norm by ~4e-9
    np.testing.assert_allclose(qh[mask], (qf / np.where(n > 0, n, 1))[mask], rtol=1e-8, atol=0)
    assert np.all(qh[0, 0, 0] == 0.0)
    np.testing.assert_array_equal(qh, kh)


def test_l2norm_epsilon_reading():
    # |q|^2 = 2^-20 is comparable to eps = 1e-6: q / sqrt(2^-20 + 1e-6)
    q = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16)
    q[..., 0] = 2.0 ** -10
    qh, _, _, _ = oracle.prologue(q, q, torch.zeros_like(q), torch.zeros(1, 1, 1, dtype=torch.bfloat16),
                                  torch.zeros(1), torch.zeros(1, 128), -5.0)
    assert qh[0, 0, 0, 0] == pytest.approx(2.0 ** -10 / math.sqrt(2.0 ** -20 + 1e-6), rel=1e-14)


def test_beta_sigmoid():
    raw = torch.tensor([[[0.0, 1.0, -3.5, 8.0, float("inf"), float("-inf"), -40.0]]]).to(torch.bfloat16)
    raw = raw.permute(0, 2, 1)  # [1, 7, 1]
    z = torch.zeros(1, 7, 1, 128, dtype=torch.bfloat16)
    _, _, _, beta = oracle.prologue(z, z, z, raw, torch.zeros(1), torch.zeros(1, 128), -5.0)
    np.testing.assert_allclose(beta[0, :, 0], expit(raw.double().numpy()[0, :, 0]), rtol=1e-15)
    assert beta[0, 0, 0] == 0.5 and beta[0, 4, 0] == 1.0 and beta[0, 5, 0] == 0.0


def _gate(g_val, a_log, dt, lb=-5.0):
    g = torch.full((1, 1, 1, 128), g_val, dtype=torch.float32).to(torch.bfloat16)
    z = torch.zeros_like(g)
    _, _, la, _ = oracle.prologue(z, z, g, torch.zeros(1, 1, 1, dtype=torch.bfloat16),
                                  torch.tensor([a_log], dtype=torch.float32),
                                  torch.full((1, 128), dt, dtype=torch.float32), lb)
    return la[0, 0, 0]


def test_safe_gate_special_values():
    lb = -5.0
    # sigmoid(0) = 1/2 whenever the argument vanishes: g + dt_bias = 0, or exp(A_log) = 0
    assert np.all(_gate(0.0, 0.0, 0.0) == lb / 2)
    assert np.all(_gate(3.0, float("-inf"), 0.25) == lb / 2)
    assert np.all(_gate(0.5, 1.0, -0.5) == lb / 2)
    # saturation: the decay tends to lower_bound (strong gate) or to 1 (open gate)
    np.testing.assert_allclose(_gate(100.0, 0.0, 0.0), lb, rtol=1e-15)
    assert np.all(np.abs(_gate(-100.0, 0.0, 0.0)) < 1e-40)
    # a value: exp(A_log)*(g+dt) = ln 3 gives sigmoid = 3/4; A_log = ln 2 pins the exp(A_log) factor
    np.testing.assert_allclose(_gate(0.0, 0.0, float(np.float32(math.log(3.0)))), 0.75 * lb, rtol=1e-7)
    np.testing.assert_allclose(_gate(0.0, float(np.float32(math.log(2.0))),
                                     float(np.float32(math.log(3.0) / 2))), 0.75 * lb, rtol=1e-6)
    # lower_bound = 0 switches the decay off exactly
    assert np.all(_gate(1.7, 0.3, 0.2, lb=0.0) == 0.0)


# --------------------------------------------------------------------------- full-forward invariants

def test_fwd_equals_prologue_then_core():
    x = kda_inputs.make_random("t", [37, 70], 3, seed=11, state_std=0.2)
    o, S = oracle.fwd_inputs(x)
    qh, kh, la, be = oracle.prologue(x.q[0], x.k[0], x.g[0], x.beta[0], x.A_log, x.dt_bias, x.lower_bound)
    o2, S2 = oracle.core(qh, kh, x.v[0].double().numpy(), la, be, x.scale, x.initial_state.double().numpy(),
                         x.cu_seqlens.numpy())
    np.testing.assert_array_equal(o[0], o2)
    np.testing.assert_array_equal(S, S2)


def test_varlen_equals_independent_documents():
    x = kda_inputs.make_random("t", [5, 64, 1, 130, 0, 17], 2, seed=12, state_std=0.1)
    o, S = oracle.fwd_inputs(x)
    cu = x.cu_seqlens.tolist()
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        on, Sn = oracle.kda_fwd(x.q[:, a:b], x.k[:, a:b], x.v[:, a:b], x.g[:, a:b], x.beta[:, a:b],
                                x.scale, x.A_log, x.dt_bias, x.lower_bound,
                                initial_state=x.initial_state[n:n + 1],
                                cu_seqlens=torch.tensor([0, b - a], dtype=torch.int32))
        np.testing.assert_array_equal(o[:, a:b], on)
        np.testing.assert_array_equal(S[n:n + 1], Sn)
    # a zero-length document hands its initial state through unchanged
    np.testing.assert_array_equal(S[4], x.initial_state[4].double().numpy())


def test_batch_mode_equals_varlen():
    x = kda_inputs.make_random("t", None, 2, seed=13, varlen=False, batch=3, seqlen=40, state_std=0.1)
    o, S = oracle.fwd_inputs(x)
    flat = lambda t: t.reshape(1, -1, *t.shape[2:])
    o2, S2 = oracle.kda_fwd(flat(x.q), flat(x.k), flat(x.v), flat(x.g), flat(x.beta), x.scale, x.A_log,
                            x.dt_bias, x.lower_bound, initial_state=x.initial_state,
                            cu_seqlens=torch.tensor([0, 40, 80, 120], dtype=torch.int32))
    np.testing.assert_array_equal(o.reshape(o2.shape), o2)
    np.testing.assert_array_equal(S, S2)


def test_split_resume_raw_inputs():
    x = kda_inputs.make_random("t", [150], 2, seed=14, state_std=0.1)
    o, S = oracle.fwd_inputs(x)
    for t1 in (64, 77):
        sl = lambda t, a, b: t[:, a:b]
        oa, Sa = oracle.kda_fwd(*(sl(t, 0, t1) for t in (x.q, x.k, x.v, x.g, x.beta)), x.scale, x.A_log,
                                x.dt_bias, x.lower_bound, initial_state=x.initial_state,
                                cu_seqlens=torch.tensor([0, t1], dtype=torch.int32))
        ob, Sb = oracle.kda_fwd(*(sl(t, t1, 150) for t in (x.q, x.k, x.v, x.g, x.beta)), x.scale, x.A_log,
                                x.dt_bias, x.lower_bound, initial_state=torch.from_numpy(Sa),
                                cu_seqlens=torch.tensor([0, 150 - t1], dtype=torch.int32))
        np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(Sb, S, rtol=0, atol=1e-12)


def test_state_layout_flag_transposes():
    x = kda_inputs.make_random("t", [20, 9], 2, seed=15, state_std=0.3)
    o, S = oracle.fwd_inputs(x)
    oT, ST = oracle.fwd_inputs(x, state_transposed=True)
    np.testing.assert_array_equal(o, oT)
    np.testing.assert_array_equal(S.transpose(0, 1, 3, 2), ST)


def test_null_states():
    x = kda_inputs.make_random("t", [33], 1, seed=16)
    o0, _ = oracle.kda_fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound,
                           initial_state=torch.zeros(1, 1, 128, 128), cu_seqlens=x.cu_seqlens)
    o1, S1 = oracle.kda_fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound,
                            initial_state=None, cu_seqlens=x.cu_seqlens, output_final_state=False)
    np.testing.assert_array_equal(o0, o1)
    assert S1 is None


def test_collinear_closed_form_raw_inputs():
    """The near-collinear stress case (vLLM PR #54859 report) has a closed form: with q = k = u
    and a channel-uniform gate, S_t = khat z_t^T with z_t = a (1 - beta c2) z_{t-1} + beta v_t,
    o_t = scale c2 z_t, where c2 = |u|^2 / (|u|^2 + eps) is the squared norm of khat."""
    x = kda_inputs.make_collinear(T=512, seed=0)
    o, S = oracle.fwd_inputs(x)
    u = x.k[0, 0, 0].double().numpy()
    ss = float(np.sum(u * u))
    c2 = ss / (ss + 1e-6)
    khat = u / math.sqrt(ss + 1e-6)
    a = math.exp(-5.0 * expit(-12.0))
    beta = expit(8.0)
    z = np.zeros(128)
    vs = x.v[0, :, 0].double().numpy()
    for t in range(512):
        z = a * (1 - beta * c2) * z + beta * vs[t]
        np.testing.assert_allclose(o[0, t, 0], x.scale * c2 * z, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(S[0, 0], np.outer(khat, z), rtol=1e-10, atol=1e-13)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))


# --------------------------------------------------------------------------- chunked algebra

def _unit_inputs(x, n=0, h=0):
    cu = x.cu_seqlens.tolist()
    a, b = cu[n], cu[n + 1]
    qh, kh, la, be = oracle.prologue(x.q[0, a:b], x.k[0, a:b], x.g[0, a:b], x.beta[0, a:b], x.A_log,
                                     x.dt_bias, x.lower_bound)
    return (qh[:, h], kh[:, h], x.v[0, a:b, h].double().numpy(), la[:, h], be[:, h],
            x.initial_state[n, h].double().numpy())


@pytest.mark.parametrize("lb", [0.0, -1.0, -5.0])
@pytest.mark.parametrize("C,blocked", [(1, False), (16, False), (64, False), (64, True), (32, True)])
def test_chunked_form_equals_recurrence(lb, C, blocked):
    x = kda_inputs.make_random("t", [200], 2, seed=17, state_std=0.1, lower_bound=lb)
    qh, kh, v, la, be, S0 = _unit_inputs(x, 0, 1)
    o_ref, S_ref = c_core(qh, kh, v, la, be, x.scale, S0)
    o, S = chunked_forward(qh, kh, v, la, be, x.scale, S0, C=C, blocked=blocked)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-10 * np.max(np.abs(o_ref)))
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-10 * np.max(np.abs(S_ref)))


def test_blocked_referencing_stays_finite_in_float32():
    """Saturated gates (log alpha = -5 on every channel) push e^{-Gamma} past float32 over a
    64-token chunk; sub-block referencing keeps every factor finite and the result accurate."""
    x = kda_inputs.make_random("t", [256], 1, seed=18, state_std=0.1)
    x.g.fill_(60.0)
    qh, kh, v, la, be, S0 = _unit_inputs(x)
    assert np.all(la <= -4.999)
    o_ref, S_ref = c_core(qh, kh, v, la, be, x.scale, S0)
    with np.errstate(over="ignore", invalid="ignore"):
        try:  # the unreferenced form overflows: a non-finite A (rejected by the solve) or O
            o_plain, _ = chunked_forward(qh, kh, v, la, be, x.scale, S0, C=64, dtype=np.float32)
            plain_finite = bool(np.all(np.isfinite(o_plain)))
        except ValueError:
            plain_finite = False
    assert not plain_finite
    with np.errstate(over="raise", invalid="raise"):
        o, S = chunked_forward(qh, kh, v, la, be, x.scale, S0, C=64, blocked=True, block=16,
                               dtype=np.float32)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-5 * np.max(np.abs(o_ref)))
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-5 * np.max(np.abs(S_ref)))


def test_collinear_inverse_entries_are_bounded():
    """With q = k collinear and alpha ~ 1, (I + A)^{-1} has entries -beta (1 - beta)^(r-s-1):
    bounded, so forward substitution stays finite (the 'unstable inverse' of the FlashKDA bump)."""
    x = kda_inputs.make_collinear(T=64)
    qh, kh, la, be = oracle.prologue(x.q[0], x.k[0], x.g[0], x.beta[0], x.A_log, x.dt_bias, x.lower_bound)
    ch = chunk_intermediates(qh[:, 0], kh[:, 0], x.v[0, :, 0].double().numpy(), la[:, 0], be[:, 0],
                             x.scale, 64, blocked=True)[0]
    T = ch["T"]
    assert np.all(np.isfinite(T)) and np.max(np.abs(T)) <= 1.0 + 1e-12
    b = be[0, 0]
    assert T[1, 0] == pytest.approx(-ch["A"][1, 0], rel=1e-12)
    assert abs(ch["A"][1, 0] - b) < 1e-4
