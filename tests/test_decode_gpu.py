"""GPU parity of the batched recurrent decode step (kda_decode) against the fp64 oracle.

Each request advances its own state in a pool by one token (or a few), the state carried from step
to step in the pool; the oracle runs the same tokens one at a time from the same initial states.
Tolerances are those of the forward pass: output max-abs <= 3e-2 and relative L2 <= 1e-2, state
relative L2 <= 1e-2, every element finite.
"""
import numpy as np
import pytest
import torch

import kda_inputs
import kimi_delta_attention_24_b200 as kda
import margins
import oracle

pytestmark = pytest.mark.gpu

O_MAX_ABS = 3e-2
O_REL_L2 = 1e-2
S_REL_L2 = 1e-2


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def check(o, s, o_ref, s_ref, what):
    assert np.isfinite(o).all(), what
    err = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    rl = rel_l2(o, o_ref)
    rs = None if s_ref is None else rel_l2(s, s_ref)
    margins.record(what, err, rl, rs)
    print(f"{what}: o max-abs {err:.3e}, o rel-L2 {rl:.3e}, state rel-L2 {rs}")
    assert err <= O_MAX_ABS and rl <= O_REL_L2, what
    if s_ref is not None:
        assert np.isfinite(s).all(), what
        assert rs <= S_REL_L2, what


def make_requests(B, T, H, seed, slots, state_std=0.1):
    """B requests of T tokens each (batch mode), a pool of `slots` states, and a slot per request."""
    x = kda_inputs.make_random("decode", None, H, seed=seed, varlen=False, batch=B, seqlen=T)
    gen = torch.Generator().manual_seed(seed + 1000)
    pool = torch.randn(slots, H, 128, 128, generator=gen) * state_std
    idx = torch.randperm(slots, generator=gen)[:B].to(torch.int32)
    return x, pool, idx


def oracle_step(x, pool, idx, transposed=False):
    """Reference: each request's tokens from its slot's state, in fp64; returns (o, new pool)."""
    s0 = pool[idx.long()]
    o, s = oracle.kda_fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound,
                          initial_state=s0.transpose(-1, -2).contiguous() if transposed else s0,
                          state_transposed=transposed)
    new = pool.double().numpy().copy()
    if transposed:
        new = np.swapaxes(new, -1, -2).copy()
    new[idx.numpy()] = s
    return o, new


@pytest.mark.parametrize("transposed", [False, True])
def test_decode_256_requests_96_heads_four_steps(cuda_device, transposed):
    """256 requests x 96 heads, one token per step, four steps in a row with the states carried in
    a 300-slot pool (updated in place); the oracle runs the four tokens one at a time."""
    B, H, steps, slots = 256, 96, 4, 300
    x, pool, idx = make_requests(B, steps, H, seed=61, slots=slots)
    o_ref, pool_ref = oracle_step(x, pool, idx, transposed)
    dev = cuda_device
    xd = x.to(dev)
    pool_d = (pool.transpose(-1, -2).contiguous() if transposed else pool.clone()).to(dev)
    idx_d = idx.to(dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    outs = []
    for t in range(steps):
        sl = lambda a: a[:, t:t + 1].contiguous()
        out = torch.full_like(sl(xd.v), float("nan"))
        kda.decode(sl(xd.q), sl(xd.k), sl(xd.v), sl(xd.g), sl(xd.beta), x.scale, out, xd.A_log, xd.dt_bias,
                   x.lower_bound, pool_d, pool_d, idx_d, state_transposed=transposed, workspace=ws)
        outs.append(out)
    assert kda.read_device_status(ws) == 0
    o = torch.cat(outs, dim=1).float().cpu().double().numpy()
    s = pool_d.cpu().double().numpy()
    check(o, s, o_ref, pool_ref, f"decode 256x96, 4 steps, transposed={transposed}")
    # slots no request points at are untouched
    free = np.setdiff1d(np.arange(slots), idx.numpy())
    ref_free = pool.numpy()[free]
    got_free = s[free].astype(np.float32)
    if transposed:
        got_free = np.swapaxes(got_free, -1, -2)
    np.testing.assert_array_equal(got_free, ref_free)


def test_decode_several_tokens_per_request(cuda_device):
    """Three tokens per request in one call (speculative tokens) equal three one-token calls and
    the oracle; separate in / out pools, the in pool left unchanged."""
    B, T, H = 33, 3, 8
    x, pool, idx = make_requests(B, T, H, seed=62, slots=40)
    o_ref, pool_ref = oracle_step(x, pool, idx)
    xd = x.to(cuda_device)
    p_in = pool.to(cuda_device)
    p_out = torch.full_like(p_in, float("nan"))
    out = torch.full_like(xd.v, float("nan"))
    kda.decode(xd.q, xd.k, xd.v, xd.g, xd.beta, x.scale, out, xd.A_log, xd.dt_bias, x.lower_bound,
               p_in, p_out, idx.to(cuda_device))
    torch.cuda.synchronize()
    assert torch.equal(p_in.cpu(), pool)
    o = out.float().cpu().double().numpy()
    s = p_out.cpu().double().numpy()[idx.numpy()]
    check(o, s, o_ref, pool_ref[idx.numpy()], "decode 3 tokens per request")


@pytest.mark.parametrize("flags", [1, 2, 4, 7])
def test_decode_input_flags(cuda_device, flags):
    """Precomputed fp32 log alpha (1), no q/k L2 norm (2), precomputed fp32 beta (4), all three (7),
    against the oracle's recurrence fed the same transformed inputs."""
    B, T, H = 16, 2, 4
    x, pool, idx = make_requests(B, T, H, seed=63, slots=20)
    qh, kh, la, be = oracle.prologue(x.q, x.k, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound)
    g_in, beta_in = x.g, x.beta
    if flags & kda.FLAG_GATE_PRECOMPUTED:
        g_in = torch.from_numpy(la).float()
        la = g_in.double().numpy()                     # the fp32 values the kernel reads
    if flags & kda.FLAG_BETA_PRECOMPUTED:
        beta_in = torch.from_numpy(be).float()
        be = beta_in.double().numpy()
    if flags & kda.FLAG_NO_QK_L2NORM:
        qh = x.q.double().numpy() * 0.2                # raw (unnormalised) q and k, scaled down
        kh = x.k.double().numpy() * 0.08               # so that the delta rule stays contractive
        q_in = torch.from_numpy(qh).to(torch.bfloat16)
        k_in = torch.from_numpy(kh).to(torch.bfloat16)
        qh, kh = q_in.double().numpy(), k_in.double().numpy()
    else:
        q_in, k_in = x.q, x.k
    s0 = pool[idx.long()].double().numpy()
    tok = lambda a: np.ascontiguousarray(a.reshape(B * T, H, *a.shape[3:]))
    cu = np.arange(B + 1, dtype=np.int32) * T
    o_ref, s_ref = oracle.core(tok(qh), tok(kh), tok(x.v.double().numpy()), tok(la), tok(be), x.scale,
                               S0=s0, cu_seqlens=cu)
    dev = cuda_device
    p = pool.to(dev)
    out = torch.full_like(x.v, float("nan"), device=dev)
    kda.decode(q_in.to(dev), k_in.to(dev), x.v.to(dev), g_in.to(dev), beta_in.to(dev), x.scale, out,
               None if flags & 1 else x.A_log.to(dev), None if flags & 1 else x.dt_bias.to(dev),
               x.lower_bound, p, p, idx.to(dev), flags=flags)
    o = out.float().cpu().double().numpy().reshape(B * T, H, 128)
    s = p.cpu().double().numpy()[idx.numpy()]
    check(o, s, o_ref, s_ref, f"decode flags={flags}")


def test_decode_padding_zero_states_and_bad_index(cuda_device):
    """A negative index skips its request (output row untouched); a NULL in pool means zero states;
    an index past the pool skips its request and raises KDA_ERR_INVALID_ARGUMENT in the status
    word, while the other requests are computed."""
    B, H = 6, 3
    x, pool, _ = make_requests(B, 1, H, seed=64, slots=8)
    idx = torch.tensor([3, -1, 0, 9, 5, -7], dtype=torch.int32)
    zero = torch.zeros(B, H, 128, 128)
    o_ref, s_ref = oracle.kda_fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound,
                                  initial_state=zero)
    dev = cuda_device
    xd = x.to(dev)
    p_out = torch.full((8, H, 128, 128), float("nan"), device=dev)
    out = torch.full_like(xd.v, float("nan"))
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    kda.decode(xd.q, xd.k, xd.v, xd.g, xd.beta, x.scale, out, xd.A_log, xd.dt_bias, x.lower_bound,
               None, p_out, idx.to(dev), workspace=ws)
    assert kda.read_device_status(ws) == 1  # index 9 >= 8 slots
    o = out.float().cpu().double().numpy()
    s = p_out.cpu().double().numpy()
    live = [0, 2, 4]
    check(o[live], s[idx.numpy()[live]], o_ref[live], s_ref[live], "decode padding / zero states")
    assert np.isnan(o[[1, 3, 5]]).all()
    untouched = [1, 2, 4, 6, 7]
    assert np.isnan(s[untouched]).all()


def test_decode_matches_chunked_prefill_continuation(cuda_device):
    """Prefill 300 tokens with kda_fwd, then decode 5 more tokens one at a time from its final
    state: the outputs and final state equal the oracle over all 305 tokens."""
    H = 4
    x = kda_inputs.make_random("t", [305], H, seed=65, state_std=0.1)
    o_ref, s_ref = oracle.fwd_inputs(x)
    dev = cuda_device
    xd = x.to(dev)
    pre = lambda a: a[:, :300].contiguous()
    out = torch.empty_like(pre(xd.v))
    state = torch.empty(1, H, 128, 128, device=dev)
    ws = kda.new_workspace(300, H, 1, dev)
    kda.fwd(pre(xd.q), pre(xd.k), pre(xd.v), pre(xd.g), pre(xd.beta), x.scale, out, ws, xd.A_log, xd.dt_bias,
            x.lower_bound, xd.initial_state, state, torch.tensor([0, 300], dtype=torch.int32, device=dev))
    outs = [out]
    for t in range(300, 305):
        sl = lambda a: a[:, t:t + 1].contiguous()
        o_t = torch.empty_like(sl(xd.v))
        kda.decode(sl(xd.q), sl(xd.k), sl(xd.v), sl(xd.g), sl(xd.beta), x.scale, o_t, xd.A_log, xd.dt_bias,
                   x.lower_bound, state, state)
        outs.append(o_t)
    o = torch.cat(outs, dim=1).float().cpu().double().numpy()
    check(o, state.cpu().double().numpy(), o_ref, s_ref, "prefill 300 + decode 5")


def test_decode_zero_tokens_copies_states(cuda_device):
    """seqlen = 0: no token, the requests' states go from the in pool to the out pool unchanged."""
    B, H = 5, 2
    gen = torch.Generator().manual_seed(66)
    pool = torch.randn(7, H, 128, 128, generator=gen).to(cuda_device)
    idx = torch.tensor([6, 0, -1, 3, 2], dtype=torch.int32, device=cuda_device)
    dev = cuda_device
    # empty token tensors (their data pointers are null: nothing of them is read)
    q, k, v, g, out = (torch.zeros(B, 0, H, 128, dtype=torch.bfloat16, device=dev) for _ in range(5))
    beta = torch.zeros(B, 0, H, dtype=torch.bfloat16, device=dev)
    p_out = torch.full_like(pool, float("nan"))
    kda.decode(q, k, v, g, beta, 0.088, out, torch.zeros(H, device=dev), torch.zeros(H, 128, device=dev), -5.0,
               pool, p_out, idx)
    torch.cuda.synchronize()
    used = [6, 0, 3, 2]
    assert torch.equal(p_out[used], pool[used])
    assert torch.isnan(p_out[[1, 4, 5]]).all()
