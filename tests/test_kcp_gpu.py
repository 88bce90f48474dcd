"""GPU parity of the sequence-parallel prefill pieces (kda_segment_map, kda_state_affine and
kcp.kcp_forward) against the fp64 oracle.

The ranks of a KCP group are emulated one after another in this process: each emulated rank runs
kcp_forward on its segment with an exchange object that hands back the maps every segment produced
on this GPU (so no kernel waits on another, and no collective runs).  The concatenated outputs and
the final states must match the oracle run over the unsplit sequences within the forward pass's
tolerances.
"""
import numpy as np
import pytest
import torch

import kda_inputs
import kimi_delta_attention_24_b200 as kda
import margins
import oracle
from kimi_delta_attention_24_b200.kcp import DeviceOps, kcp_forward

pytestmark = pytest.mark.gpu

O_MAX_ABS = 3e-2
O_REL_L2 = 1e-2
S_REL_L2 = 1e-2


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def check(o, s, o_ref, s_ref, what):
    assert np.isfinite(o).all() and np.isfinite(s).all(), what
    err = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    rl, rs = rel_l2(o, o_ref), rel_l2(s, s_ref)
    margins.record(what, err, rl, rs)
    print(f"{what}: o max-abs {err:.3e}, o rel-L2 {rl:.3e}, state rel-L2 {rs:.3e}")
    assert err <= O_MAX_ABS and rl <= O_REL_L2, what
    assert rs <= S_REL_L2, what


def test_segment_map_against_oracle(cuda_device):
    """M = the state reached from the identity with v = 0, B = the state reached from zero, per
    (sequence, head); a 300-token batch (partial last chunk, two stages' worth of units) and an
    empty segment (M = I, B = 0)."""
    x = kda_inputs.make_random("t", None, 3, seed=91, varlen=False, batch=2, seqlen=300)
    x.g.fill_(-6.0)  # slow decay (log alpha ~ -1e-2 per token): M stays far from zero
    B, T, H, K = x.q.shape
    _, B_ref = oracle.kda_fwd(x.q, x.k, x.v, x.g, x.beta, 1.0, x.A_log, x.dt_bias, x.lower_bound)
    eye = np.broadcast_to(np.eye(K), (B, H, K, K)).copy()
    _, M_ref = oracle.kda_fwd(x.q, x.k, torch.zeros_like(x.v), x.g, x.beta, 1.0, x.A_log, x.dt_bias,
                              x.lower_bound, initial_state=eye)
    xd = x.to(cuda_device)
    M, Bm = DeviceOps().segment_map(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.A_log, xd.dt_bias, x.lower_bound, 0)
    M, Bm = M.cpu().double().numpy(), Bm.cpu().double().numpy()
    for name, got, want in (("M", M, M_ref), ("B", Bm, B_ref)):
        err = rel_l2(got, want)
        margins.note(f"segment map {name}: rel-L2 {err:.2e} (tol 1e-02)")
        assert np.isfinite(got).all() and err <= S_REL_L2, f"{name}: rel-L2 {err:.3e}"
    # an empty sequence maps every state to itself (varlen: documents of 0 and 150 tokens)
    y = kda_inputs.make_random("t", [0, 150], H, seed=94).to(cuda_device)
    M2 = torch.full((2, H, K, K), float("nan"), device=cuda_device)
    B2 = torch.full((2, H, K, K), float("nan"), device=cuda_device)
    ws = kda.new_workspace(150, H, 2, cuda_device)
    kda.segment_map(y.q, y.k, y.v, y.g, y.beta, ws, y.A_log, y.dt_bias, y.lower_bound, M2, B2, y.cu_seqlens)
    assert kda.read_device_status(ws) == 0
    assert torch.equal(M2[0].cpu(), torch.eye(K).expand(H, K, K))
    assert torch.count_nonzero(B2[0]) == 0
    assert torch.isfinite(M2[1]).all() and torch.isfinite(B2[1]).all()


@pytest.mark.parametrize("transposed", [False, True])
def test_state_affine_against_numpy(cuda_device, transposed):
    """S_out = M S_in + B on 5 units, both layouts, out of place and in place; zero state input."""
    gen = torch.Generator().manual_seed(92)
    M = torch.randn(5, 128, 128, generator=gen) * 0.1
    Bm = torch.randn(5, 128, 128, generator=gen)
    S = torch.randn(5, 128, 128, generator=gen)
    want = M.double() @ S.double() + Bm.double()
    S_in = S.transpose(-1, -2).contiguous() if transposed else S
    want_l = want.transpose(-1, -2) if transposed else want
    dev = cuda_device
    out = torch.empty_like(S_in, device=dev)
    kda.state_affine(M.to(dev), Bm.to(dev), S_in.to(dev), out, state_transposed=transposed)
    np.testing.assert_allclose(out.cpu().double().numpy(), want_l.numpy(), rtol=0, atol=2e-4)
    inplace = S_in.to(dev)
    kda.state_affine(M.to(dev), Bm.to(dev), inplace, inplace, state_transposed=transposed)
    np.testing.assert_allclose(inplace.cpu().double().numpy(), want_l.numpy(), rtol=0, atol=2e-4)
    zero = torch.empty_like(out)
    kda.state_affine(None, Bm.to(dev), None, zero, state_transposed=transposed)
    want0 = Bm.transpose(-1, -2) if transposed else Bm
    assert torch.equal(zero.cpu(), want0.contiguous())


class _EmulatedComm:
    """One emulated rank of a group whose members' maps are already on this GPU."""

    def __init__(self, rank, all_maps):
        self.rank, self.world, self.all_maps = rank, len(all_maps), all_maps

    def all_gather(self, t):
        torch.testing.assert_close(t, self.all_maps[self.rank], rtol=0, atol=0)
        return list(self.all_maps)


@pytest.mark.parametrize("cuts,transposed,flags,slow", [([0, 100, 400, 401, 1000], False, 0, True),
                                                        ([0, 100, 400, 401, 1000], False, 0, False),
                                                        ([0, 64, 128, 1000], True, 0, True),
                                                        ([0, 333, 1000], False, 7, True)])
def test_kcp_emulated_ranks_match_unsplit_oracle(cuda_device, cuts, transposed, flags, slow):
    """A batch of two 1000-token sequences cut into uneven segments, one per emulated rank.  With
    slow gates (raw gate -6: log alpha ~ -1e-2 per token) the initial state and every earlier
    segment still weigh on the last segment's output, so the fold of the maps is exercised."""
    H = 4
    x = kda_inputs.make_random("t", None, H, seed=93, varlen=False, batch=2, seqlen=cuts[-1], state_std=0.1)
    if slow:
        x.g.fill_(-6.0)
    q_in, k_in, g_in, beta_in = x.q, x.k, x.g, x.beta
    if flags:
        qh, kh, la, be = oracle.prologue(x.q, x.k, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound)
        g_in, beta_in = torch.from_numpy(la).float(), torch.from_numpy(be).float()
        q_in = (x.q.float() * 0.2).to(torch.bfloat16)
        k_in = (x.k.float() * 0.08).to(torch.bfloat16)
        B, T = x.q.shape[:2]
        tok = lambda a: np.ascontiguousarray(a.reshape(B * T, H, *a.shape[3:]))
        o_ref, s_ref = oracle.core(tok(q_in.double().numpy()), tok(k_in.double().numpy()), tok(x.v.double().numpy()),
                                   tok(g_in.double().numpy()), tok(beta_in.double().numpy()), x.scale,
                                   S0=x.initial_state.double().numpy(), cu_seqlens=np.arange(B + 1, dtype=np.int32) * T)
        o_ref = o_ref.reshape(x.v.shape)
        if transposed:
            s_ref = np.swapaxes(s_ref, -1, -2)
    else:
        o_ref, s_ref = oracle.fwd_inputs(x, state_transposed=transposed)
    dev = cuda_device
    ins = [t.to(dev) for t in (q_in, k_in, x.v, g_in, beta_in)]
    s0 = x.initial_state.transpose(-1, -2).contiguous() if transposed else x.initial_state
    s0 = s0.to(dev)
    segs = [[t[:, a:b].contiguous() for t in ins] for a, b in zip(cuts[:-1], cuts[1:])]
    A_log, dt_bias = x.A_log.to(dev), x.dt_bias.to(dev)
    ops = DeviceOps()
    all_maps = []
    for q, k, v, g, b in segs:  # what every rank contributes to the all-gather
        M, Bm = ops.segment_map(q, k, v, g, b, None if flags & 1 else A_log, None if flags & 1 else dt_bias,
                                x.lower_bound, flags)
        all_maps.append(torch.stack([M, Bm]).contiguous())
    outs, finals = [], []
    for r, (q, k, v, g, b) in enumerate(segs):
        o, f = kcp_forward(q, k, v, g, b, x.scale, A_log, dt_bias, x.lower_bound, initial_state=s0,
                           state_transposed=transposed, flags=flags, comm=_EmulatedComm(r, all_maps))
        outs.append(o)
        finals.append(f)
    o = torch.cat(outs, dim=1).float().cpu().double().numpy()
    for r, f in enumerate(finals):
        check(o, f.cpu().double().numpy(), o_ref, s_ref, f"kcp {len(segs)} ranks {cuts} transposed={transposed} "
                                                         f"flags={flags} slow={slow}, rank {r} final")
