"""Host logic of the sequence-parallel prefill (kcp.kcp_forward) on CPU gloo process groups.

Two and three ranks each hold one segment of the same batch of sequences; the kernels are replaced
by fp64 stand-ins built on the oracle (segment maps from two oracle runs, the fold as M S + B, the
forward as the oracle), so what is checked is the host side: which maps are gathered, in what
order they are folded, and what each rank returns.  The result must equal the oracle run over the
unsplit sequences to fp64 rounding.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import kda_inputs
import oracle


class OracleOps:
    """fp64 CPU stand-ins of the three device operations kcp_forward calls."""

    def segment_map(self, q, k, v, g, beta, A_log, dt_bias, lower_bound, flags):
        assert flags == 0
        B, T, H, K = q.shape
        _, Bm = oracle.kda_fwd(q, k, v, g, beta, 1.0, A_log, dt_bias, lower_bound, initial_state=None)
        eye = np.broadcast_to(np.eye(K), (B, H, K, K)).copy()
        _, M = oracle.kda_fwd(q, k, torch.zeros_like(v), g, beta, 1.0, A_log, dt_bias, lower_bound,
                              initial_state=eye)
        return torch.from_numpy(M), torch.from_numpy(Bm)

    def fold(self, M, Bm, S, state_transposed):
        if S is None:
            out = Bm.clone()
        else:
            S = S.double()
            out = M @ (S.transpose(-1, -2) if state_transposed else S) + Bm
        return out.transpose(-1, -2).contiguous() if state_transposed else out

    def forward(self, q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, S_in, flags, state_transposed):
        o, s = oracle.kda_fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound,
                              initial_state=None if S_in is None else S_in.double(),
                              state_transposed=state_transposed)
        return torch.from_numpy(o), torch.from_numpy(s)


def _problem(T):
    """Two sequences of T tokens with slow gates (raw gate -6: log alpha ~ -1e-2 per token), so that
    the initial state and every earlier segment still weigh on the last segment."""
    x = kda_inputs.make_random("kcp", None, 2, seed=81, varlen=False, batch=2, seqlen=T, state_std=0.1)
    x.g.fill_(-6.0)
    return x


def _worker(rank, world, port, cuts, transposed, result_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    from kimi_delta_attention_24_b200.kcp import kcp_forward

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = _problem(cuts[-1])
        a, b = cuts[rank], cuts[rank + 1]
        sl = lambda t: t[:, a:b].contiguous()
        s0 = x.initial_state.double()
        if transposed:
            s0 = s0.transpose(-1, -2).contiguous()
        o, final = kcp_forward(sl(x.q), sl(x.k), sl(x.v), sl(x.g), sl(x.beta), x.scale, x.A_log, x.dt_bias,
                               x.lower_bound, initial_state=s0, state_transposed=transposed, ops=OracleOps())
        result_q.put((rank, o.numpy(), final.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,cuts,transposed", [(2, [0, 130, 300], False), (3, [0, 90, 91, 300], False),
                                                   (3, [0, 64, 250, 300], True)])
def test_kcp_host_logic_matches_unsplit_oracle(world, cuts, transposed):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, transposed, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            r, o, f = q.get(timeout=240)
            results[r] = (o, f)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    x = _problem(cuts[-1])
    o_ref, s_ref = oracle.fwd_inputs(x, state_transposed=transposed)
    o = np.concatenate([results[r][0] for r in range(world)], axis=1)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-10)
    for r in range(world):  # every rank returns the whole sequences' final states
        np.testing.assert_allclose(results[r][1], s_ref, rtol=0, atol=1e-10)
