"""GPU parity of kda_fwd_ex at head sizes below 128 (zero padding to the 128-wide kernels) against
the fp64 oracle, which takes any head size."""
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


def sliced(x, K, V):
    """The same problem cut to head sizes (K, V): the first K key channels, the first V values."""
    c = lambda t, n: t[..., :n].contiguous()
    s0 = None if x.initial_state is None else x.initial_state[:, :, :K, :V].contiguous()
    return kda_inputs.KDAInputs(x.name, c(x.q, K), c(x.k, K), c(x.v, V), c(x.g, K), x.beta, x.A_log,
                                c(x.dt_bias, K), x.lower_bound, x.scale, s0, x.cu_seqlens, x.output_final_state)


@pytest.mark.parametrize("K,V,transposed", [(64, 64, False), (64, 128, True), (128, 32, False), (8, 8, False),
                                            (96, 72, True)])
def test_padded_head_sizes_against_oracle(cuda_device, K, V, transposed):
    x = sliced(kda_inputs.make_random("t", [130, 0, 64, 257], 3, seed=121, state_std=0.2), K, V)
    s0 = x.initial_state.transpose(-1, -2).contiguous() if transposed else x.initial_state
    o_ref, s_ref = oracle.kda_fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound,
                                  initial_state=s0, cu_seqlens=x.cu_seqlens, state_transposed=transposed)
    xd = x.to(cuda_device)
    N, H = x.num_seqs, x.num_heads
    out = torch.full_like(xd.v, float("nan"))
    fin = torch.full((N, H, V, K) if transposed else (N, H, K, V), float("nan"), device=cuda_device)
    ws = kda.new_workspace(x.total_tokens, H, N, cuda_device, K, V)
    kda.fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, x.scale, out, ws, xd.A_log, xd.dt_bias, x.lower_bound,
            s0.to(cuda_device), fin, xd.cu_seqlens, state_transposed=transposed)
    assert kda.read_device_status(ws) == 0
    o = out.float().cpu().double().numpy()
    s = fin.cpu().double().numpy()
    err, rl, rs = float(np.max(np.abs(o - o_ref))), rel_l2(o, o_ref), rel_l2(s, s_ref)
    margins.record(f"K={K} V={V} transposed={transposed}", err, rl, rs)
    assert np.isfinite(o).all() and np.isfinite(s).all()
    assert err <= O_MAX_ABS and rl <= O_REL_L2 and rs <= S_REL_L2, (err, rl, rs)


def test_padded_head_size_with_precomputed_gate_and_chunk_kda(cuda_device):
    """K = V = 64 through chunk_kda with use_gate_in_kernel=False (fp32 log alpha [T, H, 64])."""
    x = sliced(kda_inputs.make_random("t", [200, 77], 2, seed=122, state_std=0.1), 64, 64)
    _, _, la, _ = oracle.prologue(x.q, x.k, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound)
    qh, kh, _, be = oracle.prologue(x.q, x.k, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound)
    T, H = x.total_tokens, x.num_heads
    o_ref, s_ref = oracle.core(qh.reshape(T, H, 64), kh.reshape(T, H, 64), x.v.double().numpy().reshape(T, H, 64),
                               la.reshape(T, H, 64), be.reshape(T, H), x.scale,
                               S0=x.initial_state.double().numpy(), cu_seqlens=x.cu_seqlens.numpy())
    dev = cuda_device
    g_log = torch.from_numpy(la).float().to(dev)
    out, fin = kda.chunk_kda(x.q.to(dev), x.k.to(dev), x.v.to(dev), g_log, x.beta.to(dev), scale=x.scale,
                             initial_state=x.initial_state.to(dev), output_final_state=True,
                             lower_bound=x.lower_bound, cu_seqlens=x.cu_seqlens.to(dev), use_gate_in_kernel=False)
    o = out.float().cpu().double().numpy().reshape(T, H, 64)
    s = fin.cpu().double().numpy()
    err, rl, rs = float(np.max(np.abs(o - o_ref))), rel_l2(o, o_ref), rel_l2(s, s_ref)
    margins.record("K=V=64 precomputed gate (chunk_kda)", err, rl, rs)
    assert err <= O_MAX_ABS and rl <= O_REL_L2 and rs <= S_REL_L2, (err, rl, rs)


def test_padded_head_size_malformed_offsets_leave_out_untouched(cuda_device):
    x = sliced(kda_inputs.make_random("t", [100, 200, 50], 2, seed=123, state_std=0.1), 64, 64).to(cuda_device)
    cu_bad = torch.tensor([0, 200, 100, 350], dtype=torch.int32, device=cuda_device)
    out = torch.full_like(x.v, float("nan"))
    fin = torch.full((3, 2, 64, 64), float("nan"), device=cuda_device)
    ws = kda.new_workspace(350, 2, 3, cuda_device, 64, 64)
    kda.fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, out, ws, x.A_log, x.dt_bias, x.lower_bound, x.initial_state, fin,
            cu_bad)
    assert kda.read_device_status(ws) == 1
    assert torch.isnan(out).all()
    assert torch.equal(fin, x.initial_state)
