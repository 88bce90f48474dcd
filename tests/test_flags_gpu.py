"""GPU parity of the chunked forward with input transforms switched off (kda_fwd_ex flags, fla
chunk_kda's use_gate_in_kernel / use_qk_l2norm_in_kernel / use_beta_sigmoid_in_kernel) against the
fp64 oracle's recurrence fed the same transformed inputs."""
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
    assert np.isfinite(o).all() and np.isfinite(s).all(), what
    err = float(np.max(np.abs(o - o_ref)))
    rl, rs = rel_l2(o, o_ref), rel_l2(s, s_ref)
    margins.record(what, err, rl, rs)
    print(f"{what}: o max-abs {err:.3e}, o rel-L2 {rl:.3e}, state rel-L2 {rs:.3e}")
    assert err <= O_MAX_ABS and rl <= O_REL_L2, what
    assert rs <= S_REL_L2, what


def transformed(x, flags, log_alpha_shift=0.0):
    """Kernel inputs for `flags` and the oracle's transformed inputs (qhat, khat, log alpha, beta)
    computed from exactly the values the kernel reads."""
    qh, kh, la, be = oracle.prologue(x.q, x.k, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound)
    q_in, k_in, g_in, beta_in = x.q, x.k, x.g, x.beta
    if flags & kda.FLAG_GATE_PRECOMPUTED:
        g_in = torch.from_numpy(la + log_alpha_shift).float()
        # the kernel clamps log alpha to [lower_bound, 0]
        la = np.clip(g_in.double().numpy(), x.lower_bound, 0.0)
    if flags & kda.FLAG_BETA_PRECOMPUTED:
        beta_in = torch.from_numpy(be).float()
        be = beta_in.double().numpy()
    if flags & kda.FLAG_NO_QK_L2NORM:
        # unnormalised q and k of moderate size, so that the delta rule stays contractive
        q_in = (x.q.float() * 0.2).to(torch.bfloat16)
        k_in = (x.k.float() * 0.08).to(torch.bfloat16)
        qh, kh = q_in.double().numpy(), k_in.double().numpy()
    return (q_in, k_in, g_in, beta_in), (qh, kh, la, be)


def run_case(dev, x, flags, log_alpha_shift=0.0):
    (q_in, k_in, g_in, beta_in), (qh, kh, la, be) = transformed(x, flags, log_alpha_shift)
    B, T, H, K = x.q.shape
    N = x.num_seqs
    cu = x.cu_seqlens.numpy() if x.cu_seqlens is not None else np.arange(B + 1, dtype=np.int32) * T
    tok = lambda a: np.ascontiguousarray(a.reshape(B * T, H, *a.shape[3:]))
    o_ref, s_ref = oracle.core(tok(qh), tok(kh), tok(x.v.double().numpy()), tok(la), tok(be), x.scale,
                               S0=x.initial_state.double().numpy(), cu_seqlens=cu)
    out = torch.full_like(x.v, float("nan"), device=dev)
    fin = torch.full((N, H, K, K), float("nan"), device=dev)
    ws = kda.new_workspace(B * T, H, N, dev)
    gate_pre = flags & kda.FLAG_GATE_PRECOMPUTED
    kda.fwd(q_in.to(dev), k_in.to(dev), x.v.to(dev), g_in.to(dev), beta_in.to(dev), x.scale, out, ws,
            None if gate_pre else x.A_log.to(dev), None if gate_pre else x.dt_bias.to(dev), x.lower_bound,
            x.initial_state.to(dev), fin, None if x.cu_seqlens is None else x.cu_seqlens.to(dev), flags=flags)
    assert kda.read_device_status(ws) == 0
    return out.float().cpu().double().numpy().reshape(B * T, H, K), fin.cpu().double().numpy(), o_ref, s_ref


@pytest.mark.parametrize("flags", [1, 2, 4, 3, 5, 6, 7])
def test_chunked_flags_varlen(cuda_device, flags):
    """Documents with partial last chunks, an empty one, and one that spans the two-stage cut."""
    x = kda_inputs.make_random("t", [300, 0, 65, 1000, 17], 4, seed=71, state_std=0.1)
    check(*run_case(cuda_device, x, flags), f"chunked flags={flags}")


def test_chunked_precomputed_gate_is_clamped(cuda_device):
    """Precomputed log alpha pushed below lower_bound on some channels (down to -7) is clamped to
    it, and exactly 0 stays 0: the oracle is fed the clamped values."""
    x = kda_inputs.make_random("t", [200, 129], 3, seed=72, state_std=0.1)
    check(*run_case(cuda_device, x, kda.FLAG_GATE_PRECOMPUTED, log_alpha_shift=-2.0), "clamped log alpha")


def test_chunked_flags_batch_mode_one_stage(cuda_device):
    """Batch mode with more units than SMs (one stage), all flags."""
    x = kda_inputs.make_random("t", None, 80, seed=73, varlen=False, batch=2, seqlen=150, state_std=0.1)
    check(*run_case(cuda_device, x, 7), "chunked flags=7 batch mode")


def test_chunk_kda_flag_keywords(cuda_device):
    """chunk_kda(use_gate_in_kernel=False, use_beta_sigmoid_in_kernel=False) equals the flagged fwd."""
    x = kda_inputs.make_random("t", [130, 70], 2, seed=74, state_std=0.1)
    o_k, s_k, o_ref, s_ref = run_case(cuda_device, x, 5)
    (q_in, k_in, g_in, beta_in), _ = transformed(x, 5)
    dev = cuda_device
    out, fin = kda.chunk_kda(q_in.to(dev), k_in.to(dev), x.v.to(dev), g_in.to(dev), beta_in.to(dev),
                             scale=x.scale, initial_state=x.initial_state.to(dev), output_final_state=True,
                             lower_bound=x.lower_bound, cu_seqlens=x.cu_seqlens.to(dev),
                             use_gate_in_kernel=False, use_beta_sigmoid_in_kernel=False)
    o = out.float().cpu().double().numpy().reshape(o_ref.shape)
    check(o, fin.cpu().double().numpy(), o_ref, s_ref, "chunk_kda keywords")
    np.testing.assert_array_equal(o, o_k)
