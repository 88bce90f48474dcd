"""GPU parity of the backward pass (kda_bwd) against the oracle's fp64 adjoint.

Every gradient (q, k, v, raw gate, raw beta, A_log, dt_bias, the initial state) is compared with
oracle.kda_bwd on the same seeded inputs: relative L2 <= 1e-2 and every element finite (the
token gradients are bf16, as the inputs are).
"""
import numpy as np
import pytest
import torch

import kda_inputs
import kimi_delta_attention_24_b200 as kda
import margins
import oracle

pytestmark = pytest.mark.gpu

G_REL_L2 = 1e-2


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def run_case(dev, x, seed, with_final=True, use_checkpoints=False):
    rng = np.random.default_rng(seed)
    d_out = torch.from_numpy(rng.standard_normal(x.v.shape)).to(torch.bfloat16)
    N, H = x.num_seqs, x.num_heads
    d_final = torch.from_numpy(rng.standard_normal((N, H, 128, 128)) * 0.3).float() if with_final else None
    ref = oracle.kda_bwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, d_out,
                         initial_state=x.initial_state, d_final=d_final, cu_seqlens=x.cu_seqlens)
    xd = x.to(dev)
    ck = None
    if use_checkpoints:
        # the training forward: output, final state and the chunk-start states for the backward
        B, T = x.q.shape[:2]
        ck = torch.empty(kda.checkpoint_size(B * T, H, N) // 4, dtype=torch.float32, device=dev)
        out = torch.empty_like(xd.v)
        ws = kda.new_workspace(B * T, H, N, dev)
        kda.fwd_checkpointed(xd.q, xd.k, xd.v, xd.g, xd.beta, x.scale, out, ws, xd.A_log, xd.dt_bias, x.lower_bound,
                             ck, initial_state=xd.initial_state, cu_seqlens=xd.cu_seqlens)
        assert kda.read_device_status(ws) == 0
    got = kda.bwd(xd.q, xd.k, xd.v, xd.g, xd.beta, x.scale, xd.A_log, xd.dt_bias, x.lower_bound, d_out.to(dev),
                  initial_state=xd.initial_state, d_final=None if d_final is None else d_final.to(dev),
                  cu_seqlens=xd.cu_seqlens, checkpoints=ck)
    torch.cuda.synchronize()
    return got, ref


def check_grads(got, ref, what, sum_scale=None):
    """Relative L2 per gradient; a gradient named in sum_scale (a sum whose terms cancel) is checked
    element-wise against the sum of its terms' magnitudes instead: |got - ref| <= 1e-3 x scale."""
    worst = []
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias", "d_initial"):
        g = got[name].float().cpu().double().numpy()
        assert np.isfinite(g).all(), f"{what}: {name} not finite"
        if sum_scale and name in sum_scale:
            err = float(np.max(np.abs(g - ref[name]) / sum_scale[name]))
            worst.append(f"{name} {err:.2e} of the terms' magnitude")
            margins.note(f"backward {what} {name}: error / sum of |terms| {err:.2e} (tol 1e-03)")
            assert err <= 1e-3, f"{what}: {name} error {err:.3e} of the sum of its terms' magnitudes"
            continue
        err = rel_l2(g, ref[name])
        worst.append(f"{name} {err:.2e}")
        margins.note(f"backward {what} {name}: rel-L2 {err:.2e} (tol 1e-02)")
        assert err <= G_REL_L2, f"{what}: {name} rel-L2 {err:.3e}"
    print(f"bwd {what}: " + ", ".join(worst))


def test_bwd_varlen_with_tails_and_empty_document(cuda_device):
    x = kda_inputs.make_random("t", [130, 0, 64, 1, 200], 3, seed=111, state_std=0.2)
    check_grads(*run_case(cuda_device, x, 1), "varlen")


def test_bwd_batch_mode_without_final_gradient(cuda_device):
    x = kda_inputs.make_random("t", None, 4, seed=112, varlen=False, batch=2, seqlen=150, state_std=0.1)
    check_grads(*run_case(cuda_device, x, 2, with_final=False), "batch, no d_final")


def test_bwd_slow_decay_and_zero_initial_state(cuda_device):
    """Gates near alpha = 1 (raw gate -6) carry gradients across many chunks; lower_bound -1."""
    x = kda_inputs.make_random("t", [300], 2, seed=113, lower_bound=-1.0)
    x.g.fill_(-6.0)
    check_grads(*run_case(cuda_device, x, 3), "slow decay")


def test_bwd_many_units_more_than_sms(cuda_device):
    """200 (sequence, head) units: the persistent CTAs take several units each."""
    x = kda_inputs.make_random("t", [40, 70, 3, 100], 50, seed=114, state_std=0.1)
    check_grads(*run_case(cuda_device, x, 4), "200 units")


@pytest.mark.parametrize("lens,H", [([130, 0, 64, 1, 200], 3), ([2000], 4), ([700, 9000], 12)])
def test_bwd_with_forward_checkpoints(cuda_device, lens, H):
    """The training path: kda_fwd_checkpointed stores the chunk-start states (the second shape runs
    the forward in two stages, the third cuts a sequence between them) and kda_bwd starts from them."""
    x = kda_inputs.make_random("t", lens, H, seed=115, state_std=0.2)
    x.g[:, :, :, :64].fill_(-6.0)  # half the channels decay slowly: states carry across chunks
    check_grads(*run_case(cuda_device, x, 5, use_checkpoints=True), f"checkpoints {lens} H={H}")


def test_forward_checkpoints_are_chunk_start_states(cuda_device):
    """The stored checkpoints equal the oracle's state after 64 c tokens (S^T layout)."""
    lens, H = [300, 130], 2
    x = kda_inputs.make_random("t", lens, H, seed=116, state_std=0.2)
    x.g.fill_(-6.0)
    xd = x.to(cuda_device)
    ck = torch.full((kda.checkpoint_size(430, H, 2) // 4,), float("nan"), device=cuda_device)
    out = torch.empty_like(xd.v)
    ws = kda.new_workspace(430, H, 2, cuda_device)
    kda.fwd_checkpointed(xd.q, xd.k, xd.v, xd.g, xd.beta, x.scale, out, ws, xd.A_log, xd.dt_bias, x.lower_bound, ck,
                         initial_state=xd.initial_state, cu_seqlens=xd.cu_seqlens)
    ck = ck.cpu().double().numpy().reshape(-1, H, 128, 128)
    cu = x.cu_seqlens.tolist()
    for n in range(2):
        for c in range((lens[n] + 63) // 64):
            t_end = cu[n] + 64 * c
            sub = lambda t: t[:, cu[n]:t_end].contiguous()
            _, s_ref = oracle.kda_fwd(sub(x.q), sub(x.k), sub(x.v), sub(x.g), sub(x.beta), x.scale, x.A_log,
                                      x.dt_bias, x.lower_bound, initial_state=x.initial_state[n:n + 1],
                                      cu_seqlens=torch.tensor([0, t_end - cu[n]], dtype=torch.int32))
            slot = cu[n] // 64 + n + c
            got = np.swapaxes(ck[slot], -1, -2)
            err = rel_l2(got, s_ref[0])
            assert np.isfinite(got).all() and err <= 1e-2, (n, c, err)


def test_bwd_long_sequence_few_heads(cuda_device):
    """One 3000-token sequence over 2 heads: 47 chunks per (sequence, head), so the state gradient
    crosses many chunk boundaries while the chunk-parallel kernels take the chunks side by side."""
    x = kda_inputs.make_random("t", [3000], 2, seed=117, state_std=0.2)
    x.g[:, :, :, 64:].fill_(-6.0)  # half the channels decay slowly
    check_grads(*run_case(cuda_device, x, 6), "3000 tokens x 2 heads")


def test_bwd_saturated_gates_and_empty_documents(cuda_device):
    """Gates at the lower bound (raw gate 60: log alpha = -5 in every channel) and empty documents
    between non-empty ones: the decay-weighted products then span e^{-80} .. e^{80} per sub-block."""
    x = kda_inputs.make_random("t", [0, 150, 0, 0, 77], 2, seed=118, state_std=0.2)
    x.g[:, :, 0, :].fill_(60.0)
    check_grads(*run_case(cuda_device, x, 7), "saturated gate, empty documents")


def test_bwd_near_collinear_keys(cuda_device):
    """The forward's stress input (every key the same vector, beta = sigmoid(8), raw gate -12: alpha
    close to 1, so (I + A) is close to I plus a strictly lower all-ones matrix) through the backward,
    over six chunks with a ragged tail.  The queries are drawn at random here: with q = k, as in the
    forward's case, every output depends on q only through khat . qhat = 1 and dq vanishes (the
    oracle's is 1e-8), which a relative comparison cannot check."""
    x = kda_inputs.make_collinear(336, seed=5)
    x.q = torch.randn(x.q.shape, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    got, ref = run_case(cuda_device, x, 9)
    # dA_log = sum over tokens and channels of dg (g + dt_bias) (the gate's chain rule); here those
    # terms cancel to 2e-7 of their magnitudes (5.9e-7 against 3.1), below what any fp32 sum
    # resolves, so dA_log is held to its terms' magnitude instead of to its own value
    terms = ref["dg"].reshape(-1, x.num_heads, 128) * (x.g.double().numpy().reshape(-1, x.num_heads, 128)
                                                       + x.dt_bias.double().numpy()[None])
    check_grads(got, ref, "near-collinear keys", sum_scale={"dA_log": np.abs(terms).sum(axis=(0, 2))})


def test_bwd_malformed_offsets_report_and_pass_the_state_gradient_through(cuda_device):
    """Out-of-order cu_seqlens: every document is empty, d_initial = d_final and the workspace's
    status word says so."""
    x = kda_inputs.make_random("t", [100, 200, 50], 2, seed=119, state_std=0.1).to(cuda_device)
    cu_bad = torch.tensor([0, 200, 100, 350], dtype=torch.int32, device=cuda_device)
    d_out = torch.randn(x.v.shape, device=cuda_device).to(torch.bfloat16)
    d_final = torch.randn(3, 2, 128, 128, device=cuda_device)
    ws = torch.empty(kda.bwd_workspace_size(350, 2, 3), dtype=torch.uint8, device=cuda_device)
    got = kda.bwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, d_out,
                  initial_state=x.initial_state, d_final=d_final, cu_seqlens=cu_bad, workspace=ws)
    assert kda.read_device_status(ws) == 1
    assert torch.equal(got["d_initial"], d_final)
    assert torch.count_nonzero(got["dA_log"]) == 0 and torch.count_nonzero(got["ddt_bias"]) == 0


def test_bwd_bench_workload_sampled_heads(cuda_device):
    """The bench's backward at its full size and in its launch configuration (B = 1, T = 4096, 96
    heads, from the checkpointing forward's states, inputs generated on the device as the bench does):
    three heads against the oracle, which takes each head alone (heads are independent)."""
    T, H = 4096, 96
    dev = cuda_device
    x = kda_inputs.make_random("bwd", [T], H, seed=0, device=dev)
    gen = torch.Generator(device=dev).manual_seed(11)
    d_out = torch.randn(x.v.shape, generator=gen, device=dev).to(torch.bfloat16)
    ck = torch.empty(kda.checkpoint_size(T, H, 1) // 4, dtype=torch.float32, device=dev)
    ws = kda.new_workspace(T, H, 1, dev)
    out = torch.empty_like(x.v)
    kda.fwd_checkpointed(x.q, x.k, x.v, x.g, x.beta, x.scale, out, ws, x.A_log, x.dt_bias, x.lower_bound, ck,
                         cu_seqlens=x.cu_seqlens)
    got = kda.bwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, d_out,
                  cu_seqlens=x.cu_seqlens, checkpoints=ck)
    torch.cuda.synchronize()
    assert kda.read_device_status(ws) == 0
    for h in (0, 47, 95):
        tok = lambda t: t[:, :, h:h + 1].contiguous().cpu()
        ref = oracle.kda_bwd(tok(x.q), tok(x.k), tok(x.v), tok(x.g), tok(x.beta), x.scale,
                             x.A_log[h:h + 1].cpu(), x.dt_bias[h:h + 1].cpu(), x.lower_bound, tok(d_out),
                             cu_seqlens=x.cu_seqlens.cpu())
        sub = {n: tok(got[n]) for n in ("dq", "dk", "dv", "dg", "dbeta")}
        sub["dA_log"] = got["dA_log"][h:h + 1].cpu()
        sub["ddt_bias"] = got["ddt_bias"][h:h + 1].cpu()
        sub["d_initial"] = got["d_initial"][:, h:h + 1].cpu()
        check_grads(sub, ref, f"bench workload T=4096 H=96, head {h}")
