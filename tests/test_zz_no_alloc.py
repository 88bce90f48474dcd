"""kda_fwd_static_workspace: the forward pass for callers that cannot allocate device memory.

Some callers must not allocate while they run an operator (runtimes that plan every device
buffer ahead of time, or code that cannot afford cudaMalloc's device-wide synchronisation).  This
entry point takes the same inputs and outputs as kda_fwd but uses scratch held by the library
itself.  The tests call it through the C ABI twice in a row on each workload and compare every
result with the fp64 oracle and with the ordinary entry point (caller-provided workspace), within
the parity tolerances of the other GPU tests; they also check that the second call allocates no
device memory.  This file is collected last.
"""
import ctypes

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


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _static_entry():
    lib = kda.load()
    fn = lib.kda_fwd_static_workspace
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    fn.argtypes = [vp, vp, vp, vp, vp, f32, vp, vp, vp, f32, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32, vp]
    fn.restype = ctypes.c_int
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _close(o, s, o_ref, s_ref, what):
    assert np.isfinite(o).all() and (s is None or np.isfinite(s).all()), what
    margins.record(what, np.max(np.abs(o - o_ref)), _rel_l2(o, o_ref),
                   None if s_ref is None else _rel_l2(s, s_ref))
    assert np.max(np.abs(o - o_ref)) <= O_MAX_ABS and _rel_l2(o, o_ref) <= O_REL_L2, what
    if s_ref is not None:
        assert _rel_l2(s, s_ref) <= S_REL_L2, what


def _workload(name):
    if name == "tail":
        return kda_inputs.make_workload("tail"), False, False
    if name == "varlen-transposed":
        return kda_inputs.make_random("t", [150, 0, 64, 1, 300], 3, seed=51, state_std=0.2), True, False
    if name == "batch-transposed":
        return kda_inputs.make_random("t", None, 2, seed=52, varlen=False, batch=3, seqlen=130,
                                      state_std=0.1), True, False
    if name == "alias":
        return kda_inputs.make_random("t", [90, 200], 2, seed=53, state_std=0.3), False, True
    if name == "collinear":
        return kda_inputs.make_workload("collinear"), False, False
    raise KeyError(name)


@pytest.mark.parametrize("name", ["tail", "varlen-transposed", "batch-transposed", "alias", "collinear"])
def test_static_workspace_matches_oracle_and_kda_fwd(cuda_device, name):
    x, transposed, alias = _workload(name)
    o_ref, s_ref = oracle.fwd_inputs(x, state_transposed=transposed)
    xd = x.to(cuda_device)
    B, T, H, K = xd.q.shape
    N = xd.num_seqs
    s0 = xd.initial_state
    if s0 is not None and transposed:
        s0 = s0.transpose(-1, -2).contiguous()

    # the ordinary entry point, with a caller-provided workspace
    kd_out = torch.empty_like(xd.v)
    kd_final = torch.empty(N, H, K, K, dtype=torch.float32, device=cuda_device)
    ws = kda.new_workspace(B * T, H, N, cuda_device)
    kda.fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.scale, kd_out, ws, xd.A_log, xd.dt_bias, xd.lower_bound,
            s0, kd_final, xd.cu_seqlens, state_transposed=transposed)
    assert kda.read_device_status(ws) == 0
    o_kd = kd_out.float().cpu().double().numpy()
    s_kd = kd_final.cpu().double().numpy()
    del ws

    fn = _static_entry()
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    for call in range(2):
        out = torch.full_like(xd.v, float("nan"))
        if alias:
            final = s0.clone()
            init = final
        else:
            final = torch.full((N, H, K, K), float("nan"), dtype=torch.float32, device=cuda_device)
            init = s0
        torch.cuda.synchronize()
        before_alloc = torch.cuda.memory_allocated(cuda_device)
        before_free = torch.cuda.mem_get_info(cuda_device)[0]
        st = fn(_p(xd.q), _p(xd.k), _p(xd.v), _p(xd.g), _p(xd.beta), xd.scale, _p(out), _p(xd.A_log),
                _p(xd.dt_bias), xd.lower_bound, _p(init), _p(final), _p(xd.cu_seqlens),
                B, T, H, K, K, 0 if xd.cu_seqlens is None else N, int(transposed), stream)
        assert st == 0, kda.load().kda_status_string(st)
        torch.cuda.synchronize()
        if call == 1:
            # the second call allocates nothing (the first may load the library's device code)
            assert torch.cuda.memory_allocated(cuda_device) == before_alloc
            assert torch.cuda.mem_get_info(cuda_device)[0] == before_free
        o = out.float().cpu().double().numpy()
        s = final.cpu().double().numpy()
        _close(o, s, o_ref, s_ref, f"{name}, call {call}: against the oracle")
        _close(o, s, o_kd, s_kd, f"{name}, call {call}: against kda_fwd")


def test_static_workspace_rejects_oversized_problems(cuda_device):
    """4100 (sequence, head) units exceed the 4096-unit limit: KDA_ERR_WORKSPACE_TOO_SMALL, after the
    arguments have been validated (null pointers give KDA_ERR_INVALID_ARGUMENT first), with
    nothing enqueued and the outputs untouched."""
    fn = _static_entry()
    x = kda_inputs.make_random("t", None, 100, seed=54, varlen=False, batch=41, seqlen=1).to(cuda_device)
    out = torch.full_like(x.v, float("nan"))
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    st = fn(_p(x.q), _p(x.k), _p(x.v), _p(x.g), _p(x.beta), x.scale, _p(out), _p(x.A_log), _p(x.dt_bias),
            x.lower_bound, None, None, None, 41, 1, 100, 128, 128, 0, 0, stream)
    assert st == 3  # KDA_ERR_WORKSPACE_TOO_SMALL
    st = fn(None, None, None, None, None, 1.0, None, None, None, -5.0, None, None, None,
            41, 1, 100, 128, 128, 0, 0, stream)
    assert st == 1  # KDA_ERR_INVALID_ARGUMENT
    torch.cuda.synchronize()
    assert torch.isnan(out).all()


def test_static_workspace_malformed_offsets_leave_documents_empty(cuda_device):
    """Offsets that do not tile the tokens in order: as with kda_fwd every document is treated as
    empty (out untouched, final state = initial state); the status is not reported by this entry."""
    fn = _static_entry()
    x = kda_inputs.make_random("t", [100, 200, 50], 2, seed=55, state_std=0.1).to(cuda_device)
    cu_bad = torch.tensor([0, 200, 100, 350], dtype=torch.int32, device=cuda_device)
    out = torch.full_like(x.v, float("nan"))
    fin = torch.full((3, 2, 128, 128), float("nan"), device=cuda_device)
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    st = fn(_p(x.q), _p(x.k), _p(x.v), _p(x.g), _p(x.beta), x.scale, _p(out), _p(x.A_log), _p(x.dt_bias),
            x.lower_bound, _p(x.initial_state), _p(fin), _p(cu_bad), 1, 350, 2, 128, 128, 3, 0, stream)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.isnan(out).all()
    assert torch.equal(fin, x.initial_state)
