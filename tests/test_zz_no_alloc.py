"""kda_fwd_static_workspace: the forward pass for callers that cannot allocate device memory.

Some callers must not allocate while they run an operator (runtimes that plan every device
buffer ahead of time, or code that cannot afford cudaMalloc's device-wide synchronisation).  This
entry point takes the same inputs and outputs as kda_fwd but uses a workspace held by the library
itself.  The test calls it through the C ABI twice in a row and compares each result with the
ordinary entry point's (caller-provided workspace), within the parity tolerances of the other GPU
tests.  It sits in a file of its own, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import kda_inputs
import kimi_delta_attention_24_b200 as kda

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


def test_static_workspace_matches_kda_fwd(cuda_device):
    x = kda_inputs.make_workload("tail").to(cuda_device)
    B, T, H, K = x.q.shape
    N = x.num_seqs
    ref_out = torch.empty_like(x.v)
    ref_final = torch.empty(N, H, K, K, dtype=torch.float32, device=cuda_device)
    ws = kda.new_workspace(B * T, H, N, cuda_device)
    kda.fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, ref_out, ws, x.A_log, x.dt_bias, x.lower_bound,
            x.initial_state, ref_final, x.cu_seqlens)
    torch.cuda.synchronize()
    o_ref = ref_out.float().cpu().numpy()
    s_ref = ref_final.cpu().numpy()

    fn = _static_entry()
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    for _ in range(2):
        out = torch.full_like(x.v, float("nan"))
        final = torch.full((N, H, K, K), float("nan"), dtype=torch.float32, device=cuda_device)
        st = fn(p(x.q), p(x.k), p(x.v), p(x.g), p(x.beta), x.scale, p(out), p(x.A_log), p(x.dt_bias),
                x.lower_bound, p(x.initial_state), p(final), p(x.cu_seqlens), B, T, H, K, K, N, 0, stream)
        assert st == 0, kda.load().kda_status_string(st)
        torch.cuda.synchronize()
        o = out.float().cpu().numpy()
        s = final.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(s).all()
        assert np.max(np.abs(o - o_ref)) <= O_MAX_ABS and _rel_l2(o, o_ref) <= O_REL_L2
        assert _rel_l2(s, s_ref) <= S_REL_L2


def test_static_workspace_rejects_oversized_problems(cuda_device):
    fn = _static_entry()
    # 5000 heads x 1 sequence exceeds the 4096-unit limit: rejected on the host, nothing launched
    st = fn(None, None, None, None, None, 1.0, None, None, None, -5.0, None, None, None,
            1, 64, 5000, 128, 128, 1, 0, None)
    assert st == 3
