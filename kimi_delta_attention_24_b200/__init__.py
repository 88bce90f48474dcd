"""B200 (sm_100a) Kimi Delta Attention forward: Python binding of libkda_b200.so.

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.

    fwd(q, k, v, g, beta, scale, out, workspace, A_log, dt_bias, lower_bound,
        initial_state, final_state, cu_seqlens)          # FlashKDA-style, writes in place
    get_workspace_size(T, H, N)
    is_supported(head_dim, dtype, lower_bound)
    chunk_kda(q, k, v, g, beta, ...) -> (out, final_state)  # fla-style, allocates outputs
    fwd_recurrent(...)                                     # token-serial CUDA-core kernel
    decode(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound,
           state_in, state_out, state_indices)             # batched recurrent step on a state pool

The argument order of ``fwd`` follows FlashKDA's ``fwd`` as printed in the vLLM PR #54859 report
(test_flashkda_near_collinear_keys_remain_finite); ``chunk_kda`` follows the fla call on the page
"What CUDA Version Is Required to Use FlashKDA?", section Usage Examples.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["get_workspace_size_ex", "fwd", "fwd_recurrent", "decode", "segment_map", "state_affine", "bwd", "bwd_workspace_size",
           "checkpoint_size", "fwd_checkpointed", "FLAG_GATE_PRECOMPUTED", "FLAG_NO_QK_L2NORM",
           "FLAG_BETA_PRECOMPUTED", "get_workspace_size", "fwd_launch_count", "new_workspace",
           "is_supported", "chunk_kda", "read_device_status", "selftest_wait_timeout", "KDAError",
           "library_path", "load"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "lib", "libkda_b200.so")
_lib = None

_STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARGUMENT", 2: "KDA_ERR_UNSUPPORTED",
           3: "KDA_ERR_WORKSPACE_TOO_SMALL", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_DEVICE_TIMEOUT"}


# input-transform flags (include/kda.h: KDA_FLAG_*)
FLAG_GATE_PRECOMPUTED = 1   # g holds fp32 log alpha
FLAG_NO_QK_L2NORM = 2       # q, k used as given
FLAG_BETA_PRECOMPUTED = 4   # beta holds fp32 beta


class KDAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load():
    """Loads libkda_b200.so.  Raises if it has not been built: there is no fallback path."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is not built; run `python -m kimi_delta_attention_24_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    fwd_args = [vp, vp, vp, vp, vp, f32, vp, vp, ctypes.c_size_t, vp, vp, f32, vp, vp, vp,
                i32, i64, i32, i32, i32, i32, i32, vp]
    for name in ("kda_fwd", "kda_fwd_recurrent"):
        fn = getattr(lib, name)
        fn.argtypes = fwd_args
        fn.restype = ctypes.c_int
    lib.kda_fwd_ex.argtypes = fwd_args[:-1] + [ctypes.c_uint32, vp]
    lib.kda_fwd_ex.restype = ctypes.c_int
    lib.kda_decode.argtypes = [vp, vp, vp, vp, vp, f32, vp, vp, vp, f32, vp, vp, vp, i32, i32, i32, i32, i32,
                               i64, i32, ctypes.c_uint32, vp, vp]
    lib.kda_decode.restype = ctypes.c_int
    lib.kda_segment_map.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp, f32, vp, vp, vp,
                                    i32, i64, i32, i32, i32, i32, ctypes.c_uint32, vp]
    lib.kda_segment_map.restype = ctypes.c_int
    lib.kda_state_affine.argtypes = [vp, vp, vp, vp, i64, i32, i32, vp]
    lib.kda_state_affine.restype = ctypes.c_int
    lib.kda_bwd_workspace_size.argtypes = [i64, i32, i32]
    lib.kda_bwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_bwd.argtypes = [vp, vp, vp, vp, vp, f32, vp, vp, f32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                            vp, ctypes.c_size_t, vp, i32, i64, i32, i32, i32, i32, vp]
    lib.kda_checkpoint_size.argtypes = [i64, i32, i32]
    lib.kda_checkpoint_size.restype = ctypes.c_size_t
    lib.kda_fwd_checkpointed.argtypes = [vp, vp, vp, vp, vp, f32, vp, vp, ctypes.c_size_t, vp, vp, f32, vp, vp, vp,
                                         ctypes.c_size_t, vp, i32, i64, i32, i32, i32, i32, vp]
    lib.kda_fwd_checkpointed.restype = ctypes.c_int
    lib.kda_bwd.restype = ctypes.c_int
    lib.kda_workspace_size_ex.argtypes = [i64, i32, i32, i32, i32]
    lib.kda_workspace_size_ex.restype = ctypes.c_size_t
    lib.kda_workspace_size.argtypes = [i64, i32, i32]
    lib.kda_workspace_size.restype = ctypes.c_size_t
    lib.kda_fwd_launch_count.argtypes = [i64, i32, i32]
    lib.kda_fwd_launch_count.restype = ctypes.c_int
    lib.kda_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint32, vp]
    lib.kda_selftest_wait_timeout.restype = ctypes.c_int
    lib.kda_is_supported.argtypes = [ctypes.c_int, ctypes.c_int, f32]
    lib.kda_is_supported.restype = ctypes.c_int
    lib.kda_read_device_status.argtypes = [vp, vp]
    lib.kda_read_device_status.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def get_workspace_size(T: int, H: int, N: int) -> int:
    return int(load().kda_workspace_size(int(T), int(H), int(N)))


def fwd_launch_count(T: int, H: int, N: int) -> int:
    """Kernel launches one fwd call over (T tokens, H heads, N sequences) enqueues on the current
    device (3, or 5 when the chunk range runs in two stages)."""
    return int(load().kda_fwd_launch_count(int(T), int(H), int(N)))


def get_workspace_size_ex(T: int, H: int, N: int, K: int = 128, V: int = 128) -> int:
    return int(load().kda_workspace_size_ex(int(T), int(H), int(N), int(K), int(V)))


def new_workspace(T: int, H: int, N: int, device, K: int = 128, V: int = 128) -> torch.Tensor:
    """A workspace for kda.fwd (head sizes K, V): uninitialised except for its 256-byte header
    (status word and item counters), which is zeroed."""
    ws = torch.empty(get_workspace_size_ex(T, H, N, K, V), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def is_supported(head_dim: int, dtype=torch.bfloat16, lower_bound: float = -5.0) -> bool:
    return bool(load().kda_is_supported(int(head_dim), int(dtype == torch.bfloat16), float(lower_bound)))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t: Optional[torch.Tensor], name: str, dtype, device):
    if t is None:
        return
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _call(fn_name, q, k, v, g, beta, scale, out, workspace, A_log, dt_bias, lower_bound,
          initial_state, final_state, cu_seqlens, state_transposed, stream, flags=0):
    lib = load()
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n, torch.bfloat16, dev)
    _check(g, "g", torch.float32 if flags & FLAG_GATE_PRECOMPUTED else torch.bfloat16, dev)
    _check(beta, "beta", torch.float32 if flags & FLAG_BETA_PRECOMPUTED else torch.bfloat16, dev)
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias"), (initial_state, "initial_state"),
                 (final_state, "final_state")):
        _check(t, n, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if workspace is not None:
        _check(workspace, "workspace", torch.uint8, dev)
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, K]")
    B, T, H, K = q.shape
    V = v.shape[-1]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(out), _ptr(workspace),
            0 if workspace is None else workspace.numel(), _ptr(A_log), _ptr(dt_bias), float(lower_bound),
            _ptr(initial_state), _ptr(final_state), _ptr(cu_seqlens), B, T, H, K, V, N,
            int(bool(state_transposed))]
    if fn_name == "kda_fwd_ex":
        args.append(int(flags))
    with torch.cuda.device(dev):
        st = getattr(lib, fn_name)(*args, ctypes.c_void_p(stream))
    if st != 0:
        raise KDAError(st, fn_name)


def fwd(q, k, v, g, beta, scale, out, workspace, A_log, dt_bias, lower_bound,
        initial_state=None, final_state=None, cu_seqlens=None, state_transposed=False, stream=None,
        flags=0):
    """The chunked forward (tcgen05 kernels).  Writes ``out`` and ``final_state`` in place.
    ``flags`` (FLAG_*) switches input transforms off (kda_fwd_ex); 0 is kda_fwd."""
    ex = flags or q.shape[-1] != 128 or v.shape[-1] != 128
    _call("kda_fwd_ex" if ex else "kda_fwd", q, k, v, g, beta, scale, out, workspace, A_log, dt_bias,
          lower_bound, initial_state, final_state, cu_seqlens, state_transposed, stream, flags)


def fwd_recurrent(q, k, v, g, beta, scale, out, workspace, A_log, dt_bias, lower_bound,
                  initial_state=None, final_state=None, cu_seqlens=None, state_transposed=False,
                  stream=None):
    """The token-serial CUDA-core kernel (same contract as ``fwd``)."""
    _call("kda_fwd_recurrent", q, k, v, g, beta, scale, out, workspace, A_log, dt_bias,
          lower_bound, initial_state, final_state, cu_seqlens, state_transposed, stream)


def decode(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound, state_in=None, state_out=None,
           state_indices=None, state_transposed=False, flags=0, workspace=None, stream=None):
    """Batched recurrent step: request b advances pool slot ``state_indices[b]`` (b when None;
    negative: skipped) by its ``T`` tokens and writes ``out`` in place.

    q, k, v, out: bf16 [B, T, H, 128] (or [B, H, 128] for one token); g: bf16 raw gate, or fp32 log
    alpha with FLAG_GATE_PRECOMPUTED; beta: bf16 [B, T, H] raw, or fp32 beta with
    FLAG_BETA_PRECOMPUTED; state pools fp32 [slots, H, 128, 128] (state_in may be state_out)."""
    lib = load()
    if q.dim() == 3:
        q, k, v, out, g = (t.unsqueeze(1) for t in (q, k, v, out, g))
        beta = beta.unsqueeze(1)
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check(t, n, torch.bfloat16, dev)
    _check(g, "g", torch.float32 if flags & FLAG_GATE_PRECOMPUTED else torch.bfloat16, dev)
    _check(beta, "beta", torch.float32 if flags & FLAG_BETA_PRECOMPUTED else torch.bfloat16, dev)
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias"), (state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, torch.float32, dev)
    _check(state_indices, "state_indices", torch.int32, dev)
    if workspace is not None:
        _check(workspace, "workspace", torch.uint8, dev)
    B, T, H, K = q.shape
    V = v.shape[-1]
    pool = state_out if state_out is not None else state_in
    slots = pool.shape[0] if pool is not None else B
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        st = lib.kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(out),
                            _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(state_in), _ptr(state_out),
                            _ptr(state_indices), B, T, H, K, V, slots, int(bool(state_transposed)),
                            int(flags), _ptr(workspace), ctypes.c_void_p(stream))
    if st != 0:
        raise KDAError(st, "kda_decode")


def segment_map(q, k, v, g, beta, workspace, A_log, dt_bias, lower_bound, map_M, map_B, cu_seqlens=None,
                flags=0, stream=None):
    """The affine map S_out = M S_in + B of every (sequence, head) unit's tokens: writes map_M
    (fp32 [N, H, K, K]) and map_B (fp32 [N, H, K, V]) in place (kda_segment_map)."""
    lib = load()
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.bfloat16, dev)
    _check(g, "g", torch.float32 if flags & FLAG_GATE_PRECOMPUTED else torch.bfloat16, dev)
    _check(beta, "beta", torch.float32 if flags & FLAG_BETA_PRECOMPUTED else torch.bfloat16, dev)
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias"), (map_M, "map_M"), (map_B, "map_B")):
        _check(t, n, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _check(workspace, "workspace", torch.uint8, dev)
    B, T, H, K = q.shape
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        st = lib.kda_segment_map(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(workspace),
                                 workspace.numel(), _ptr(A_log), _ptr(dt_bias), float(lower_bound),
                                 _ptr(map_M), _ptr(map_B), _ptr(cu_seqlens), B, T, H, K, v.shape[-1], N,
                                 int(flags), ctypes.c_void_p(stream))
    if st != 0:
        raise KDAError(st, "kda_segment_map")


def state_affine(map_M, map_B, state_in, state_out, state_transposed=False, stream=None):
    """state_out = map_M state_in + map_B per (sequence, head) unit (state_in None: zero state);
    state_out may be state_in (kda_state_affine)."""
    lib = load()
    dev = map_B.device
    for t, n in ((map_M, "map_M"), (map_B, "map_B"), (state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, torch.float32, dev)
    units = map_B.numel() // (map_B.shape[-1] * map_B.shape[-2])
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        st = lib.kda_state_affine(_ptr(map_M), _ptr(map_B), _ptr(state_in), _ptr(state_out), units,
                                  map_B.shape[-1], int(bool(state_transposed)), ctypes.c_void_p(stream))
    if st != 0:
        raise KDAError(st, "kda_state_affine")


def bwd_workspace_size(T: int, H: int, N: int) -> int:
    return int(load().kda_bwd_workspace_size(int(T), int(H), int(N)))


def checkpoint_size(T: int, H: int, N: int) -> int:
    return int(load().kda_checkpoint_size(int(T), int(H), int(N)))


def fwd_checkpointed(q, k, v, g, beta, scale, out, workspace, A_log, dt_bias, lower_bound, checkpoints,
                     initial_state=None, final_state=None, cu_seqlens=None, stream=None):
    """kda.fwd that also stores the state at the start of every 64-token chunk in ``checkpoints``
    (fp32, at least checkpoint_size(T, H, N) bytes' worth) for kda.bwd (kda_fwd_checkpointed)."""
    lib = load()
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta"), (out, "out")):
        _check(t, n, torch.bfloat16, dev)
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias"), (initial_state, "initial_state"),
                 (final_state, "final_state"), (checkpoints, "checkpoints")):
        _check(t, n, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _check(workspace, "workspace", torch.uint8, dev)
    B, T, H, K = q.shape
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        st = lib.kda_fwd_checkpointed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(out),
                                      _ptr(workspace), workspace.numel(), _ptr(A_log), _ptr(dt_bias),
                                      float(lower_bound), _ptr(initial_state), _ptr(final_state), _ptr(checkpoints),
                                      checkpoints.numel() * 4, _ptr(cu_seqlens), B, T, H, K, v.shape[-1], N,
                                      ctypes.c_void_p(stream))
    if st != 0:
        raise KDAError(st, "kda_fwd_checkpointed")


def bwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, d_out, initial_state=None, d_final=None,
        cu_seqlens=None, workspace=None, stream=None, checkpoints=None):
    """Gradients of sum(d_out * o) + sum(d_final * final_state) w.r.t. every input (kda_bwd), using
    ``checkpoints`` from fwd_checkpointed when given.  Returns a dict: dq, dk, dv, dg (bf16, shaped
    like the inputs), dbeta (bf16, like beta), dA_log [H], ddt_bias [H, K] and d_initial
    [N, H, K, V] (fp32)."""
    lib = load()
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta"), (d_out, "d_out")):
        _check(t, n, torch.bfloat16, dev)
    for t, n in ((A_log, "A_log"), (dt_bias, "dt_bias"), (initial_state, "initial_state"), (d_final, "d_final"),
                 (checkpoints, "checkpoints")):
        _check(t, n, torch.float32, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    B, T, H, K = q.shape
    V = v.shape[-1]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B * T, H, N), dtype=torch.uint8, device=dev)
    r = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v), "dg": torch.empty_like(g),
         "dbeta": torch.empty_like(beta), "dA_log": torch.empty(H, dtype=torch.float32, device=dev),
         "ddt_bias": torch.empty(H, K, dtype=torch.float32, device=dev),
         "d_initial": torch.empty(N, H, K, V, dtype=torch.float32, device=dev)}
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    with torch.cuda.device(dev):
        st = lib.kda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(A_log), _ptr(dt_bias),
                         float(lower_bound), _ptr(initial_state), _ptr(d_out), _ptr(d_final), _ptr(checkpoints),
                         _ptr(r["dq"]),
                         _ptr(r["dk"]), _ptr(r["dv"]), _ptr(r["dg"]), _ptr(r["dbeta"]), _ptr(r["dA_log"]),
                         _ptr(r["ddt_bias"]), _ptr(r["d_initial"]), _ptr(workspace), workspace.numel(),
                         _ptr(cu_seqlens), B, T, H, K, V, N, ctypes.c_void_p(stream))
    if st != 0:
        raise KDAError(st, "kda_bwd")
    return r


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the workspace's device status code."""
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device).cuda_stream
    with torch.cuda.device(workspace.device):
        return int(load().kda_read_device_status(_ptr(workspace), ctypes.c_void_p(stream)))


def selftest_wait_timeout(workspace: torch.Tensor, limit_us: int = 2000, stream=None) -> None:
    """Enqueues the device time-out self-test: a bounded wait on a barrier nothing completes,
    which records KDA_ERR_DEVICE_TIMEOUT in the workspace status word after ``limit_us``."""
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device).cuda_stream
    with torch.cuda.device(workspace.device):
        st = int(load().kda_selftest_wait_timeout(_ptr(workspace), int(limit_us), ctypes.c_void_p(stream)))
    if st != 0:
        raise KDAError(st, "kda_selftest_wait_timeout")


def chunk_kda(q, k, v, g, beta, scale=None, initial_state=None, output_final_state=False,
              A_log=None, dt_bias=None, lower_bound=-5.0, cu_seqlens=None,
              transpose_state_layout=False, recurrent=False, use_gate_in_kernel=True,
              use_qk_l2norm_in_kernel=True, use_beta_sigmoid_in_kernel=True,
              safe_gate=True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """fla-style call (flags as in the chunk_kda usage example).

    ``use_gate_in_kernel=False``: ``g`` is fp32 log alpha (the safe gate already applied);
    ``use_qk_l2norm_in_kernel=False``: q and k are used as given; ``use_beta_sigmoid_in_kernel=False``:
    ``beta`` is fp32 beta.  ``safe_gate`` must stay True (the chunked kernels rely on the lower bound).
    Returns ``(out, final_state)``; ``final_state`` is None unless ``output_final_state``.
    With ``transpose_state_layout`` the states are [N, H, V, K] (S transposed)."""
    if not safe_gate:
        raise ValueError("safe_gate=False is not supported: the chunked kernels need lower_bound")
    flags = ((0 if use_gate_in_kernel else FLAG_GATE_PRECOMPUTED)
             | (0 if use_qk_l2norm_in_kernel else FLAG_NO_QK_L2NORM)
             | (0 if use_beta_sigmoid_in_kernel else FLAG_BETA_PRECOMPUTED))
    if recurrent and flags:
        raise ValueError("the token-serial kernel runs the in-kernel transforms only")
    B, T, H, K = q.shape
    V = v.shape[-1]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    if scale is None:
        scale = K ** -0.5
    if A_log is None and use_gate_in_kernel:
        A_log = torch.zeros(H, dtype=torch.float32, device=q.device)
    if dt_bias is None and use_gate_in_kernel:
        dt_bias = torch.zeros(H, K, dtype=torch.float32, device=q.device)
    out = torch.empty_like(v)
    final = None
    if output_final_state:
        shape = (N, H, V, K) if transpose_state_layout else (N, H, K, V)
        final = torch.empty(shape, dtype=torch.float32, device=q.device)
    ws = new_workspace(B * T, H, N, q.device, K, V)
    if recurrent:
        fwd_recurrent(q, k, v, g, beta, scale, out, ws, A_log, dt_bias, lower_bound, initial_state, final,
                      cu_seqlens, state_transposed=transpose_state_layout)
    else:
        fwd(q, k, v, g, beta, scale, out, ws, A_log, dt_bias, lower_bound, initial_state, final,
            cu_seqlens, state_transposed=transpose_state_layout, flags=flags)
    return out, final
