"""CPU fp64 oracle for the KDA forward pass — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The CUDA library never does, and the two share no code: this package holds the
plain C token recurrence (``kda_oracle.c``), its ctypes wrapper, and two numpy companions used to
pin it (``brute`` — explicit products — and ``chunked`` — the chunked WY/UT form).

Parity status: every function here is pinned by the ``-m "not gpu"`` tests against closed forms,
invariants and brute force (see ``tests/test_oracle_pins.py``); the backward (``kda_bwd``) against
central finite differences of ``kda_fwd_f64`` and a closed form (``tests/test_oracle_bwd_pins.py``).  Agreement with upstream FlashKDA
or fla outputs is unpinned: neither their code nor any of their outputs is available, so the
state layout, the L2-norm epsilon and the gate form are readings (they are listed in the
design notes).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_fp = ctypes.POINTER(ctypes.c_float)
_i32p = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.kda_oracle_fwd.restype = ctypes.c_int
        lib.kda_oracle_fwd.argtypes = [_u16p, _u16p, _u16p, _u16p, _u16p, ctypes.c_double, _fp, _fp,
                                       ctypes.c_double, _dp, _dp, _dp, _i32p, ctypes.c_int32,
                                       ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        lib.kda_oracle_prologue.restype = None
        lib.kda_oracle_prologue.argtypes = [_u16p, _u16p, _u16p, _u16p, _fp, _fp, ctypes.c_double,
                                            ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _dp, _dp,
                                            _dp, _dp]
        lib.kda_oracle_fwd_f64.restype = ctypes.c_int
        lib.kda_oracle_fwd_f64.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_double, _dp, _dp, ctypes.c_double,
                                           _dp, _dp, _dp, _i32p, ctypes.c_int32, ctypes.c_int64,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        lib.kda_oracle_bwd.restype = ctypes.c_int
        lib.kda_oracle_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_double, _dp, _dp, ctypes.c_double,
                                       _dp, _dp, _dp, _i32p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int32, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                       ctypes.c_int32]
        lib.kda_oracle_core.restype = ctypes.c_int
        lib.kda_oracle_core.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_double, _dp, _dp, _dp,
                                        _i32p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int32]
        _lib = lib
    return _lib


def _bf16_bits(t) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor (torch bf16 or an already-uint16 numpy array)."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float32)
    return np.ascontiguousarray(t.detach().cpu().to(torch.float32).numpy())


def _f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float64)
    return np.ascontiguousarray(t.detach().cpu().to(torch.float64).numpy())


def _ptr(a: Optional[np.ndarray], typ):
    if a is None:
        return ctypes.cast(None, typ)
    return a.ctypes.data_as(typ)


def _cu_and_shape(q_shape, cu_seqlens):
    B, T, H, _ = q_shape
    if cu_seqlens is None:
        cu = (np.arange(B + 1, dtype=np.int64) * T).astype(np.int32)
    else:
        if B != 1:
            raise ValueError("cu_seqlens requires batch size 1")
        cu = np.ascontiguousarray(np.asarray(cu_seqlens.cpu() if torch.is_tensor(cu_seqlens)
                                             else cu_seqlens, dtype=np.int32))
    return cu, B * T, H


def kda_fwd(q, k, v, g, beta, scale: float, A_log, dt_bias, lower_bound: float,
            initial_state=None, cu_seqlens=None, output_final_state: bool = True,
            state_transposed: bool = False, num_threads: int = 0
            ) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """The KDA forward from the raw inputs, in fp64.

    Token tensors are [B, T, H, D] bf16 (B = 1 with ``cu_seqlens``), beta is [B, T, H] bf16,
    A_log [H] and dt_bias [H, K] fp32, initial_state [N, H, K, V] (or [N, H, V, K] when
    ``state_transposed``).  Returns ``(o, final_state)`` as fp64 arrays shaped like ``v`` and
    like the state (``final_state`` is None unless requested).
    """
    lib = _load()
    cu, total, H = _cu_and_shape(tuple(q.shape), cu_seqlens)
    N = cu.size - 1
    dk, dv = q.shape[-1], v.shape[-1]
    qb, kb, vb, gb, bb = (_bf16_bits(x) for x in (q, k, v, g, beta))
    al, db = _f32(A_log), _f32(dt_bias)
    s0 = None if initial_state is None else _f64(initial_state)
    out = np.empty((total, H, dv), dtype=np.float64)
    sf = np.empty((N, H, dv, dk) if state_transposed else (N, H, dk, dv), dtype=np.float64) \
        if output_final_state else None
    rc = lib.kda_oracle_fwd(_ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(vb, _u16p), _ptr(gb, _u16p),
                            _ptr(bb, _u16p), float(scale), _ptr(al, _fp), _ptr(db, _fp),
                            float(lower_bound), _ptr(s0, _dp), _ptr(sf, _dp), _ptr(out, _dp),
                            _ptr(cu, _i32p), int(N), int(total), int(H), int(dk), int(dv),
                            int(bool(state_transposed)), int(num_threads))
    if rc != 0:
        raise ValueError("oracle rejected the sizes or cu_seqlens")
    return out.reshape(tuple(v.shape)), sf


def prologue(q, k, g, beta, A_log, dt_bias, lower_bound: float):
    """qhat, khat, log_alpha ([..., D] fp64) and beta ([...] fp64) for every token and head."""
    lib = _load()
    shape = tuple(q.shape)
    total = int(np.prod(shape[:-2]))
    H, dk = shape[-2], shape[-1]
    qb, kb, gb, bb = (_bf16_bits(x) for x in (q, k, g, beta))
    al, db = _f32(A_log), _f32(dt_bias)
    qh = np.empty((total, H, dk)); kh = np.empty((total, H, dk)); la = np.empty((total, H, dk))
    be = np.empty((total, H))
    lib.kda_oracle_prologue(_ptr(qb, _u16p), _ptr(kb, _u16p), _ptr(gb, _u16p), _ptr(bb, _u16p),
                            _ptr(al, _fp), _ptr(db, _fp), float(lower_bound), int(total), int(H),
                            int(dk), _ptr(qh, _dp), _ptr(kh, _dp), _ptr(la, _dp), _ptr(be, _dp))
    return (qh.reshape(shape), kh.reshape(shape), la.reshape(shape), be.reshape(shape[:-1]))


def core(qhat, khat, v, log_alpha, beta, scale: float, S0=None, cu_seqlens=None):
    """The recurrence alone on transformed fp64 inputs shaped [T, H, D] (packed) with
    ``cu_seqlens`` (default: one sequence).  State is [N, H, K, V].  Returns (o, S_final)."""
    lib = _load()
    qhat, khat, v, log_alpha, beta = (np.ascontiguousarray(x, dtype=np.float64)
                                      for x in (qhat, khat, v, log_alpha, beta))
    total, H, dk = qhat.shape
    dv = v.shape[-1]
    cu = np.asarray([0, total] if cu_seqlens is None else cu_seqlens, dtype=np.int32)
    N = cu.size - 1
    s0 = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
    out = np.empty((total, H, dv))
    sf = np.empty((N, H, dk, dv))
    rc = lib.kda_oracle_core(_ptr(qhat, _dp), _ptr(khat, _dp), _ptr(v, _dp), _ptr(log_alpha, _dp),
                             _ptr(beta, _dp), float(scale), _ptr(s0, _dp), _ptr(sf, _dp),
                             _ptr(out, _dp), _ptr(cu, _i32p), int(N), int(total), int(H), int(dk),
                             int(dv))
    if rc != 0:
        raise ValueError("oracle rejected the sizes or cu_seqlens")
    return out, sf


def fwd_inputs(x, num_threads: int = 0, state_transposed: bool = False):
    """Run the oracle on a ``kda_inputs.KDAInputs`` problem."""
    s0 = x.initial_state
    if s0 is not None and state_transposed:
        s0 = s0.transpose(-1, -2).contiguous()
    return kda_fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound,
                   initial_state=s0, cu_seqlens=x.cu_seqlens,
                   output_final_state=x.output_final_state, state_transposed=state_transposed,
                   num_threads=num_threads)


def kda_fwd_f64(q, k, v, g, beta, scale: float, A_log, dt_bias, lower_bound: float, initial_state=None,
                cu_seqlens=None):
    """The forward from fp64 raw inputs (no bf16 widening), states [N, H, K, V]: the function whose
    finite differences pin ``kda_bwd``.  Returns (o, final_state)."""
    lib = _load()
    cu, total, H = _cu_and_shape(tuple(q.shape), cu_seqlens)
    N = cu.size - 1
    dk, dv = q.shape[-1], v.shape[-1]
    qd, kd, vd, gd, bd, al, db = (_f64(x) for x in (q, k, v, g, beta, A_log, dt_bias))
    s0 = None if initial_state is None else _f64(initial_state)
    out = np.empty((total, H, dv))
    sf = np.empty((N, H, dk, dv))
    rc = lib.kda_oracle_fwd_f64(_ptr(qd, _dp), _ptr(kd, _dp), _ptr(vd, _dp), _ptr(gd, _dp), _ptr(bd, _dp),
                                float(scale), _ptr(al, _dp), _ptr(db, _dp), float(lower_bound), _ptr(s0, _dp),
                                _ptr(sf, _dp), _ptr(out, _dp), _ptr(cu, _i32p), int(N), int(total), int(H),
                                int(dk), int(dv))
    if rc != 0:
        raise ValueError("oracle rejected the sizes or cu_seqlens")
    return out.reshape(tuple(v.shape)), sf


def kda_bwd(q, k, v, g, beta, scale: float, A_log, dt_bias, lower_bound: float, d_out, initial_state=None,
            d_final=None, cu_seqlens=None, num_threads: int = 0):
    """Gradients of sum(d_out * o) + sum(d_final * S_final) w.r.t. the raw inputs, in fp64 (inputs
    are taken as fp64 values; bf16 tensors are widened exactly).  Returns a dict with dq, dk, dv, dg
    (shaped like q), dbeta (like beta), dA_log [H], ddt_bias [H, K] and d_initial [N, H, K, V]."""
    lib = _load()
    cu, total, H = _cu_and_shape(tuple(q.shape), cu_seqlens)
    N = cu.size - 1
    dk, dv = q.shape[-1], v.shape[-1]
    qd, kd, vd, gd, bd, al, db = (_f64(x) for x in (q, k, v, g, beta, A_log, dt_bias))
    s0 = None if initial_state is None else _f64(initial_state)
    do = _f64(d_out)
    dF = None if d_final is None else _f64(d_final)
    r = {n: np.empty((total, H, dk)) for n in ("dq", "dk", "dg")}
    r["dv"] = np.empty((total, H, dv))
    r["dbeta"] = np.empty((total, H))
    r["dA_log"] = np.empty(H)
    r["ddt_bias"] = np.empty((H, dk))
    r["d_initial"] = np.empty((N, H, dk, dv))
    rc = lib.kda_oracle_bwd(_ptr(qd, _dp), _ptr(kd, _dp), _ptr(vd, _dp), _ptr(gd, _dp), _ptr(bd, _dp),
                            float(scale), _ptr(al, _dp), _ptr(db, _dp), float(lower_bound), _ptr(s0, _dp),
                            _ptr(do, _dp), _ptr(dF, _dp), _ptr(cu, _i32p), int(N), int(total), int(H), int(dk),
                            int(dv), _ptr(r["dq"], _dp), _ptr(r["dk"], _dp), _ptr(r["dv"], _dp), _ptr(r["dg"], _dp),
                            _ptr(r["dbeta"], _dp), _ptr(r["dA_log"], _dp), _ptr(r["ddt_bias"], _dp),
                            _ptr(r["d_initial"], _dp), int(num_threads))
    if rc != 0:
        raise ValueError("oracle rejected the sizes or cu_seqlens")
    shp = tuple(q.shape)
    for n in ("dq", "dk", "dg"):
        r[n] = r[n].reshape(shp)
    r["dv"] = r["dv"].reshape(tuple(v.shape))
    r["dbeta"] = r["dbeta"].reshape(shp[:-1])
    return r
