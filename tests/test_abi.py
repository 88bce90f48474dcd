"""The C-ABI library loads, exports every declared entry point, and rejects bad arguments on the
host before touching a GPU (CPU only: no call here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

import kimi_delta_attention_24_b200 as kda
from kimi_delta_attention_24_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "kda_fwd" in names and "kda_workspace_size" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings(lib):
    for code, name in [(0, b"KDA_OK"), (1, b"KDA_ERR_INVALID_ARGUMENT"), (2, b"KDA_ERR_UNSUPPORTED"),
                       (3, b"KDA_ERR_WORKSPACE_TOO_SMALL"), (4, b"KDA_ERR_CUDA"),
                       (5, b"KDA_ERR_DEVICE_TIMEOUT")]:
        assert lib.kda_status_string(code) == name


def test_support_predicate(lib):
    assert lib.kda_is_supported(128, 1, -5.0) == 1
    assert lib.kda_is_supported(128, 1, 0.0) == 1
    assert lib.kda_is_supported(128, 1, -5.5) == 0
    assert lib.kda_is_supported(128, 1, 0.5) == 0
    assert lib.kda_is_supported(64, 1, -5.0) == 0
    assert lib.kda_is_supported(128, 0, -5.0) == 0


def test_workspace_size_covers_every_chunk_and_head(lib):
    # one 81 KB item per (chunk, head): 512 chunks x 96 heads at T = 32768, plus one fp32
    # 128 x 128 hand-over state per head for the sequence cut between two stages
    item = 82944
    a = lib.kda_workspace_size(32768, 96, 1)
    assert a >= 512 * 96 * item + 96 * 128 * 128 * 4 and a % 256 == 0
    assert lib.kda_workspace_size(1, 96, 1) >= 96 * item
    # 8 sequences of 100 tokens or fewer hold at most (100 + 63 * 8) / 64 chunks in total
    assert lib.kda_workspace_size(100, 32, 8) >= (100 + 63 * 8) // 64 * 32 * item
    assert lib.kda_workspace_size(0, 32, 0) >= 256


# Fake device pointers: aligned, never dereferenced because validation fails first.
P = 0x10000000


def call(lib, name="kda_fwd", **kw):
    a = dict(q=P, k=P, v=P, g=P, beta=P, scale=0.088, out=P, ws=P, ws_bytes=1 << 20, A_log=P,
             dt_bias=P, lb=-5.0, s0=None, sT=None, cu=None, batch=1, seqlen=64, H=1, K=128, V=128,
             N=1, transposed=0)
    a.update(kw)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return getattr(lib, name)(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["g"]), vp(a["beta"]), a["scale"],
                              vp(a["out"]), vp(a["ws"]), a["ws_bytes"], vp(a["A_log"]), vp(a["dt_bias"]),
                              a["lb"], vp(a["s0"]), vp(a["sT"]), vp(a["cu"]), a["batch"], a["seqlen"],
                              a["H"], a["K"], a["V"], a["N"], a["transposed"], None)



@pytest.mark.parametrize("T,H,N", [(4096, 96, 1), (350, 2, 3), (1, 1, 1), (100000, 8, 40)])
def test_bwd_workspace_size_is_its_documented_parts(lib, T, H, N):
    """kda_bwd_workspace_size as kda.h describes it: the forward's workspace, the checkpoints and the
    recomputed output, the chunk table, per (chunk, head) the chunk's factors (336.5 KB) and dDelta
    (32 KB), one 128 x 128 fp32 state gradient per chunk slot and head, the per-token partials
    (3 x 128 + 1 fp32), and the larger of 296 CTAs' scratch (369.75 KB each) and one 64 x 128 fp32
    buffer per (sequence, head); every region 256-byte aligned."""
    a256 = lambda b: (b + 255) // 256 * 256
    chunks, slots = T // 64 + N, T // 64 + N + 1
    parts = [lib.kda_workspace_size(T, H, N), lib.kda_checkpoint_size(T, H, N), T * H * 128 * 2, (N + 1) * 4,
             chunks * H * 344576, slots * H * 128 * 128 * 4, chunks * H * 64 * 128 * 4, (3 * 128 + 1) * 4 * T * H,
             max(296 * 378624, N * H * 64 * 128 * 4)]
    assert lib.kda_bwd_workspace_size(T, H, N) == sum(a256(p) for p in parts)

@pytest.mark.parametrize("name", ["kda_fwd", "kda_fwd_recurrent"])
def test_host_validation(lib, name):
    assert call(lib, name, K=64) == 2
    assert call(lib, name, V=64) == 2
    assert call(lib, name, lb=-5.01) == 2
    assert call(lib, name, lb=0.1) == 2
    assert call(lib, name, lb=float("nan")) == 2
    assert call(lib, name, q=None) == 1
    assert call(lib, name, out=P + 8) == 1          # misaligned
    assert call(lib, name, H=0) == 1
    assert call(lib, name, seqlen=-1) == 1
    assert call(lib, name, transposed=2) == 1
    assert call(lib, name, cu=P, batch=2) == 1      # varlen needs batch 1
    assert call(lib, name, N=3) == 1                # batch mode: N must equal batch
    assert call(lib, name, scale=float("inf")) == 1
    assert call(lib, name, s0=P + 4) == 1
    assert call(lib, name, beta=P + 1) == 1         # beta needs 2-byte alignment
    assert call(lib, name, batch=4, seqlen=1 << 30, N=4) == 1  # 2^32 tokens: int32 token coordinates


def test_workspace_checks(lib):
    assert call(lib, ws=None) == 1
    assert call(lib, ws=P + 16) == 1                # workspace must be 256-byte aligned
    assert call(lib, ws_bytes=16, H=4) == 3
    # empty problems launch nothing and succeed
    assert call(lib, batch=0, N=0) == 0
    assert call(lib, "kda_fwd_recurrent", batch=0, N=0) == 0


def test_read_status_rejects_null(lib):
    assert lib.kda_read_device_status(None, None) == 1


def test_python_binding_requires_built_library(tmp_path, monkeypatch):
    monkeypatch.setattr(kda, "_lib", None)
    monkeypatch.setattr(kda, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        kda.load()


def call_decode(lib, **kw):
    a = dict(q=P, k=P, v=P, g=P, beta=P, scale=0.088, out=P, A_log=P, dt_bias=P, lb=-5.0, s_in=P, s_out=P,
             idx=None, batch=4, seqlen=1, H=2, K=128, V=128, slots=4, transposed=0, flags=0, ws=None)
    a.update(kw)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    fn = lib.kda_decode
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int32] * 5 + \
        [ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["g"]), vp(a["beta"]), a["scale"], vp(a["out"]),
              vp(a["A_log"]), vp(a["dt_bias"]), a["lb"], vp(a["s_in"]), vp(a["s_out"]), vp(a["idx"]),
              a["batch"], a["seqlen"], a["H"], a["K"], a["V"], a["slots"], a["transposed"], a["flags"],
              vp(a["ws"]), None)


def test_decode_host_validation(lib):
    assert call_decode(lib, K=64) == 2
    assert call_decode(lib, lb=-6.0) == 2
    assert call_decode(lib, q=None) == 1
    assert call_decode(lib, A_log=None) == 1
    assert call_decode(lib, out=P + 8) == 1
    assert call_decode(lib, s_out=P + 4) == 1
    assert call_decode(lib, flags=8) == 1                      # unknown flag bit
    assert call_decode(lib, transposed=2) == 1
    assert call_decode(lib, slots=3) == 1                      # no indices: request b uses slot b
    assert call_decode(lib, ws=P + 16) == 1                    # workspace must be 256-byte aligned
    assert call_decode(lib, beta=P + 2, flags=4) == 1          # fp32 beta needs 4-byte alignment
    assert call_decode(lib, H=0) == 1
    # a precomputed gate needs neither A_log nor dt_bias, and lower_bound is not checked
    assert call_decode(lib, A_log=None, dt_bias=None, lb=-9.0, flags=1, batch=0) == 0
    assert call_decode(lib, batch=0) == 0     # no request: nothing launched
    assert call_decode(lib, q=None, batch=0, seqlen=0) == 0  # no token: token tensors may be null
    assert call_decode(lib, q=None, seqlen=1) == 1


def test_fwd_ex_flags_validation(lib):
    fn = lib.kda_fwd_ex
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def ex(flags, A_log=P, dt_bias=P, beta=P, lb=-5.0, batch=1):
        return fn(vp(P), vp(P), vp(P), vp(P), vp(beta), ctypes.c_float(0.088), vp(P), vp(P),
                  ctypes.c_size_t(1 << 20), vp(A_log), vp(dt_bias), ctypes.c_float(lb), None, None, None,
                  ctypes.c_int32(batch), ctypes.c_int64(64), ctypes.c_int32(1), ctypes.c_int32(128),
                  ctypes.c_int32(128), ctypes.c_int32(batch), ctypes.c_int32(0), ctypes.c_uint32(flags), None)

    assert ex(8) == 1                                    # unknown flag bit
    assert ex(0, A_log=None) == 1                        # the in-kernel gate needs A_log
    assert ex(1, A_log=None, dt_bias=None, batch=0) == 0  # a precomputed gate does not
    assert ex(4, beta=P + 2) == 1                        # fp32 beta needs 4-byte alignment
    assert ex(1, lb=-6.0) == 2                           # the clamp range must still be supported


def test_kcp_entry_points_validation(lib):
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    sm = lib.kda_segment_map
    sm.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                           ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_uint32, ctypes.c_void_p]
    sm.restype = ctypes.c_int

    def seg(M=P, Bm=P, ws=P, ws_bytes=1 << 20, K=128, batch=1):
        return sm(vp(P), vp(P), vp(P), vp(P), vp(P), vp(ws), ws_bytes, vp(P), vp(P), -5.0, vp(M), vp(Bm), None,
                  batch, 64, 1, K, 128, batch, 0, None)

    assert seg(M=None) == 1
    assert seg(Bm=P + 8) == 1
    assert seg(ws=None) == 1
    assert seg(ws_bytes=16) == 3
    assert seg(K=64) == 2
    assert seg(batch=0) == 0
    af = lib.kda_state_affine
    af.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
    af.restype = ctypes.c_int
    assert af(vp(P), vp(P), vp(P), vp(P), 4, 64, 0, None) == 2
    assert af(None, vp(P), vp(P), vp(P), 4, 128, 0, None) == 1   # a state input needs M
    assert af(vp(P), None, vp(P), vp(P), 4, 128, 0, None) == 1
    assert af(vp(P), vp(P), vp(P + 4), vp(P), 4, 128, 0, None) == 1
    assert af(vp(P), vp(P), vp(P), vp(P), 4, 128, 2, None) == 1
    assert af(vp(P), vp(P), vp(P), vp(P), 0, 128, 0, None) == 0


def test_fwd_ex_head_sizes(lib):
    fn = lib.kda_fwd_ex
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def ex(K, V, ws_bytes=1 << 40):
        return fn(vp(P), vp(P), vp(P), vp(P), vp(P), ctypes.c_float(0.088), vp(P), vp(P), ctypes.c_size_t(ws_bytes),
                  vp(P), vp(P), ctypes.c_float(-5.0), None, None, None, ctypes.c_int32(0), ctypes.c_int64(64),
                  ctypes.c_int32(1), ctypes.c_int32(K), ctypes.c_int32(V), ctypes.c_int32(0), ctypes.c_int32(0),
                  ctypes.c_uint32(0), None)

    assert ex(60, 64) == 2      # not a multiple of 8
    assert ex(136, 128) == 2    # above 128
    assert ex(0, 64) == 2
    assert ex(64, 64) == 0      # empty batch: accepted, nothing launched
    assert ex(64, 64, ws_bytes=16) == 3
    # kda_fwd itself stays at 128 (FlashKDA's fwd)
    assert call(lib, K=64, V=64) == 2
    # padded sizes need room for the 128-wide copies; 128 needs exactly kda_workspace_size
    assert lib.kda_workspace_size_ex(32768, 96, 1, 128, 128) == lib.kda_workspace_size(32768, 96, 1)
    assert lib.kda_workspace_size_ex(4096, 8, 2, 64, 64) > lib.kda_workspace_size(4096, 8, 2) + 5 * 4096 * 8 * 256
