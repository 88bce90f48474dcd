"""bench.py's roofline arithmetic, checked on CPU against quantities derived independently: the
byte counts from the tensors the operator reads and writes (shapes and dtypes), the FLOP count
from the GEMM shapes of the chunked form, and the peaks from the measured-peaks file."""
import json
import os

import pytest
import torch

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bytes(shape, dtype):
    return torch.empty(shape, dtype=dtype, device="meta").numel() * torch.empty((), dtype=dtype).element_size()


@pytest.mark.parametrize("T,H,N", [(32768, 96, 1), (400, 12, 2), (64, 1, 1)])
def test_algorithmic_bytes_are_the_operator_tensors(T, H, N):
    """Inputs read once (q, k, v, g bf16 [1, T, H, 128]; raw beta bf16 [1, T, H]), the output
    written once (bf16 [1, T, H, 128]) and the fp32 final state [N, H, 128, 128]; the initial state
    is NULL (zero) in the bench workload, so it is not read."""
    D = 128
    want = (4 * _bytes((1, T, H, D), torch.bfloat16) + _bytes((1, T, H), torch.bfloat16)
            + _bytes((1, T, H, D), torch.bfloat16) + _bytes((N, H, D, D), torch.float32))
    assert bench.algorithmic_bytes(T, H, N) == want


def test_prefill_bytes_and_intensity():
    alg = bench.algorithmic_bytes(32768, 96, 1)
    assert alg == 4_039_114_752
    # arithmetic intensity of the chunked form below the B200 ridge: the HBM roofline binds
    flops = bench.FLOPS_PER_TOKEN_HEAD * 32768 * 96
    assert flops / alg < 2.25e15 / 7.7e12


def test_flops_per_token_head_from_gemm_shapes():
    """Per chunk of C tokens and one head: the recurrence's W S, Qtil S (C x K . K x V) and
    Ktil^T Delta (K x C . C x V), P Delta (C x C . C x V); the intra-chunk K K^T, Q K^T
    (C x K . K x C), T K (C x C . C x K) and T V (C x C . C x V); the triangular solve C^3 / 3."""
    C, K, V = bench.CHUNK, bench.D, bench.D
    gemm = lambda m, n, k: 2 * m * n * k
    per_chunk = (gemm(C, V, K) + gemm(C, V, K) + gemm(K, V, C) + gemm(C, V, C)
                 + gemm(C, C, K) + gemm(C, C, K) + gemm(C, K, C) + gemm(C, V, C) + C ** 3 // 3)
    assert bench.FLOPS_PER_TOKEN_HEAD == per_chunk // C == 181_589


def test_peaks_come_from_the_measured_file():
    hbm, tf, kind = bench.load_peaks()
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        assert (hbm, tf, kind) == (6650.0, 1590.0, "fallback")
        return
    with open(p) as f:
        d = json.load(f)
    assert kind == "measured" and hbm == d["hbm_gbs"] and tf == d["bf16_tflops"]
    assert 4000 < hbm < 8000 and 1000 < tf < 2300


def test_traffic_summary_is_consistent():
    """The committed DRAM traffic of one call (measured at 32 heads) is the sum of its launches'
    reads and writes, at least the operator's own bytes at 32 heads (the items' round trip comes on
    top), and scales to 96 heads by the head ratio."""
    with open(os.path.join(ROOT, "profiles", "kda_fwd_prefill_h32_traffic.json")) as f:
        d = json.load(f)
    total = sum(v["read"] + v["write"] for v in d["per_kernel_measured"].values())
    assert abs(total - d["dram_bytes_per_call_measured"]) <= 1e-3 * d["dram_bytes_per_call_measured"]
    assert d["dram_bytes_per_call_measured"] >= bench.algorithmic_bytes(32768, d["measured_heads"], 1)
    assert d["scale_to_96_heads"] == 96 / d["measured_heads"]
    assert abs(d["dram_bytes_per_call"] - d["scale_to_96_heads"] * d["dram_bytes_per_call_measured"]) <= 1e6
