"""The workloads built from the pages' printed parameters match those parameters (CPU)."""
import os

import torch

import kda_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (x.strip() for x in line.split("=", 1))
                out[k] = v
    return out


def test_near_collinear_workload_matches_printed_parameters():
    p = _read("near_collinear_case.txt")
    x = kda_inputs.make_workload("collinear")
    T, H, D = int(p["T"]), int(p["H"]), int(p["D"])
    assert tuple(x.q.shape) == (1, T, H, D) and x.q.dtype == torch.bfloat16
    assert torch.equal(x.q, x.k) and torch.equal(x.q, x.q[:, :1].expand_as(x.q))
    blk = int(p["value_block_tokens"])
    assert torch.equal(x.v, x.v[:, :blk].repeat(1, T // blk, 1, 1))
    assert torch.all(x.g.float() == float(p["raw_gate"]))
    assert torch.all(x.beta.float() == float(p["raw_beta"]))
    assert x.lower_bound == float(p["lower_bound"])
    assert torch.all(x.A_log == float(p["A_log"])) and torch.all(x.dt_bias == float(p["dt_bias"]))
    assert torch.all(x.initial_state == float(p["initial_state"]))
    assert x.scale == D ** -0.5
    assert x.cu_seqlens.tolist() == [int(c) for c in p["cu_seqlens"].split(",")]


def test_usage_example_workload_matches_printed_parameters():
    p = _read("usage_example_case.txt")
    x = kda_inputs.make_workload("usage")
    assert tuple(x.q.shape) == (int(p["B"]), int(p["T"]), int(p["H"]), int(p["K"]))
    assert tuple(x.v.shape) == (int(p["B"]), int(p["T"]), int(p["H"]), int(p["V"]))
    assert x.cu_seqlens is None and x.initial_state is None and not x.output_final_state
    assert x.scale == float(p["scale"]) and x.lower_bound == float(p["lower_bound"])
    assert torch.all(x.A_log == float(p["A_log"])) and torch.all(x.dt_bias == float(p["dt_bias"]))
