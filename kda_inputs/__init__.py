"""Seeded synthetic inputs for the KDA forward pass.

This module only draws random tensors with the shapes, dtypes and value distributions of the
workloads; it holds none of the method's arithmetic.  Both the CUDA library's tests and the
oracle consume what it produces.

Workloads (head dims K = V = 128, lower_bound = -5, scale = 128**-0.5, seed 0 unless noted):

  ``tiny``       one chunk: B=1, T=64, H=1; A_log = 0, dt_bias = 0, zero initial state.
  ``tail``       packed varlen cu_seqlens=[0,200,400], H=12 (multi-chunk with a partial tail);
                 A_log ~ U(-1,1), dt_bias ~ N(0, 0.5), initial state ~ N(0, 0.1).
  ``varlen``     8 documents with lengths ~ U{1..4096} drawn from the seed, H=32, packed.
  ``prefill``    B=1, T=32768, H=96 (the throughput workload), zero initial state.
  ``collinear``  B=1, T=16384, H=1: q = k = one N(0,1) vector at every token, v = one 16-token
                 N(0,1) block tiled, raw gate -12, raw beta 8, A_log = 0, dt_bias = 0.  This is the
                 near-collinear stress case of the vLLM PR #54859 report
                 (test_flashkda_near_collinear_keys_remain_finite).
  ``usage``      batch mode B=2, T=64, H=12, scale = 1.0, A_log = 0, dt_bias = 0, no states: the
                 shapes of the FlashKDA usage example ("What CUDA Version Is Required to Use
                 FlashKDA?", Usage Examples).

"N(0, s)" reads s as the standard deviation.  All draws come from one ``torch.Generator`` in
the order q, k, v, g, beta, A_log, dt_bias, initial_state, then are cast (bf16 for the token
tensors, fp32 for the parameters and the state).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

HEAD_DIM = 128
LOWER_BOUND = -5.0
DEFAULT_SCALE = HEAD_DIM ** -0.5

WORKLOADS = ("tiny", "tail", "varlen", "prefill", "collinear", "usage")


@dataclass
class KDAInputs:
    """One forward problem.  Token tensors are [B, T, H, D] (B = 1 when cu_seqlens is set)."""

    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor  # [B, T, H]
    A_log: torch.Tensor  # [H] fp32
    dt_bias: torch.Tensor  # [H, K] fp32
    lower_bound: float
    scale: float
    initial_state: Optional[torch.Tensor]  # [N, H, K, V] fp32 or None
    cu_seqlens: Optional[torch.Tensor]  # [N+1] int32 or None
    output_final_state: bool = True
    meta: dict = field(default_factory=dict)

    @property
    def num_heads(self) -> int:
        return self.q.shape[2]

    @property
    def num_seqs(self) -> int:
        if self.cu_seqlens is not None:
            return self.cu_seqlens.numel() - 1
        return self.q.shape[0]

    @property
    def total_tokens(self) -> int:
        return self.q.shape[0] * self.q.shape[1]

    def to(self, device) -> "KDAInputs":
        def mv(t):
            return None if t is None else t.to(device)

        return KDAInputs(self.name, mv(self.q), mv(self.k), mv(self.v), mv(self.g), mv(self.beta),
                         mv(self.A_log), mv(self.dt_bias), self.lower_bound, self.scale,
                         mv(self.initial_state), mv(self.cu_seqlens), self.output_final_state,
                         dict(self.meta))


def _randn(gen, shape, std=1.0, device="cpu"):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std


def _uniform(gen, shape, lo, hi, device="cpu"):
    return torch.rand(shape, generator=gen, device=device, dtype=torch.float32) * (hi - lo) + lo


def make_random(name: str, lengths, num_heads: int, *, seed: int = 0, device="cpu",
                varlen: bool = True, batch: int = 1, seqlen: int = 0,
                a_log_range=(-1.0, 1.0), dt_bias_std: float = 0.5,
                state_std: Optional[float] = None, lower_bound: float = LOWER_BOUND,
                scale: float = DEFAULT_SCALE, zero_gate_params: bool = False,
                output_final_state: bool = True) -> KDAInputs:
    """Gaussian token tensors for packed documents of the given lengths (or a [B, T] batch)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    if varlen:
        lengths = [int(x) for x in lengths]
        total = sum(lengths)
        shape_tok = (1, total, num_heads)
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
        n = len(lengths)
    else:
        shape_tok = (batch, seqlen, num_heads)
        cu = None
        n = batch
    D = HEAD_DIM
    q = _randn(gen, shape_tok + (D,), device=device).to(torch.bfloat16)
    k = _randn(gen, shape_tok + (D,), device=device).to(torch.bfloat16)
    v = _randn(gen, shape_tok + (D,), device=device).to(torch.bfloat16)
    g = _randn(gen, shape_tok + (D,), device=device).to(torch.bfloat16)
    beta = _randn(gen, shape_tok, device=device).to(torch.bfloat16)
    if zero_gate_params:
        A_log = torch.zeros(num_heads, dtype=torch.float32, device=device)
        dt_bias = torch.zeros(num_heads, D, dtype=torch.float32, device=device)
    else:
        A_log = _uniform(gen, (num_heads,), *a_log_range, device=device)
        dt_bias = _randn(gen, (num_heads, D), std=dt_bias_std, device=device)
    if state_std is None:
        s0 = torch.zeros(n, num_heads, D, D, dtype=torch.float32, device=device)
    else:
        s0 = _randn(gen, (n, num_heads, D, D), std=state_std, device=device)
    return KDAInputs(name, q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, s0,
                     None if cu is None else cu.to(device), output_final_state)


def varlen_lengths(num_docs: int, max_len: int, seed: int = 0):
    gen = torch.Generator()
    gen.manual_seed(seed)
    return torch.randint(1, max_len + 1, (num_docs,), generator=gen).tolist()


def make_collinear(T: int = 16384, *, seed: int = 0, device="cpu") -> KDAInputs:
    """q = k = one seeded vector repeated; v = one seeded 16-token block tiled T/16 times."""
    H, D = 1, HEAD_DIM
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    key = _randn(gen, (1, 1, H, D), device=device).to(torch.bfloat16)
    value_block = _randn(gen, (1, 16, H, D), device=device).to(torch.bfloat16)
    qk = key.expand(1, T, H, D).contiguous()
    v = value_block.repeat(1, T // 16, 1, 1)
    g = torch.full_like(qk, -12.0)
    beta = torch.full((1, T, H), 8.0, dtype=torch.bfloat16, device=device)
    A_log = torch.zeros(H, dtype=torch.float32, device=device)
    dt_bias = torch.zeros(H, D, dtype=torch.float32, device=device)
    s0 = torch.zeros(1, H, D, D, dtype=torch.float32, device=device)
    cu = torch.tensor([0, T], dtype=torch.int32, device=device)
    return KDAInputs("collinear", qk, qk.clone(), v, g, beta, A_log, dt_bias, LOWER_BOUND,
                     DEFAULT_SCALE, s0, cu, True)


def make_workload(name: str, *, seed: int = 0, device="cpu") -> KDAInputs:
    if name == "tiny":
        return make_random(name, [64], 1, seed=seed, device=device, zero_gate_params=True)
    if name == "tail":
        return make_random(name, [200, 200], 12, seed=seed, device=device, state_std=0.1)
    if name == "varlen":
        lens = varlen_lengths(8, 4096, seed)
        x = make_random(name, lens, 32, seed=seed, device=device)
        x.meta["lengths"] = lens
        return x
    if name == "prefill":
        return make_random(name, [32768], 96, seed=seed, device=device)
    if name == "collinear":
        return make_collinear(seed=seed, device=device)
    if name == "usage":
        x = make_random(name, None, 12, seed=seed, device=device, varlen=False, batch=2, seqlen=64,
                        scale=1.0, zero_gate_params=True, output_final_state=False)
        x.initial_state = None
        return x
    raise KeyError(name)
