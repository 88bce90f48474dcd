"""Sequence-parallel prefill (KCP, the KDA context parallelism named in torchtitan PR #4374).

A batch of sequences is cut along time into one contiguous segment per rank of a process group:
rank r holds tokens [t_r, t_{r+1}) of every sequence, as a [B, T_r, H, K] batch.  The forward pass
is affine in the state a segment starts from (S_out = M S_in + B, see ``kda_segment_map`` in
include/kda.h), so the ranks need one exchange:

  1. every rank computes its segment's maps (M, B) for every (sequence, head) unit (one intra-chunk
     pass and one recurrence launch of 2 N H CTAs on its GPU);
  2. one all-gather of the maps over the group (NCCL over NVLink between GPUs);
  3. rank r folds the maps of segments 0 .. r-1 over the sequences' initial states
     (``kda_state_affine``) and runs the ordinary chunked forward on its segment from that state;
     the final states of the whole sequences are the fold of the remaining maps over its segment's
     final state, so every rank returns them without a second collective.

Every step of the computation runs in the library's kernels; this module only orders the calls
and the collective.  The kernels are reached through an ``ops`` object (``DeviceOps`` by default)
so that the host logic can also be exercised with stand-ins on CPU process groups.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import FLAG_GATE_PRECOMPUTED, fwd, new_workspace, segment_map, state_affine

__all__ = ["DeviceOps", "ProcessGroupComm", "kcp_forward"]


class ProcessGroupComm:
    """The exchange over a torch.distributed process group (NCCL between GPUs); a group of one
    rank, or no initialised group at all, needs no collective."""

    def __init__(self, group=None):
        self.group = group
        if dist.is_available() and dist.is_initialized():
            self.rank = dist.get_rank(group)
            self.world = dist.get_world_size(group)
        else:
            self.rank, self.world = 0, 1

    def all_gather(self, t):
        if self.world == 1:
            return [t]
        out = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(out, t, group=self.group)
        return out


class DeviceOps:
    """The library's CUDA kernels, on the device of the inputs."""

    def segment_map(self, q, k, v, g, beta, A_log, dt_bias, lower_bound, flags):
        B, T, H, K = q.shape
        V = v.shape[-1]
        M = torch.empty(B, H, K, K, dtype=torch.float32, device=q.device)
        Bm = torch.empty(B, H, K, V, dtype=torch.float32, device=q.device)
        ws = new_workspace(B * T, H, B, q.device)
        segment_map(q, k, v, g, beta, ws, A_log, dt_bias, lower_bound, M, Bm, flags=flags)
        return M, Bm

    def fold(self, M, Bm, S, state_transposed):
        out = torch.empty_like(Bm)
        state_affine(M, Bm, S, out, state_transposed=state_transposed)
        return out

    def forward(self, q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, S_in, flags, state_transposed):
        B, T, H, K = q.shape
        V = v.shape[-1]
        out = torch.empty_like(v)
        shape = (B, H, V, K) if state_transposed else (B, H, K, V)
        final = torch.empty(shape, dtype=torch.float32, device=q.device)
        ws = new_workspace(B * T, H, B, q.device)
        fwd(q, k, v, g, beta, scale, out, ws, A_log, dt_bias, lower_bound, S_in, final,
            state_transposed=state_transposed, flags=flags)
        return out, final


def kcp_forward(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state=None, group=None,
                output_final_state=True, state_transposed=False, flags=0,
                ops=None, comm=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The forward pass of sequences split along time over the ranks of ``group``.

    Arguments are kda.fwd's for this rank's segment (batch mode, [B, T_r, H, K]); ``initial_state``
    is the sequences' initial state ([B, H, K, V], or [B, H, V, K] with ``state_transposed``), the
    same on every rank, None for zero.  Returns this rank's output segment and, with
    ``output_final_state``, the final states of the whole sequences (the same on every rank).
    Every rank must call it with the same B, H and flags; segment lengths may differ but must be at
    least one token."""
    if q.shape[1] == 0:
        raise ValueError("kcp_forward: every rank's segment must hold at least one token")
    ops = DeviceOps() if ops is None else ops
    comm = ProcessGroupComm(group) if comm is None else comm
    rank, world = comm.rank, comm.world
    if flags & FLAG_GATE_PRECOMPUTED:
        A_log = dt_bias = None

    # 1. this segment's maps, packed for one collective: [2, B, H, K, K] (K = V)
    M, Bm = ops.segment_map(q, k, v, g, beta, A_log, dt_bias, lower_bound, flags)
    maps = torch.stack([M, Bm]).contiguous()
    # 2. all-gather over the group
    gathered = comm.all_gather(maps)
    # 3. the state this segment starts from: fold of the earlier segments' maps
    S = initial_state
    for j in range(rank):
        S = ops.fold(gathered[j][0], gathered[j][1], S, state_transposed)
    out, S_end = ops.forward(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, S, flags, state_transposed)
    final = None
    if output_final_state:
        final = S_end
        for j in range(rank + 1, world):
            final = ops.fold(gathered[j][0], gathered[j][1], final, state_transposed)
    return out, final
