"""Throughput of the KDA chunked forward on the 32K-token, 96-head prefill (B=1, T=32768, H=96,
K=V=128, bf16 in/out, fp32 state, lower_bound=-5).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one kda_fwd over the whole workload: the full hot path in five launches (chunk table,
then over two ranges of chunks the chunk-parallel intra-chunk kernel with the gate, norms, decays,
Gram products and solve, and the per-(sequence, head) recurrence kernel with the output and
final-state epilogues; the second intra-chunk launch overlaps the first recurrence).  Inputs are
seeded synthetic tensors resident in HBM; they are 4 GB, far larger than the 126 MB L2, so no
flush is needed between steps.  The roofline block treats the whole call as the kernel: the
pages' algorithmic bytes of the operation over its measured duration.  For N > 1
each rank runs an independent replica of the workload (the operator has no cross-GPU step):
weak scaling, value = all ranks' token-heads / max-over-ranks time.  Prints one JSON line on rank 0.

--impl reference times the CPU fp64 oracle on the host cores instead, on a bounded sample of the
same workload (it is the only reference implementation available).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "KDA fwd Mtok·head/s at H=96,T=32K; TFLOP/s as % of binding roofline"
UNIT = "Mtok·head/s"
T_TOK, HEADS, D = 32768, 96, 128
CHUNK = 64
BYTES_PER_TOKEN_HEAD = 4 * 2 * D + 2 + 2 * D          # q, k, v, g in; raw beta in; o out
FLOPS_PER_TOKEN_HEAD = 6 * D * D + 2 * CHUNK * D + 3 * 2 * CHUNK * D + 2 * CHUNK * D + CHUNK * CHUNK // 3
STATE_OUT_BYTES_PER_UNIT = D * D * 4                  # fp32 final state per (sequence, head); initial state is zero (NULL)
WORKLOAD = "prefill B=1 T=32768 H=96 K=V=128 bf16, lower_bound=-5, zero initial state, final state out"


def algorithmic_bytes(tokens, heads, seqs):
    return BYTES_PER_TOKEN_HEAD * tokens * heads + STATE_OUT_BYTES_PER_UNIT * seqs * heads


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every ~2 ms by a background thread
    during the timed region (nvidia-smi starts too slowly for a timed region of tens of ms)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device):
        self.device = device
        self.samples = []
        self.error = None

    def _handle(self, nvml):
        props = torch.cuda.get_device_properties(self.device)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return nvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def _run(self):
        nvml = self.nvml
        while not self.stop:
            try:
                sm = nvml.nvmlDeviceGetClockInfo(self.h, nvml.NVML_CLOCK_SM)
                rs = nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception as e:  # keep the bench running; report the failure
                self.error = str(e)
                return
            time.sleep(0.002)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = self._handle(pynvml)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.stop = False
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception as e:
            self.error = str(e)
            self.thread = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"no samples ({self.error})"]}
        sm = [x for x, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, b in self.REASONS.items() if r & b})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "source": "NVML, every ~2 ms during the timed region"}


def dist_setup(n_gpus):
    """One process per GPU from the launcher's environment; NCCL on GPUs, gloo without (tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(token_heads_per_rank, ms_per_step, world):
    """Whole-job Mtok·head/s: every rank runs its own replica of the workload (weak scaling), and
    the step time is the slowest rank's."""
    return world * token_heads_per_rank / (ms_per_step * 1e-3) / 1e6


DECODE_REQUESTS = 256


def bench_decode(dev, steps, warmup, seed=0):
    """The batched decode step on 256 requests x 96 heads, one token each, states updated in place
    in a 256-slot pool (3.2 GB, far larger than L2): microseconds per step and achieved HBM GB/s of
    its algorithmic bytes (state read + written, token inputs and output)."""
    import kda_inputs
    import kimi_delta_attention_24_b200 as kda

    B, H = DECODE_REQUESTS, HEADS
    x = kda_inputs.make_random("decode", None, H, seed=seed, varlen=False, batch=B, seqlen=1, device=dev)
    gen = torch.Generator(device=dev).manual_seed(seed + 7)
    pool = torch.randn(B, H, D, D, generator=gen, device=dev) * 0.1
    idx = torch.randperm(B, generator=gen, device=dev).to(torch.int32)
    out = torch.empty_like(x.v)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.decode(x.q, x.k, x.v, x.g, x.beta, x.scale, out, x.A_log, x.dt_bias, x.lower_bound, pool, pool, idx,
                   stream=stream.cuda_stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / steps
    units = B * H
    alg = units * (2 * D * D * 4 + BYTES_PER_TOKEN_HEAD)
    hbm_peak, _, peak_kind = load_peaks()
    gbs = alg / (us * 1e-6) / 1e9
    return {"workload": f"decode: {B} requests x {H} heads, 1 token each, fp32 states in place in a {B}-slot pool",
            "us_per_step": us, "requests_per_s": B / (us * 1e-6),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg,
                         "bytes_per_unit": 2 * D * D * 4 + BYTES_PER_TOKEN_HEAD},
            "gpu_launches": steps, "l2": "state pool (3.2 GB) exceeds L2; no flush"}


BWD_TOKENS = 4096
BWD_BYTES_PER_TOKEN_HEAD = BYTES_PER_TOKEN_HEAD + 2 * D + (4 * 2 * D + 2)  # + d_out in; dq, dk, dv, dg, dbeta out


# Chunked-form FLOPs of the backward per token-head (64-token chunks, K = V = 128; a multiply-add is 2
# FLOPs): per (chunk, head), the chunk factors in both chunk-parallel kernels (the Gram and P blocks of
# the four 16-row sub-blocks, the solve), the prep products (W, Qt - P W, P^T dO, (Qt - P W)^T dO), the
# reverse state walk (Kt dS', W^T E) and the gradient products (W, U, dP, dT_b twice, dv, dKg; Delta,
# dKt, dQs, dW; T^T dT, dA; the four decay-weighted products).
_CB = 64
_BWD_MACS_PER_CHUNK = (2 * (2 * 16 * 160 * D + _CB ** 3 // 6) + 3 * _CB * _CB * D + _CB * D * D
                       + 2 * _CB * D * D
                       + 7 * _CB * _CB * D + 4 * _CB * D * D + 2 * _CB ** 3 + 4 * 16 * 160 * D)
BWD_FLOPS_PER_TOKEN_HEAD = 2 * _BWD_MACS_PER_CHUNK / _CB


def bench_backward(dev, steps, warmup, seed=0, heads=HEADS):
    """The backward pass (chunked, from the checkpointing forward's states) on the
    prefill's heads with T = 4096 tokens: milliseconds per step, token-heads/s, TFLOP/s of its
    chunked-form FLOPs against the tf32 tensor peak (the binding roofline: about 193 FLOP per
    algorithmic byte, above the tf32 ridge) and HBM GB/s of its algorithmic bytes (inputs and d_out
    read once, the five token gradients written once)."""
    import kda_inputs
    import kimi_delta_attention_24_b200 as kda

    HEADS = heads  # noqa: N806 (the workload's head count)
    x = kda_inputs.make_random("bwd", [BWD_TOKENS], HEADS, seed=seed, device=dev)
    gen = torch.Generator(device=dev).manual_seed(seed + 11)
    d_out = torch.randn(x.v.shape, generator=gen, device=dev).to(torch.bfloat16)
    ws = torch.empty(kda.bwd_workspace_size(BWD_TOKENS, HEADS, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the training forward stores the chunk-start states the backward starts from
    ck = torch.empty(kda.checkpoint_size(BWD_TOKENS, HEADS, 1) // 4, dtype=torch.float32, device=dev)
    fws = kda.new_workspace(BWD_TOKENS, HEADS, 1, dev)
    out = torch.empty_like(x.v)
    kda.fwd_checkpointed(x.q, x.k, x.v, x.g, x.beta, x.scale, out, fws, x.A_log, x.dt_bias, x.lower_bound, ck,
                         cu_seqlens=x.cu_seqlens, stream=stream.cuda_stream)

    def timed(checkpoints):
        def step():
            kda.bwd(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, d_out,
                    cu_seqlens=x.cu_seqlens, workspace=ws, stream=stream.cuda_stream, checkpoints=checkpoints)
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms = timed(ck)
    ms_without = timed(None)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        kda.fwd_checkpointed(x.q, x.k, x.v, x.g, x.beta, x.scale, out, fws, x.A_log, x.dt_bias, x.lower_bound, ck,
                             cu_seqlens=x.cu_seqlens, stream=stream.cuda_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_fwd_ck = e0.elapsed_time(e1) / steps
    th = BWD_TOKENS * HEADS
    alg = BWD_BYTES_PER_TOKEN_HEAD * th
    flops = BWD_FLOPS_PER_TOKEN_HEAD * th
    hbm_peak, bf16_peak, peak_kind = load_peaks()
    # the products are tf32 contractions: the tf32 peak is the measured bf16 one times the nominal
    # dense tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s); at 192 FLOP per byte the backward sits above the
    # tf32 ridge, so the tensor roofline binds
    tf32_peak = bf16_peak * 1.1 / 2.25
    gbs = alg / (ms * 1e-3) / 1e9
    tflops = flops / (ms * 1e-3) / 1e12
    bound = "tensor" if flops / (tf32_peak * 1e12) >= alg / (hbm_peak * 1e9) else "hbm"
    roof = ({"bound": "tensor", "achieved": tflops, "peak": tf32_peak, "unit": "TFLOP/s", "frac": tflops / tf32_peak}
            if bound == "tensor" else
            {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak})
    roof.update({"peak_source": f"{peak_kind} (tf32: measured bf16 x 1.1 / 2.25)" if bound == "tensor" else peak_kind,
                 "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": alg,
                 "hbm_achieved_gbs": gbs, "hbm_frac": gbs / hbm_peak,
                 "note": "chunked form, products on the tensor cores (mma.sync tf32, each operand split hi + lo: "
                         "three products per product of the form); latency-bound on each chunk's chain of "
                         "steps"})
    return {"workload": f"backward: B=1 T={BWD_TOKENS} H={HEADS} K=V=128, gradients of every input, from the "
                        "chunk-start states the checkpointing forward stored",
            "ms_per_step": ms, "value": th / (ms * 1e-3) / 1e6, "unit": UNIT,
            "ms_per_step_without_checkpoints": ms_without,
            "checkpointing_forward_ms": ms_fwd_ck,
            "roofline": roof,
            "chunked_tflops": tflops,
            "gpu_launches": steps}


KCP_RANKS = 8


def bench_kcp_rank(dev, steps, warmup, seed=0):
    """The device work one rank of an 8-rank sequence-parallel prefill does on its 4096-token
    segment of the 32K x 96-head prefill (the rank in the middle: segment map, the fold of four
    earlier maps, the forward from the folded state, the fold of three later maps), timed on one GPU
    with the other ranks' maps stood in by this rank's own (the all-gather is not included: every GPU
    call here has one GPU)."""
    import kda_inputs
    import kimi_delta_attention_24_b200 as kda
    from kimi_delta_attention_24_b200.kcp import DeviceOps

    T = T_TOK // KCP_RANKS
    x = kda_inputs.make_random("kcp", None, HEADS, seed=seed, varlen=False, batch=1, seqlen=T, device=dev)
    ops = DeviceOps()
    r = KCP_RANKS // 2

    def step():
        M, Bm = ops.segment_map(x.q, x.k, x.v, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound, 0)
        S = None
        for _ in range(r):
            S = ops.fold(M, Bm, S, False)
        _, S_end = ops.forward(x.q, x.k, x.v, x.g, x.beta, x.scale, x.A_log, x.dt_bias, x.lower_bound, S, 0, False)
        for _ in range(KCP_RANKS - r - 1):
            S_end = ops.fold(M, Bm, S_end, False)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"workload": f"sequence-parallel prefill, device work of rank {r} of {KCP_RANKS}: a {T}-token segment "
                        f"of the B=1 T={T_TOK} H={HEADS} prefill (segment map, {KCP_RANKS - 1} folds, forward); "
                        "the all-gather of the maps is not included",
            "ms_per_step": ms, "segment_token_heads_per_s_M": T * HEADS / (ms * 1e-3) / 1e6,
            "note": "one GPU only: measures a rank's device work, not a multi-GPU run"}


def cpu_oracle_sample(target_s=15.0):
    """Times the fp64 oracle on a bounded sample of the prefill: the first m heads over the
    first L tokens, sized from a short calibration to take about target_s seconds."""
    import oracle
    import kda_inputs

    cores = os.cpu_count() or 1
    oracle.build()
    x = kda_inputs.make_random("prefill", [T_TOK], HEADS, seed=0)
    def run(m, L):
        sl = lambda t: t[:, :L, :m].contiguous()
        t0 = time.perf_counter()
        oracle.kda_fwd(sl(x.q), sl(x.k), sl(x.v), sl(x.g), sl(x.beta), x.scale, x.A_log[:m], x.dt_bias[:m],
                       x.lower_bound, initial_state=None, cu_seqlens=torch.tensor([0, L], dtype=torch.int32),
                       num_threads=cores)
        return time.perf_counter() - t0
    m = min(HEADS, cores)
    cal = run(m, 1024)
    # grow the sample to about target_s: first the token count, then the heads (multiples of cores)
    scale = target_s / max(cal, 1e-3)
    L = int(min(T_TOK, max(1024, 1024 * scale)))
    m = int(min(HEADS, max(m, m * scale * 1024 / L // m * m)))
    dt = run(m, L)
    return {"value": m * L / dt / 1e6, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"heads 0..{m - 1}, tokens 0..{L - 1} of the prefill workload (fp64 C oracle, "
                      f"OpenMP over heads), {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    steps = []
    cb = None
    for i in range(args.warmup + args.steps):
        cb = cpu_oracle_sample(target_s=min(20.0, 150.0 / max(1, args.warmup + args.steps)))
        if i >= args.warmup:
            steps.append(cb["value"])
    v = statistics.median(steps)
    cb["value"] = v
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": cb["sample"]},
            "cpu_baseline": cb, "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-step measurement")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass measurement")
    ap.add_argument("--no-kcp", action="store_true", help="skip the sequence-parallel rank-work measurement")
    ap.add_argument("--bwd-heads", type=int, default=HEADS,
                    help="heads of the backward workload (default 96; fewer only for small profiling runs)")
    ap.add_argument("--heads", type=int, default=HEADS,
                    help="heads of the prefill workload (default 96; fewer only for small profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import kda_inputs
    import kimi_delta_attention_24_b200 as kda

    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    kda.load()
    if args.heads == HEADS:
        x = kda_inputs.make_workload("prefill", seed=rank, device=dev)
    else:
        x = kda_inputs.make_random("prefill", [T_TOK], args.heads, seed=rank, device=dev)
    B, T, H, K = x.q.shape
    N = x.num_seqs
    out = torch.empty_like(x.v)
    final = torch.empty(N, H, K, K, dtype=torch.float32, device=dev)
    ws = kda.new_workspace(B * T, H, N, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.fwd(x.q, x.k, x.v, x.g, x.beta, x.scale, out, ws, x.A_log, x.dt_bias, x.lower_bound,
                None, final, x.cu_seqlens, stream=stream.cuda_stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert kda.read_device_status(ws) == 0
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    launch_ms = [a.elapsed_time(b) for a, b in evs]
    kernel_ms = max_over_ranks(statistics.mean(launch_ms), world)
    status = kda.read_device_status(ws)
    ms_per_step = total_ms / args.steps
    token_heads = B * T * H
    value = replica_throughput(token_heads, ms_per_step, world)

    # end to end through the public API with pinned host buffers: H2D inputs, kernel, D2H outputs
    host = {n: getattr(x, n).cpu().pin_memory() for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "cu_seqlens")}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    fin_h = torch.empty(final.shape, dtype=final.dtype).pin_memory()
    dev_bufs = {n: torch.empty_like(t, device=dev) for n, t in host.items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + fin_h.numel() * fin_h.element_size()

    # Each step copies its inputs in on a copy-in stream, runs kda.fwd on the compute stream and
    # copies o and the final state out on a copy-out stream (the two directions use different copy
    # engines).  Inputs and outputs alternate between two device buffer sets, so step i + 1's
    # inputs travel in while step i computes and step i - 1's outputs travel back; a set is
    # rewritten only after the work that read it has finished.
    h2d_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)
    ins = [dev_bufs, {n: torch.empty_like(t) for n, t in dev_bufs.items()}]
    outs = [out, torch.empty_like(out)]
    finals = [final, torch.empty_like(final)]
    outs_h = [out_h, torch.empty(out.shape, dtype=out.dtype).pin_memory()]
    fins_h = [fin_h, torch.empty(final.shape, dtype=final.dtype).pin_memory()]
    in_ready = [torch.cuda.Event(), torch.cuda.Event()]  # inputs of set b copied in
    ready = [torch.cuda.Event(), torch.cuda.Event()]     # kda.fwd on set b finished
    done = [torch.cuda.Event(), torch.cuda.Event()]      # copy-out of set b finished

    def e2e_step(i):
        b = i & 1
        d = ins[b]
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(ready[b])
            for n, t in host.items():
                d[n].copy_(t, non_blocking=True)
            in_ready[b].record(h2d_stream)
        stream.wait_event(in_ready[b])
        stream.wait_event(done[b])
        kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], x.scale, outs[b], ws, d["A_log"], d["dt_bias"],
                x.lower_bound, None, finals[b], d["cu_seqlens"], stream=stream.cuda_stream)
        ready[b].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ready[b])
            outs_h[b].copy_(outs[b], non_blocking=True)
            fins_h[b].copy_(finals[b], non_blocking=True)
            done[b].record(d2h_stream)

    e2e = None
    if args.e2e_steps > 0:
        for b in range(2):
            ready[b].record(stream)
            done[b].record(d2h_stream)
        e2e_step(0)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d_stream.wait_stream(stream)  # the first copy-in starts inside the timed region
        for i in range(args.e2e_steps):
            e2e_step(i)
        stream.wait_stream(h2d_stream)
        stream.wait_stream(d2h_stream)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world)
        e2e = {"value": replica_throughput(token_heads, e2e_ms, world), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    in_bytes = sum(t.numel() * t.element_size() for t in (x.q, x.k, x.v, x.g, x.beta))
    hbm_peak, tf_peak, peak_kind = load_peaks()
    alg_bytes = algorithmic_bytes(B * T, H, N)
    achieved = alg_bytes / (kernel_ms * 1e-3) / 1e9
    flops = FLOPS_PER_TOKEN_HEAD * token_heads
    traffic = None
    tp = os.path.join(ROOT, "profiles", "kda_fwd_prefill_h32_traffic.json")
    if os.path.exists(tp) and H == HEADS:
        with open(tp) as f:
            traffic = json.load(f).get("dram_bytes_per_call")  # measured at 32 heads, scaled to 96

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD if H == HEADS else WORKLOAD.replace("H=96", f"H={H}"), "batch": B, "seq_len": T, "heads": H, "head_dim": K, "chunk": CHUNK,
                   "parallelism": f"replicas{world}",
                   "l2": f"inputs ({in_bytes / 1e9:.2f} GB) exceed L2 (126 MB); no flush"},
        "tflops": flops / (kernel_ms * 1e-3) / 1e12,
        "tflops_frac_of_bf16_peak": flops / (kernel_ms * 1e-3) / 1e12 / tf_peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": alg_bytes, "kernel_ms": kernel_ms},
        "e2e": e2e,
        "gpu_launches": kda.fwd_launch_count(B * T, H, N) * args.steps,
        "clocks": clk.summary(),
        "device_status": status,
    }
    if not args.no_decode:
        line["decode"] = bench_decode(dev, steps=max(args.steps, 10), warmup=args.warmup, seed=rank)
    if not args.no_backward:
        line["backward"] = bench_backward(dev, steps=2, warmup=1, seed=rank, heads=args.bwd_heads)
    if not args.no_kcp:
        line["kcp_rank_work"] = bench_kcp_rank(dev, steps=5, warmup=2, seed=rank)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample()
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
