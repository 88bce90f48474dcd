"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks (one process each, as torchrun starts
them) set up the process group from the launcher's environment, meet at the barrier, agree on the
slowest rank's step time and compute the whole-job throughput from it.  The path has no data
exchange (replicas only), so this is all of its multi-rank logic.  No GPU is used."""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    r, w, _ = bench.dist_setup(world)
    bench.barrier(w)
    ms = 2.0 + rank  # rank 1 is the slower one
    slowest = bench.max_over_ranks(ms, w)
    value = bench.replica_throughput(1000, slowest, w)
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((r, w, dist.is_initialized(), slowest, value))


def test_two_gloo_ranks_agree_on_the_slowest_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[:3] for r in results] == [(0, 2, False), (1, 2, False)]
    for _, _, _, slowest, value in results:
        assert slowest == 3.0  # max over ranks, not the local time
        # weak scaling: both replicas' token-heads over the slowest rank's time
        assert abs(value - 2 * 1000 / 3e-3 / 1e6) < 1e-12


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        gpus, steps, warmup = 2, 1, 3

    bench.run_reference(Args, rank=1, world=2)  # returns at once: no oracle work, no output
    assert capsys.readouterr().out == ""
