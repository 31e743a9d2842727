"""The multi-process path of bench.py on CPU: two ranks over gloo, started the
way torchrun starts them (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR/PORT in the
environment). The path runs independent replicas (weak scaling): each rank
draws its own inputs, the ranks meet only at barriers, and the timed result is
the slowest rank's time."""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import tri_inputs
    import torch.distributed as dist

    r, wsz, local = bench.dist_setup(backend="gloo")
    try:
        bench.barrier(wsz)
        # each rank reports a different local time; all receive the slowest
        slowest = bench.max_over_ranks(10.0 + rank, wsz)
        # replicas draw distinct inputs (seed + rank), as run_ours does
        w = tri_inputs.WORKLOADS["n32_f32"]
        q = tri_inputs.workload_inputs(w.name, seed=w.seed + r)["q"]
        gathered = [torch.zeros_like(q) for _ in range(wsz)]
        dist.all_gather(gathered, q)
        distinct = not torch.equal(gathered[0], gathered[1])
        value = bench.whole_job_tflops(wsz, 2e12, slowest)
        bench.barrier(wsz)
        queue.put((r, wsz, local, slowest, distinct, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        # read the results before joining: a rank exits only after its queue
        # data has been taken
        results = sorted(queue.get(timeout=180) for _ in range(world))
        for p in procs:
            p.join(timeout=60)
        codes = [p.exitcode for p in procs]
    finally:
        for p in procs:
            if p.is_alive():
                p.kill()
    assert codes == [0, 0], f"rank exit codes {codes}"
    for rank, (r, wsz, local, slowest, distinct, value) in enumerate(results):
        assert (r, wsz, local) == (rank, world, rank)
        assert slowest == 11.0                     # the max over ranks, on every rank
        assert distinct                            # independent replicas
        # two replicas of 2 TFLOP each in 11 ms: 2 * 2e12 / 0.011 s
        assert value == pytest.approx(2 * 2e12 / 11e-3 / 1e12)


def test_reference_arm_other_ranks_do_no_work():
    """Under torchrun the reference arm runs on rank 0 only; other ranks return
    at once without touching the oracle."""
    sys.path.insert(0, ROOT)
    import bench
    import tri_inputs

    class Args:
        steps, warmup, ref_budget_s = 3, 1, 1.0

    assert bench.run_reference(Args, rank=1, world=2, w=tri_inputs.WORKLOADS["n768_bf16"]) is None


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tflops(1, 1e12, 1.0) == pytest.approx(1000.0)
