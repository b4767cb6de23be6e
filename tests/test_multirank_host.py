"""The bench's multi-rank plumbing with two gloo ranks on the CPU.

With N GPUs, bench.py runs one process per GPU; every rank decodes its own
sequence (weak scaling, no data-path collective).  The ranks meet only at a
barrier around the timed region, and rank 0 reports the slowest rank's time.
These tests run that plumbing (rendezvous from the environment, barrier,
max over ranks) in two processes over gloo, and check that the reference arm
does its work on rank 0 only.
"""
import importlib.util
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    bench = _bench()
    r, w, local = bench.dist_init(world)
    import torch.distributed as dist
    try:
        bench.barrier(w)
        mx = bench.max_over_ranks(10.0 + 5.0 * r, w, torch.device("cpu"))   # rank 1 is the slower one
        bench.barrier(w)
        out.put((r, w, local, mx, dist.get_backend()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_barrier_and_max_over_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(out.get(timeout=10) for _ in range(2))
    assert [x[0] for x in res] == [0, 1]
    for r, w, local, mx, backend in res:
        assert w == 2 and local == r and backend == "gloo"
        assert mx == 15.0          # every rank sees the slowest rank's time


def test_single_rank_needs_no_process_group():
    bench = _bench()
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)              # a no-op with one rank


@pytest.mark.parametrize("workload", ["decode", "tiny", "single", "ragged", "verify", "prefill", "quantize"])
def test_reference_arm_runs_on_rank_zero_only(workload, capsys):
    bench = _bench()

    class Args:
        gpus, steps, warmup, impl = 2, 1, 3, "reference"

    Args.workload = workload
    bench.run_reference(Args(), 1, 2)   # rank 1 of 2: no oracle work, no output
    assert capsys.readouterr().out == ""
