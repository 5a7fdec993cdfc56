"""The N > 1 path of the benchmark on CPU: two gloo ranks, each an independent
replica, combine their timings as the benchmark does (max over ranks, bytes of
all ranks), and the reference arm does work on rank 0 only.  No GPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0][rank]             # each replica's own device time
        nbytes = 1_000_000_000            # each replica's algorithmic bytes
        value, ms_max = bench.replica_throughput(nbytes, ms, dist, device="cpu")
        q.put((rank, value, ms_max, bench.max_over_ranks(ms, dist, device="cpu")))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_combine_as_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, ms_max, mx in got:
        assert ms_max == 5.0 and mx == 5.0          # the slowest rank's time
        assert value == pytest.approx(2 * 1e9 / 5e-3 / 1e9)  # bytes of both ranks / that time


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    value, ms = bench.replica_throughput(2_000_000, 4.0, None)
    assert ms == 4.0 and value == pytest.approx(2e6 / 4e-3 / 1e9)


def test_reference_arm_works_on_rank_zero_only(capsys):
    """Under torchrun the oracle arm runs and prints on rank 0; other ranks exit
    0 at once without work."""
    sys.path.insert(0, ROOT)
    import bench
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.reference_arm(args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
