"""The multi-rank logic of bench.py (one process per GPU, no data-path
collective; max-over-ranks device time; whole-job weak-scaling throughput;
only rank 0 reports), run as two gloo ranks on CPU."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist

    import bench
    r, w, local = bench.dist_setup(world, backend="gloo")
    assert (r, w, local) == (rank, world, rank)
    # each rank timed a different device time; everyone must see the slowest
    slow = bench.max_over_ranks(10.0 + 3.0 * rank, w, device="cpu")
    bench.barrier(w)
    value = bench.weak_scaling_value(32768, w, slow)
    # the reference arm: only rank 0 prints (the others return 0, silently)
    buf = io.StringIO()
    rc = 0
    if rank != 0:
        class A:  # noqa: N801
            gpus, steps, warmup = world, 1, 0
        with redirect_stdout(buf):
            rc = bench.run_reference(A)
    out[rank] = (slow, value, rc, buf.getvalue())
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        slow, value, rc, printed = out[r]
        assert slow == 13.0
        assert abs(value - 2 * 32768 / 0.013) < 1e-6 * value
        assert rc == 0
    assert out[1][3] == ""
