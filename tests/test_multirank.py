"""The multi-rank host path of bench.py on CPU: two gloo ranks.

With N GPUs bench.py runs N independent replicas (decode sequences are
independent; no data-path collective).  Its only cross-rank steps are the
barrier and the max-over-ranks of the device timings, and the reference arm
runs on rank 0 alone.  Both are exercised here with world_size 2 over gloo.
"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports (10 + r, 3 - r) ms: the job's times are the maxima
        got = bench.max_over_ranks([10.0 + rank, 3.0 - rank], "cpu")
        dist.barrier()
        with open(os.path.join(out_dir, f"max_{rank}.txt"), "w") as f:
            f.write(" ".join(str(v) for v in got))
        # the reference arm prints on rank 0 only; other ranks return at once
        if rank != 0:
            class A:
                workload, steps, warmup = "tiny", 1, 0
            bench.run_reference(A())
            with open(os.path.join(out_dir, f"ref_{rank}.txt"), "w") as f:
                f.write("returned")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_only_rank0_runs_the_reference(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        vals = [float(v) for v in (tmp_path / f"max_{r}.txt").read_text().split()]
        assert vals == [11.0, 3.0]
    assert (tmp_path / "ref_1.txt").read_text() == "returned"


def test_max_over_ranks_without_a_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], "cpu") == [1.5, 2.5]
