"""The bench's multi-rank plumbing on CPU: two gloo ranks agree on the slowest
rank's time, and the replicas' throughput counts every rank's bytes over it.
No GPU: the ranks exchange host tensors."""
import json
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")   # rank 1 is slower
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump([ms, bench.replica_gbs(1e9, ms, world)], f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time(tmp_path):
    world = 2
    mp.spawn(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)   # spawn, not fork
    got = {r: json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)}
    assert got[0][0] == got[1][0] == 15.0
    # 2 ranks x 1 GB over 15 ms
    assert abs(got[0][1] - 2 * 1e9 / 15e-3 / 1e9) < 1e-9


def test_one_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert abs(bench.replica_gbs(1e9, 2.0, 1) - 500.0) < 1e-9
