"""World-size-2 checks of the multi-GPU host logic on CPU (gloo): each rank draws its own batch
of the same shape, and the job time is the maximum over ranks.  The attention path itself
needs no collective (every (batch, head) is independent)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads
        w = workloads.sweep(4096, 16, 128, False)
        wr = bench.rank_workload(w, rank)
        small = workloads.custom(1, 1, 16, 64, False, seed=wr.seed)
        first = workloads.make_inputs(small).q.float().sum().item()
        mx = bench.reduce_max([1.0 + rank, 10.0 - rank], world)
        gathered = [None] * world
        dist.all_gather_object(gathered, (wr.seed, wr.B, wr.H, wr.N, wr.d, first))
        out[rank] = (mx, gathered)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_independent_batches_and_max_time():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        mx, gathered = out[rank]
        assert mx == [2.0, 10.0]
        (s0, *shape0, f0), (s1, *shape1, f1) = gathered
        assert shape0 == shape1          # same per-GPU shape: weak scaling
        assert s0 != s1 and f0 != f1     # different seeded data per rank


def test_bench_launches_its_own_ranks():
    """`bench.py --gpus 2` without a launcher starts two ranks itself (torch.distributed.run on
    127.0.0.1); the rank self-test runs the same launch and max-over-ranks path on gloo, and
    rank 0 alone prints one line that reports both ranks."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                          "--selftest-ranks", "--launch-timeout", "240"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2
    assert line["ms_max_over_ranks"] == [11.0, 100.0]  # rank 1's first, rank 0's second value
