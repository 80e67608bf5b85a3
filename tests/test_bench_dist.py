"""bench.py's multi-rank plumbing on CPU: two gloo ranks (no GPU).

The N > 1 bench runs one replica per GPU; the only cross-rank steps are the barrier
around the timed region, the max over ranks of the device time, and "rank 0 alone
prints" (the reference arm: ranks other than 0 exit without work).  Those helpers are
exercised here with torch.distributed over gloo on 127.0.0.1.
"""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    got = bench.dist_env()
    bench.barrier()
    t_max = bench.reduce_max(1.5 + rank)          # per-rank "device time"
    bench.barrier()
    # the reference arm: every rank but 0 returns 0 before doing any work
    skipped = None
    if rank != 0:
        skipped = bench.run_reference(type("A", (), dict(iters=1, steps=1, warmup=0))())
    bench.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(f"{got[0]} {got[1]} {got[2]} {t_max} {skipped}\n")


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    rows = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for r, row in enumerate(rows):
        assert [int(x) for x in row[:3]] == [r, r, world]
        assert float(row[3]) == 1.5 + (world - 1)      # max over ranks on every rank
    assert rows[0][4] == "None" and rows[1][4] == "0"


def test_single_process_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25) == 3.25
    bench.barrier()                                      # no process group: nothing to do
