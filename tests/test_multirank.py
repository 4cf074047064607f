"""The multi-rank host logic of bench.py on CPU: two gloo ranks (world_size 2) agree on the
slowest rank's time, compute the whole-job throughput from it, run independent replicas of the
same size, and only rank 0 works in the reference arm. No GPU."""
import os
import socket
import sys

import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from atomistic_neighbor_list_b200 import synth
    r, w, lr = bench.rank_info()
    mx = bench.max_over_ranks([3.0, 5.0][rank], w, "cpu")
    pos, gp = bench.rank_system(synth.scaled(synth.WORKLOADS["cfg2"], 200), rank)
    dist.barrier()
    out[rank] = (r, w, lr, mx, bench.job_value(w, 10, mx), float(pos.sum()), pos.shape, len(gp))
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_timing_and_run_independent_systems():
    world, port = 2, _free_port()
    mgr = tmp.get_context("spawn").Manager()
    out = mgr.dict()
    tmp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                        start_method="spawn")
    a, b = out[0], out[1]
    assert (a[0], a[1], a[2]) == (0, 2, 0) and (b[0], b[1], b[2]) == (1, 2, 1)
    assert a[3] == b[3] == 5.0                 # the max over ranks, seen by both
    assert a[4] == b[4] == 2 * 10 / 0.005      # world * steps / max seconds
    assert a[6] == b[6] and a[7] == b[7] == 2  # same size ...
    assert a[5] != b[5]                        # ... different systems (seeded by rank)


def test_reference_arm_only_rank_zero_works(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload, steps, warmup = "cfg2", 1, 1

    assert bench.reference_arm(Args()) == 0  # returns at once: no oracle work on rank 1
