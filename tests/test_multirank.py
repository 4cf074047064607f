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


def _shard_main(rank, world, port, out):
    import numpy as np
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from atomistic_neighbor_list_b200 import mp, synth
    pos, gp = synth.positions_for(synth.WORKLOADS["cfg3"])  # 64 chains of 1,000 beads
    g0, g1, a0, a1 = mp.shard_graphs(gp, rank, world)
    # this rank's own system: its atoms and its graphs, rebased; a per-graph host quantity stands
    # in for the per-graph energies (no GPU here)
    sub_pos, sub_gp = pos[a0:a1], gp[g0:g1 + 1] - a0
    mine = [float(np.asarray(sub_pos[sub_gp[g]:sub_gp[g + 1]], dtype=np.float64).sum())
            for g in range(len(sub_gp) - 1)]
    got = [None] * world
    dist.all_gather_object(got, (g0, g1, a0, a1, mine))
    out[rank] = got
    dist.destroy_process_group()


def test_replica_shards_cover_every_graph_once_and_reassemble_in_order():
    import numpy as np
    sys.path.insert(0, ROOT)
    from atomistic_neighbor_list_b200 import synth
    pos, gp = synth.positions_for(synth.WORKLOADS["cfg3"])
    full = [float(np.asarray(pos[gp[g]:gp[g + 1]], dtype=np.float64).sum())
            for g in range(len(gp) - 1)]
    for world in (2, 3):
        port = _free_port()
        out = tmp.get_context("spawn").Manager().dict()
        tmp.start_processes(_shard_main, args=(world, port, out), nprocs=world, join=True,
                            start_method="spawn")
        shards = out[0]
        assert shards == out[world - 1]  # every rank saw the same gathered list
        assert shards[0][0] == 0 and shards[-1][1] == len(gp) - 1
        for a, b in zip(shards, shards[1:]):
            assert a[1] == b[0] and a[3] == b[2]  # contiguous, in rank order
        sizes = [s[3] - s[2] for s in shards]
        assert max(sizes) - min(sizes) <= int(np.max(np.diff(gp)))
        assert [v for s in shards for v in s[4]] == full


def test_shard_graphs_edge_cases():
    import numpy as np
    import pytest
    sys.path.insert(0, ROOT)
    from atomistic_neighbor_list_b200 import mp
    gp = np.array([0, 10, 30, 35, 60, 100], dtype=np.int32)
    assert [mp.shard_graphs(gp, r, 2) for r in range(2)] == [(0, 4, 0, 60), (4, 5, 60, 100)]
    assert [mp.shard_graphs(gp, r, 3)[:2] for r in range(3)] == [(0, 3), (3, 4), (4, 5)]
    seven = [mp.shard_graphs(gp, r, 7)[:2] for r in range(7)]  # more ranks than graphs
    assert seven[0][0] == 0 and seven[-1][1] == 5
    assert all(a[1] == b[0] for a, b in zip(seven, seven[1:]))
    assert mp.shard_graphs(np.array([5, 9], dtype=np.int32), 0, 4) == (0, 0, 5, 5)
    for bad in ((gp, 2, 2), (gp, -1, 2), (np.array([0, 5, 3], dtype=np.int32), 0, 2)):
        with pytest.raises(mp.MpError):
            mp.shard_graphs(*bad)


def test_bench_sharded_systems_make_up_the_workload():
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    from atomistic_neighbor_list_b200 import synth
    wl = synth.WORKLOADS["cfg3"]
    pos, gp = synth.positions_for(wl)
    parts = [bench.rank_system(wl, r, 3, True) for r in range(3)]
    assert np.array_equal(np.concatenate([p for p, _ in parts]), pos)
    starts = np.cumsum([0] + [len(p) for p, _ in parts])
    rebuilt = np.concatenate([[0]] + [g[1:] + s for (_, g), s in zip(parts, starts)])
    assert np.array_equal(rebuilt, gp)
    assert all(g[0] == 0 for _, g in parts)
    # without sharding each rank runs its own full-size replica system
    p1, g1 = bench.rank_system(wl, 1, 3, False)
    assert len(p1) == len(pos) and not np.array_equal(p1, pos)
