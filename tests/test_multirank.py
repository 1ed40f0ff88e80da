"""The multi-GPU host logic of the benchmark on CPU: two gloo ranks.

--split sequences: every rank runs its own sequences of the job (its own
seed, no data-path collective); the only exchange is the max-over-ranks
reduction of the step time, and the job's throughput counts every rank's
queries over that time.  --split queries: one workload is split over the
ranks by causal work and the shards' index rows are assembled with one
all-gather; here each rank runs the CPU oracle on its shard, and the
assembled result must equal the one-process oracle result.  The reference
arm runs on rank 0 alone."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from hierarchical_top_key_b200 import synthetic
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synthetic.WORKLOADS["tiny"]
        inp = synthetic.generate(wl, bench.replica_seed(0, rank), batch=1)
        # a per-rank step time: rank r is (r + 1) ms slow
        ms_max = bench.max_over_ranks(1.0 + rank, world)
        e2e_max = bench.max_over_ranks(10.0 - rank, world)
        out[rank] = (float(inp.q[0, 0, 0, 0]), ms_max, e2e_max,
                     bench.job_rate(wl.batch * wl.num_queries, world, ms_max))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_reduce_max_time():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    q0, q1 = res[0][0], res[1][0]
    assert q0 != q1                                        # independent replicas
    for r in range(world):
        assert res[r][1] == 2.0 and res[r][2] == 10.0       # every rank sees the slowest time
    from hierarchical_top_key_b200 import synthetic
    wl = synthetic.WORKLOADS["tiny"]
    np.testing.assert_allclose(res[0][3], wl.batch * wl.num_queries * 2 / 2e-3)


def _oracle_rows(inp, t0, t1):
    from oracle.run import Sequence
    from oracle import hisa_oracle as ho
    wl = inp.workload
    seq = Sequence(inp, 0)
    rows = np.full((t1 - t0, wl.top_k), -1, np.int32)
    for i, t in enumerate(range(t0, t1)):
        _, idx, _ = seq.hisa(t)
        rows[i] = ho.pad_row(idx, wl.top_k, -1)
    return rows


def _split_rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from hierarchical_top_key_b200 import partition, synthetic
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synthetic.WORKLOADS["tiny"]
        inp = synthetic.generate(wl, 0, batch=1)                 # one job: every rank draws the same inputs
        shards = partition.shard_job(inp.n_visible, wl.block_size, wl.top_m, world)
        s = shards[rank]
        mine = torch.from_numpy(_oracle_rows(inp, s.t0, s.t1))[None]
        full = bench.gather_shards(mine, shards, wl.batch, wl.num_queries, wl.top_k, world)
        out[rank] = (full.numpy(), [(x.t0, x.t1) for x in shards],
                     partition.shard_work(inp.n_visible, wl.block_size, wl.top_m, shards))
    finally:
        dist.destroy_process_group()


def test_query_split_reassembles_the_one_rank_result():
    from hierarchical_top_key_b200 import partition, synthetic
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_split_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    wl = synthetic.WORKLOADS["tiny"]
    inp = synthetic.generate(wl, 0, batch=1)
    whole = _oracle_rows(inp, 0, wl.num_queries)[None]
    for r in range(world):
        np.testing.assert_array_equal(res[r][0], whole)          # every rank holds the assembled [1, Q, k]
    ranges = res[0][1]
    assert ranges[0][0] == 0 and ranges[-1][1] == wl.num_queries
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))  # contiguous, disjoint, covering
    # balanced by causal work, not by count: each shard within one query's work of an equal share
    work = partition.query_work(inp.n_visible, wl.block_size, wl.top_m)
    for w_r in res[0][2]:
        assert w_r <= work.sum() / world + work.max()
    assert ranges[0][1] - ranges[0][0] > wl.num_queries // world  # early queries are cheaper


def test_sequence_split_keeps_whole_sequences():
    from hierarchical_top_key_b200 import partition
    nv = np.full((64, 1), 131072, np.int32)
    nv[::3] = 4096                                               # uneven sequences
    for world in (1, 2, 3, 8):
        shards = partition.shard_job(nv, 128, 64, world)
        assert [s.seq0 for s in shards][0] == 0 and shards[-1].seq1 == 64
        assert all(a.seq1 == b.seq0 for a, b in zip(shards, shards[1:]))
        assert all(s.t0 == 0 and s.t1 == 1 for s in shards)
        work = partition.query_work(nv, 128, 64).sum(axis=1)
        for w_r in partition.shard_work(nv, 128, 64, shards):
            assert w_r <= work.sum() / world + work.max()


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0", "--cpu-seconds", "1"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def _leaving_rank_main(rank, world, port, out):
    import datetime
    import time
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from hierarchical_top_key_b200 import partition, synthetic
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        # this rank leaves between steps, before the shard all-gather
        dist.destroy_process_group()
        out[rank] = "left"
        return
    wl = synthetic.WORKLOADS["tiny"]
    inp = synthetic.generate(wl, 0, batch=1)
    shards = partition.shard_job(inp.n_visible, wl.block_size, wl.top_m, world)
    mine = torch.full((1, shards[0].t1 - shards[0].t0, wl.top_k), -1, dtype=torch.int32)
    t0 = time.monotonic()
    try:
        bench.gather_shards(mine, shards, wl.batch, wl.num_queries, wl.top_k, world)
        out[rank] = ("gathered", time.monotonic() - t0)
    except Exception as e:                              # the collective ends with an error, not a hang
        out[rank] = ("error", time.monotonic() - t0, type(e).__name__)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


@pytest.mark.timeout(180)
def test_a_rank_that_leaves_fails_the_gather_instead_of_hanging():
    """Failure detection on the host: a rank that leaves before the shard
    all-gather of a query split makes the remaining rank's collective end with
    an error within the process group's timeout (10 s here), not wait for good."""
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_leaving_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[1] == "left"
    assert res[0][0] == "error", res[0]
    assert res[0][1] < 60.0
