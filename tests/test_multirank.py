"""The multi-GPU host logic of the benchmark on CPU: two gloo ranks.

Every rank runs an independent replica (its own seed, no data-path
collective); the only exchange is the max-over-ranks reduction of the step
time, and the job's throughput counts every rank's queries over that time.
The reference arm runs on rank 0 alone."""
import os
import socket
import subprocess
import sys

import numpy as np
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


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0", "--cpu-seconds", "1"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
