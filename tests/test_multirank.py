"""Multi-rank host logic on CPU with the gloo backend (world size 2): each rank runs its own
independent batch (no collective on the data path); barriers bracket the timed region and the
slowest rank's time sets the job's throughput."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from sequence_ring_self_b200 import dist as rdist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np

    from oracle import oracle
    from sequence_ring_self_b200.inputs import make_inputs

    assert rdist.init("gloo", timeout_s=60)
    r, w, lr = rdist.env_ranks()
    assert (r, w, lr) == (rank, world, rank)
    # each rank: its own seeded batch, its share of the heads
    x = make_inputs(1, 4, 32, 8, seed=10 + rank, dtype="bf16")
    heads = rdist.shard(4, rank, world)
    o, _ = oracle.forward(x.q[:, heads.start:heads.stop], x.k[:, heads.start:heads.stop],
                          x.v[:, heads.start:heads.stop])
    rdist.barrier()
    my_time = 1.0 + rank  # stand-in per-rank times: the slowest must win
    slowest = rdist.max_over_ranks(my_time)
    thr = rdist.weak_scaling_throughput(100.0, world, slowest)
    out.put((rank, slowest, thr, float(np.abs(o).sum())))
    rdist.finish()


def test_two_rank_gloo_timing_and_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [2.0, 2.0]          # max over ranks
    assert [r[2] for r in res] == [100.0, 100.0]      # 100 units x 2 ranks / 2 s
    assert res[0][3] != res[1][3]                     # independent batches per rank


def test_shard_covers_every_unit_once():
    for n in (1, 5, 96, 97):
        for world in (1, 2, 3, 8):
            got = [i for r in range(world) for i in rdist.shard(n, r, world)]
            assert got == list(range(n))


def test_weak_scaling_rejects_bad_time():
    with pytest.raises(ValueError):
        rdist.weak_scaling_throughput(1.0, 2, 0.0)


def test_reference_arm_under_torchrun_two_ranks():
    """bench.py --impl reference launched like the driver's N=2 run: rank 0 prints one JSON
    line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-budget", "4"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json

    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
