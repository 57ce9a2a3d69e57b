"""Multi-rank host logic of the benchmark, on CPU with the gloo backend (world size 2).

Tail replays of different requests are independent (Tail-Replay reading notes §2.4: every
group restarts from its own exact cached hiddens), so ranks share no data: each replays its
own request, and only the step time crosses ranks (the slowest rank sets the job time).
These tests run two real processes that rendezvous on 127.0.0.1 and check that:
- the max over ranks is what every rank sees;
- the job throughput counts the units of all ranks against that max time;
- ranks draw different requests, reproducibly;
- the reference arm does its work on rank 0 only and prints one line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank step times: rank 1 is the slow one
        mine = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(mine, world, "cpu")
        value = bench.job_throughput(1639, world, mx / 4)
        seed = bench.rank_seed(rank)
        h = synth.hidden_prefix(64, 32, seed)
        # gather what every rank drew, to compare on rank 0
        hs = [torch.empty_like(h) for _ in range(world)]
        dist.all_gather(hs, h)
        res = {"rank": rank, "max": mx, "value": value, "seed": seed,
               "same_as_other": bool(torch.equal(hs[0], hs[1])),
               "again": bool(torch.equal(h, synth.hidden_prefix(64, 32, seed)))}
        with open(os.path.join(out_dir, "r%d.json" % rank), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, "rank exited with %s" % p.exitcode
    res = [json.load(open(tmp_path / ("r%d.json" % r))) for r in range(world)]
    for r in res:
        assert r["max"] == 15.0                      # the slow rank's time, seen by both
        assert r["value"] == pytest.approx(2 * 1639 / (15.0 / 4 * 1e-3))
        assert not r["same_as_other"]                # independent requests
        assert r["again"]                            # reproducible per rank
    assert res[0]["seed"] != res[1]["seed"]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_throughput(100, 1, 2.0) == pytest.approx(50000.0)


def test_reference_arm_rank_split(tmp_path):
    """Under torchrun with 2 ranks, rank 0 alone times the oracle and prints; rank 1 exits 0."""
    port = _free_port()
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--sample-tokens", "8"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=str(tmp_path))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
