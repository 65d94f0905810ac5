"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the job's
time is the maximum over ranks, every rank rotates its own inputs, and the
reference arm runs on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import seeded_inputs as S  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports times r+1 and 10-r: the job's are the maxima
        q.put((rank, bench.max_over_ranks([rank + 1.0, 10.0 - rank], world, "cpu")))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1] == [2.0, 10.0]


def test_max_over_ranks_one_rank_is_identity():
    assert bench.max_over_ranks([3.5, 1.25], 1, "cpu") == [3.5, 1.25]


def test_every_rank_rotates_its_own_inputs():
    m = S.master_seed(1)
    seeds = {bench.rank_seed(m, r) for r in range(8)}
    assert len(seeds) == 8
    a = S.uniform_residues(bench.rank_seed(m, 0), "ct_residues", [1099511627689], 1024, lead=(1,))
    b = S.uniform_residues(bench.rank_seed(m, 1), "ct_residues", [1099511627689], 1024, lead=(1,))
    assert not np.array_equal(a, b)


def test_reference_arm_two_ranks_prints_once():
    """torchrun with 2 ranks (gloo): rank 0 times the oracle and prints one
    line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.5"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_oracle_baselines_of_the_rotation_cases():
    """The reference leg of the hoisted and rotate-and-sum cases: the oracle
    on a bounded full-size sample, reported as rotations/s."""
    for case in ("hoisted", "rotsum"):
        r = bench.workload_cpu_baseline(case, 0.5)
        assert r["kind"] == "oracle" and r["unit"] == "rotations/s" and r["value"] > 0 and r["cores"] >= 1
        assert "key generation excluded" in r["sample"]
