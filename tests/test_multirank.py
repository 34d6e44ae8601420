"""The multi-GPU path of bench.py on CPU: world size 2 over gloo.

Every rank runs an independent replica of the workload (the batches do not
interact, so there is no collective on the data path); only the timing
crosses ranks: the job's time is the slowest rank's and its throughput the
units of all ranks over that time.  These tests run that aggregation, the
barrier and the reference arm's rank handling as real processes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist("gloo")
    try:
        d.barrier()
        res = {
            "max": d.max(float(rank + 1)),
            "sum": d.sum(10.0 * (rank + 1)),
            # rank r scored 24 positions in (r + 1) * 0.1 ms
            "agg": bench.replica_throughput(d, 24.0, 0.1 * (rank + 1)),
        }
        d.barrier()
    finally:
        d.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_dist_and_replica_throughput_world2(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == 2.0 and r["sum"] == 30.0
        ms, value = r["agg"]
        assert ms == pytest.approx(0.2)
        assert value == pytest.approx(48.0 / 0.2e-3)   # all ranks' units over the slowest time
    assert res[0]["agg"] == res[1]["agg"]


def test_reference_arm_under_torchrun_world2():
    """Rank 0 alone runs the reference arm and prints one JSON line; rank 1
    exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny_f32"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
