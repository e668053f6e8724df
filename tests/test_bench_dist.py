"""The multi-rank path of bench.py on CPU (gloo, world size 2).

Each rank of a multi-GPU run decodes its own batch (replicas, no collective on the
data path); the job's time is the slowest rank's and its value is the work of all
ranks over that time.  These tests run that reduction over two gloo ranks, and the
reference arm under torchrun, where rank 0 alone times the oracle and prints.
"""
import json
import os
import socket
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = bench._max_over_ranks(10.0 * rank + 1.0, world)  # rank 1 is the slow one: 11 ms
        value = bench._job_value(world, 16, 100, ms)
        with open(os.path.join(outdir, f"r{rank}.json"), "w") as fh:
            json.dump({"ms": ms, "value": value}, fh)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_on_two_gloo_ranks():
    import torch.multiprocessing as mp
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(2, port, d), nprocs=2, start_method="spawn", join=True)
        got = [json.load(open(os.path.join(d, f"r{r}.json"))) for r in range(2)]
    for g in got:
        assert g["ms"] == 11.0  # every rank sees the slowest rank's time
        assert g["value"] == pytest.approx(2 * 16 * 100 / 0.011)  # both ranks' tokens over that time


def test_job_value_one_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._max_over_ranks(3.5, 1) == 3.5
    assert bench._job_value(1, 16, 1000, 40.0) == pytest.approx(16 * 1000 / 0.040)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--workload", "tiny", "--steps", "2", "--warmup", "1", "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["workload"] == "tiny" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
