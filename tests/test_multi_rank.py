"""The N > 1 plumbing of bench.py on CPU ranks (gloo, world size 2): the max-over-ranks device time,
the whole-job throughput of independent replicas, and the reference arm under torchrun (rank 0
prints the one JSON line, the other rank exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    bench.init_dist(world, rank, "gloo")
    try:
        # each rank "timed" a different duration; every rank must see the slowest one
        ms = bench.max_over_ranks(torch, 10.0 + 5.0 * rank, world, torch.device("cpu"))
        torch.distributed.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": bench.replica_throughput(1e9, 10, world, ms)}, f)
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_replica_value_gloo(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["ms"] == 15.0
        # 2 replicas x 10 steps x 1 GB in 15 ms
        assert g["value"] == pytest.approx(2 * 10 * 1e9 / 15e-3 / 1e9)


def test_replica_throughput_is_whole_job():
    assert bench.replica_throughput(81346560, 100, 1, 10.0) == pytest.approx(813.4656)
    assert bench.replica_throughput(81346560, 100, 8, 10.0) == pytest.approx(8 * 813.4656)


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
