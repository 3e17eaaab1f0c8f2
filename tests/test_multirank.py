"""The multi-GPU host logic of the bench on CPU ranks (gloo, world size 2):
the slowest rank's timing is the job's, every rank contributes its own
tokens, and ranks decode different batches with no data-path collective."""
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
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (10 + r) ms for the run and (2 - r) ms per decode call
        got = bench.reduce_over_ranks([10.0 + rank, 2.0 - rank], "cpu")
        out[rank] = got + [bench.rank_seed(rank)]
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_distinct_seeds():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][:2] == [11.0, 2.0] and res[1][:2] == [11.0, 2.0]
    assert res[0][2] != res[1][2]


def test_single_process_and_job_value():
    assert bench.reduce_over_ranks([3.0, 4.0], "cpu") == [3.0, 4.0]
    # two ranks of 64 sequences, 100 steps in 50 ms: 256,000 tokens/s
    assert bench.job_value(2, 64, 100, 50.0) == pytest.approx(256000.0)


def test_reference_arm_prints_one_json_line():
    """--impl reference times the CPU oracle on a bounded sample and prints
    the bench's JSON line with the reference-arm keys."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--cpu-seconds", "1"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "query-tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "long_mqa_b64_m8k"
