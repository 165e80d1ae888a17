"""Multi-process plumbing of bench.py on CPU (gloo, world size 2): the timed
region's length is the slowest rank's, the reported value aggregates every
rank's replica (weak scaling), and the CPU reference arm runs on rank 0 only.
No GPU is involved: the data path has no collective, only this bookkeeping
does."""
import json
import os
import socket
import subprocess
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["SBA_ROOT"])
import bench
pg = bench.dist_init("gloo", timeout_s=60)
rank = int(os.environ["RANK"])
ws = int(os.environ["WORLD_SIZE"])
slowest = bench.max_over_ranks(10.0 + 5.0 * rank, pg)
value = bench.whole_job_tflops(2e12, ws, slowest)
pg.barrier()
pg.destroy_process_group()
print(json.dumps({"rank": rank, "slowest_ms": slowest, "value": value}))
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_gloo_ranks_agree_on_the_slowest_time_and_the_job_value():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                   RANK=str(rank), LOCAL_RANK=str(rank), SBA_ROOT=ROOT)
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=120)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("gloo ranks did not finish")
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["slowest_ms"] == 15.0
        assert abs(o["value"] - 2 * 2e12 / 15e-3 / 1e12) < 1e-9


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_init("gloo") is None or int(os.environ.get("WORLD_SIZE", "1")) > 1
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.whole_job_tflops(1e12, 1, 1000.0) == 1.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = types.SimpleNamespace(workload="wan", steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args) == 0  # returns at once, no data generated


def test_block_lengths_count_every_real_token_once():
    """The bench's real-token FLOP count: block lengths sum to N in both
    orders, cube order follows the grid's edge cubes, Hilbert order has full
    blocks but the last (checked against the oracle's own lengths)."""
    sys.path.insert(0, ROOT)
    import bench
    import datagen
    import numpy as np
    import oracle
    for wl in (datagen.WORKLOADS["wan"], datagen.WORKLOADS["small"],
               datagen.with_order(datagen.WORKLOADS["wan"], "hilbert"),
               datagen.custom("odd", 1, 1, 3, 17, 17, 128, (1, 8, 8))):
        lens = bench._block_lens(wl)
        g = oracle.Geom(wl.T, wl.Hh, wl.W, *wl.cube, order=getattr(wl, "order", "cube"))
        assert sum(lens) == wl.T * wl.Hh * wl.W
        assert np.array_equal(np.array(lens), oracle.block_len(g))
