"""The head-sharded layer (block_sparse_attention_sba_b200/sharded.py) on CPU
ranks: longest-first placement against brute force, the data and results of
migrating heads over gloo point-to-point transfers, and a rank that leaves
between steps (the others stop with RankLost instead of waiting). The GPU
kernels are replaced by a CPU engine whose per-head results depend only on
that head's data, so any mix-up of heads shows in the outputs."""
import itertools
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_sparse_attention_sba_b200.sharded import lpt_placement, migrations, static_heads  # noqa: E402


def test_lpt_placement_is_longest_first_and_within_grahams_bound():
    import numpy as np
    rng = np.random.default_rng(0)
    for trial in range(300):
        H = int(rng.integers(1, 9))
        W = int(rng.integers(1, 4))
        costs = [int(c) for c in rng.integers(0, 50, size=H)]
        if trial % 5 == 0:
            costs = [7] * H  # all equal: ties go to the lower head and the lower rank
        owner = lpt_placement(costs, W)
        # replay: heads by cost desc (ties lower head), each to the least-loaded rank
        load = [0] * W
        for h in sorted(range(H), key=lambda x: (-costs[x], x)):
            r = min(range(W), key=lambda x: (load[x], x))
            assert owner[h] == r
            load[r] += costs[h]
        # Graham: makespan <= (4/3 - 1/(3W)) * optimum (brute force)
        best = min(max(sum(costs[h] for h in range(H) if a[h] == r) for r in range(W))
                   for a in itertools.product(range(W), repeat=H))
        assert max(load) <= (4 / 3 - 1 / (3 * W)) * best + 1e-9
    assert lpt_placement([5, 1, 1, 1, 1, 1], 2) == [0, 1, 1, 1, 1, 1]


def test_fewer_heads_than_ranks_is_rejected():
    import datetime
    import torch.distributed as dist
    from block_sparse_attention_sba_b200.sharded import HeadShardedAttention
    store = dist.HashStore()
    dist.init_process_group("gloo", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=10))
    try:
        HeadShardedAttention(object(), 1, dist.group.WORLD)  # 1 head, 1 rank: fine
        with pytest.raises(ValueError):
            HeadShardedAttention(object(), 0, dist.group.WORLD)
    finally:
        dist.destroy_process_group()


def test_static_split_and_moves():
    assert static_heads(5, 2, 0) == [0, 2, 4] and static_heads(5, 2, 1) == [1, 3]
    assert migrations([0, 1, 0, 0, 1], 2) == [(3, 1, 0), (4, 0, 1)]


WORKER = r"""
import json, os, sys, datetime
sys.path.insert(0, os.environ["SBA_ROOT"])
import torch
import torch.distributed as dist
from block_sparse_attention_sba_b200.sharded import HeadShardedAttention, RankLost

class CpuEngine:
    # per-head results that depend only on that head's data
    def reorder(self, q, k, v):
        perm = torch.arange(q.shape[2] - 1, -1, -1)
        return q[:, :, perm].clone(), k[:, :, perm].clone(), v[:, :, perm].clone()
    def route_cost(self, qt, kt, top_p, top_k):
        return (qt[0, :, 0, 0] * 100).round().long()
    def attend(self, qt, kt, vt, top_p, top_k):
        return qt + 2 * kt - vt * torch.tensor(top_p).view(1, -1, 1, 1)
    def unreorder(self, ot):
        perm = torch.arange(ot.shape[2] - 1, -1, -1)
        return ot[:, :, perm].clone()

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
pg = dist.group.WORLD
store = dist.TCPStore("127.0.0.1", int(os.environ["STORE_PORT"]), world, rank == 0,
                      timeout=datetime.timedelta(seconds=20))
H, N, d = 7, 6, 4
g = torch.Generator().manual_seed(0)
Q = torch.randn(1, H, N, d, generator=g); K = torch.randn(1, H, N, d, generator=g)
V = torch.randn(1, H, N, d, generator=g)
Q[0, :, N - 1, 0] = torch.tensor([9.0, 0.5, 0.4, 0.3, 0.2, 0.1, 0.05])  # head 0 is heavy
top_p = [0.5 + 0.05 * h for h in range(H)]
layer = HeadShardedAttention(CpuEngine(), H, pg, store=store, checkin_timeout_s=3.0)
mine = layer.my_heads()
eng = CpuEngine()
res = {"rank": rank, "steps": []}
leave_after = int(os.environ.get("LEAVE_AFTER", "-1"))
try:
    for step in range(2):
        if rank == leave_after and step == 1:
            res["left"] = True
            print(json.dumps(res), flush=True)
            os._exit(0)
        o = layer(Q[:, mine], K[:, mine], V[:, mine], top_p, 8)
        # the same heads computed locally, without sharding
        qt, kt, vt = eng.reorder(Q[:, mine], K[:, mine], V[:, mine])
        ref = eng.unreorder(eng.attend(qt, kt, vt, [top_p[h] for h in mine], 8))
        res["steps"].append({"ok": bool(torch.equal(o, ref)), "owner": layer.last_owner,
                             "moves": layer.last_moves})
except RankLost as e:
    res["rank_lost"] = str(e)
print(json.dumps(res), flush=True)
os._exit(0)
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _run(world, leave_after=-1):
    port, sport = _free_port(), _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                   RANK=str(rank), SBA_ROOT=ROOT, STORE_PORT=str(sport), LEAVE_AFTER=str(leave_after))
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=120)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            pytest.fail("ranks did not finish")
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    return outs


def test_three_gloo_ranks_move_heavy_heads_and_return_their_outputs():
    outs = _run(3)
    for o in outs:
        assert len(o["steps"]) == 2
        for s in o["steps"]:
            assert s["ok"], o
    owner = outs[0]["steps"][0]["owner"]
    costs = [900, 50, 40, 30, 20, 10, 5]
    assert owner == lpt_placement(costs, 3)
    moves = [list(m) for m in migrations(owner, 3)]
    assert moves and outs[0]["steps"][0]["moves"] == moves
    assert all(o["steps"][0]["owner"] == owner for o in outs)


def test_a_rank_that_leaves_between_steps_is_reported_not_waited_for():
    outs = _run(3, leave_after=2)
    assert outs[2].get("left")
    for o in outs[:2]:
        assert len(o["steps"]) == 1 and o["steps"][0]["ok"]
        assert "rank_lost" in o and "[2]" in o["rank_lost"], o
