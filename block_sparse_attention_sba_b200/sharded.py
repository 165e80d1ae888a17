"""Head-sharded block-sparse attention over several GPUs, with longest-first
head placement (FVAttn: Adaptive Sparse Attention with Runtime Load Balancing
for Video Generation, abstract and reviews: adaptive Top-p routing leaves
heads with very different workloads, so heads are placed by their routed cost
and heavy heads migrate between ranks).

An opt-in layer above the single-GPU calls; it changes none of them. One
process per GPU (torch.distributed). Every step:

1. each rank reorders its own heads (a static split: head h starts on rank
   h mod world) and routes them (Top-p mask); a head's cost is its number of
   selected (row, key block) pairs;
2. the costs are all-gathered and every rank computes the same longest-first
   placement: heads by cost, descending (ties: lower head first), each onto
   the rank with the least cost so far (ties: lower rank);
3. a head whose placement differs from its start moves: its reordered q, k, v
   go from the start rank to the placed rank by point-to-point send/recv;
4. each rank runs the routing and attention on the heads it now holds (a
   moved head is routed again where it lands: routing is deterministic, so the
   mask is the one its cost came from, and no mask crosses the link);
5. outputs of moved heads go back to their start rank, which unreorders its
   heads.

Only plain point-to-point transfers and one small all-gather are used (no
multicast); no library kernel is given another GPU's memory. Before every
step the ranks check in through the store: a rank that left between steps is
reported as an error on the others before any collective runs (the process
group's own timeout bounds the rest).

The per-rank work goes through an engine object with four calls
(``reorder``, ``route_cost``, ``attend``, ``unreorder``); ``LibraryEngine``
binds them to the CUDA library.
"""
from __future__ import annotations

import datetime
from typing import Dict, List, Optional, Sequence, Tuple


class RankLost(RuntimeError):
    """A rank did not check in before a step."""


def lpt_placement(costs: Sequence[int], world: int) -> List[int]:
    """Owner rank of every head: longest processing time first. Heads sorted
    by cost descending (ties: lower head first); each goes to the rank whose
    assigned cost is smallest (ties: lower rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda h: (-int(costs[h]), h))
    load = [0] * world
    owner = [0] * len(costs)
    for h in order:
        r = min(range(world), key=lambda x: (load[x], x))
        owner[h] = r
        load[r] += int(costs[h])
    return owner


def static_heads(H: int, world: int, rank: int) -> List[int]:
    """Heads a rank starts with: h mod world == rank."""
    return [h for h in range(H) if h % world == rank]


def migrations(owner: Sequence[int], world: int) -> List[Tuple[int, int, int]]:
    """(head, source rank, destination rank) of every head that moves, in
    head order."""
    return [(h, h % world, r) for h, r in enumerate(owner) if r != h % world]


class LibraryEngine:
    """The per-rank calls on this rank's GPU through the CUDA library: plans
    are made per head count and kept."""

    def __init__(self, B: int, T: int, Hh: int, W: int, d: int, cube, device, dtype="bf16",
                 order: str = "cube"):
        import torch

        from . import Plan, SparseAttention
        self._Plan, self._SA = Plan, SparseAttention
        self.B, self.T, self.Hh, self.W, self.d, self.cube = B, T, Hh, W, d, tuple(cube)
        self.dtype, self.order = dtype, order
        self.device = torch.device(device)
        self._cache: Dict[int, object] = {}

    def _sa(self, nheads: int):
        if nheads not in self._cache:
            plan = self._Plan(self.B, nheads, self.T, self.Hh, self.W, self.d, self.cube, self.dtype,
                              order=self.order)
            self._cache[nheads] = self._SA(plan, device=self.device)
        return self._cache[nheads]

    def reorder(self, q, k, v):
        """Raster [B, h, N, d] -> cube order [B, h, Npad, d] (new tensors)."""
        from . import sba_reorder
        sa = self._sa(q.shape[1])
        q, k, v = (x.contiguous() for x in (q, k, v))  # the plans assume [B, h, N, d] storage
        sba_reorder(sa.plan.handle, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace)
        return sa.qt.clone(), sa.kt.clone(), sa.vt.clone()

    def route_cost(self, qt, kt, top_p: Sequence[float], top_k: int):
        """Selected (row, key block) pairs of every head, int64 [h] on the GPU."""
        from . import sba_build_mask
        sa = self._sa(qt.shape[1])
        sba_build_mask(sa.plan.handle, qt, kt, list(top_p), top_k, sa.bitmask, sa.row_cnt,
                       sa.row_ptr, sa.col_idx, sa.work_order, sa.workspace)
        nb = sa.plan.info.nb
        return sa.row_cnt.view(self.B, qt.shape[1], nb).sum(dim=(0, 2)).long()

    def attend(self, qt, kt, vt, top_p: Sequence[float], top_k: int):
        """Routing and attention of the held heads; returns ot (cube order)."""
        from . import SBA_SCHED_LPT, sba_attention, sba_build_mask
        sa = self._sa(qt.shape[1])
        h = sa.plan.handle
        sba_build_mask(h, qt, kt, list(top_p), top_k, sa.bitmask, sa.row_cnt, sa.row_ptr,
                       sa.col_idx, sa.work_order, sa.workspace)
        sba_attention(h, qt, kt, vt, sa.row_ptr, sa.col_idx, sa.work_order, sa.ot, sa.lse,
                      SBA_SCHED_LPT, None, sa.workspace)
        return sa.ot.clone()

    def unreorder(self, ot):
        """Cube order -> raster [B, h, N, d]."""
        import torch

        from . import sba_unreorder
        sa = self._sa(ot.shape[1])
        o = torch.empty(self.B, ot.shape[1], self.T * self.Hh * self.W, self.d, dtype=ot.dtype,
                        device=ot.device)
        sba_unreorder(sa.plan.handle, ot, o, sa.workspace)
        return o


class HeadShardedAttention:
    """One rank's part of the head-sharded layer (see the module docstring).

    ``pg`` is the process group (NCCL for GPUs, gloo in CPU tests); ``store``
    (optional) is the key-value store every rank can reach, used for the
    check-in before each step, with ``checkin_timeout_s``."""

    def __init__(self, engine, H: int, pg, store=None, checkin_timeout_s: float = 10.0):
        import torch.distributed as dist
        self.engine = engine
        self.H = H
        self.pg = pg
        self.world = dist.get_world_size(pg)
        self.rank = dist.get_rank(pg)
        if H < self.world:
            raise ValueError(f"{H} heads on {self.world} ranks: every rank must start with a head")
        self.store = store
        self.checkin_timeout = datetime.timedelta(seconds=checkin_timeout_s)
        self.step_no = 0
        self.last_owner: Optional[List[int]] = None
        self.last_moves: List[Tuple[int, int, int]] = []

    def my_heads(self) -> List[int]:
        return static_heads(self.H, self.world, self.rank)

    def _checkin(self):
        if self.store is None:
            return
        key = f"sba/step{self.step_no}/rank"
        self.store.set(f"{key}{self.rank}", "1")
        keys = [f"{key}{r}" for r in range(self.world)]
        try:
            self.store.wait(keys, self.checkin_timeout)
        except Exception as e:  # the store raises on timeout
            missing = []
            for r, k in enumerate(keys):
                try:
                    self.store.wait([k], datetime.timedelta(milliseconds=1))
                except Exception:
                    missing.append(r)
            raise RankLost(f"step {self.step_no}: ranks {missing} did not check in") from e

    def __call__(self, q, k, v, top_p: Sequence[float], top_k: int):
        """q, k, v: this rank's heads (``my_heads()``), raster [B, h, N, d].
        top_p: one value per global head. Returns this rank's output heads."""
        import torch
        import torch.distributed as dist
        self._checkin()
        mine = self.my_heads()
        if q.shape[1] != len(mine):
            raise ValueError(f"rank {self.rank} holds heads {mine}, got {q.shape[1]}")
        qt, kt, vt = self.engine.reorder(q, k, v)
        cost_mine = self.engine.route_cost(qt, kt, [top_p[h] for h in mine], top_k)
        # all costs, in global head order
        width = (self.H + self.world - 1) // self.world
        buf = torch.full((width,), -1, dtype=torch.int64, device=cost_mine.device)
        buf[:len(mine)] = cost_mine
        gathered = [torch.empty_like(buf) for _ in range(self.world)]
        dist.all_gather(gathered, buf, group=self.pg)
        costs = [0] * self.H
        for r in range(self.world):
            for i, h in enumerate(static_heads(self.H, self.world, r)):
                costs[h] = int(gathered[r][i])
        owner = lpt_placement(costs, self.world)
        moves = migrations(owner, self.world)
        self.last_owner, self.last_moves = owner, moves
        # move the reordered q, k, v of migrating heads (sends and receives in
        # head order, the same on every rank)
        held: Dict[int, Tuple] = {h: (qt[:, i], kt[:, i], vt[:, i]) for i, h in enumerate(mine)
                                  if owner[h] == self.rank}
        ops = []
        for h, src, dst in moves:
            if src == self.rank:
                i = mine.index(h)
                for t in (qt, kt, vt):
                    ops.append(dist.P2POp(dist.isend, t[:, i].contiguous(), dst, group=self.pg))
            elif dst == self.rank:
                recv = tuple(torch.empty_like(qt[:, 0]) for _ in range(3))
                for t in recv:
                    ops.append(dist.P2POp(dist.irecv, t, src, group=self.pg))
                held[h] = recv
        for req in (dist.batch_isend_irecv(ops) if ops else []):
            req.wait()
        # attention on the held heads (head order)
        hs = sorted(held)
        out_by_head: Dict[int, object] = {}
        if hs:
            hq = torch.stack([held[h][0] for h in hs], dim=1)
            hk = torch.stack([held[h][1] for h in hs], dim=1)
            hv = torch.stack([held[h][2] for h in hs], dim=1)
            ot = self.engine.attend(hq, hk, hv, [top_p[h] for h in hs], top_k)
            out_by_head = {h: ot[:, i] for i, h in enumerate(hs)}
        # outputs of moved heads go back to their start rank
        ops = []
        back: Dict[int, object] = {}
        for h, src, dst in moves:
            if dst == self.rank:
                ops.append(dist.P2POp(dist.isend, out_by_head[h].contiguous(), src, group=self.pg))
            elif src == self.rank:
                back[h] = torch.empty_like(qt[:, 0])
                ops.append(dist.P2POp(dist.irecv, back[h], dst, group=self.pg))
        for req in (dist.batch_isend_irecv(ops) if ops else []):
            req.wait()
        out_by_head.update(back)
        ot_mine = torch.stack([out_by_head[h] for h in mine], dim=1)
        self.step_no += 1
        return self.engine.unreorder(ot_mine)
