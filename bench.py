#!/usr/bin/env python
"""Benchmark of the block-sparse attention hot path on B200.

One step = the whole path on one batch: sba_reorder (q, k, v) ->
sba_build_mask -> sba_attention -> sba_unreorder, on the Wan-2.1-14B-480p
shaped layer (B=1, H=40, 21x30x52 latent grid = 32760 tokens, d=128, cubes
2x8x8, Top-p 0.9, Top-k 8, bf16, seeded synthetic Q/K/V).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline metric: effective TFLOPS over the selected blocks, F_tile = sum over
selected (row, key block) pairs of 4*bs^2*d, divided by the device time of a
whole step (all four calls). Under torchrun every rank runs its own replica of
the workload (weak scaling, no data-path collective); the time is the max over
ranks. `--impl reference` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn effective TFLOPS (selected blocks) & % BF16 peak; ms/call"
UNIT = "TFLOPS"
WORKLOAD = "wan"
L2_NOTE = "inputs (1.0 GB q/k/v) larger than the 126 MB L2, and L2 flushed by a 256 MiB write before every step (outside the timed events)"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sched-report", action="store_true")
    ap.add_argument("--no-lowbit", action="store_true", help="skip the low-bit P.V measurement")
    ap.add_argument("--no-sweep", action="store_true", help="skip the Top-p 0.4 / 0.5 / 0.7 report")
    ap.add_argument("--sched-workload", default="stress",
                    help="workload of the scheduler report (LPT persistent vs head-major grid)")
    ap.add_argument("--sched-reps", type=int, default=3, help="launches per schedule in that report")
    ap.add_argument("--report-all", action="store_true",
                    help="per-call timings, rooflines, density and SM idle for every workload "
                         "(one JSON line each; not the benchmark line)")
    ap.add_argument("--gen-device", choices=["gpu", "cpu"], default="gpu",
                    help="where the synthetic inputs are generated (cpu: no GPU launches "
                         "before the timed kernels, for profiler captures)")
    return ap.parse_args()


def _config(wl, extra=None):
    cfg = {"workload": f"{wl.name}: B={wl.B} H={wl.H} grid {wl.T}x{wl.Hh}x{wl.W} "
                       f"({wl.N} tokens) d={wl.d} cube {'x'.join(map(str, wl.cube))} "
                       f"top_p={','.join(str(p) for p in sorted(set(wl.top_p)))} top_k={wl.top_k}",
           "global_batch": wl.B, "seq_len": wl.N, "heads": wl.H, "head_dim": wl.d,
           "parallelism": "replicas", "l2": L2_NOTE}
    if extra:
        cfg.update(extra)
    return cfg


def _block_lens(wl):
    """Real tokens per block (for the valid-FLOP count): row-major over cubes,
    or, in Hilbert order, full blocks but the last."""
    ct, ch, cw = wl.cube
    if getattr(wl, "order", "cube") == "hilbert":
        bs, N = ct * ch * cw, wl.T * wl.Hh * wl.W
        nb = -(-N // bs)
        return [bs] * (nb - 1) + [N - (nb - 1) * bs]
    nT, nH, nW = -(-wl.T // ct), -(-wl.Hh // ch), -(-wl.W // cw)
    lens = []
    for tt in range(nT):
        for th in range(nH):
            for tw in range(nW):
                lens.append(min(ct, wl.T - tt * ct) * min(ch, wl.Hh - th * ch) * min(cw, wl.W - tw * cw))
    return lens


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0) or 0), float(d["hbm_gbs"]), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def _traffic_from_profile(kernel_src: str):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "attn_sm100_wan.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"source sha256:\s*([0-9a-f]{16,64})", text)
    m_bytes = re.search(r"dram bytes per launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes:
        return None
    cur = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
    if not cur.startswith(m_hash.group(1)):
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def dist_init(backend: str, device=None, timeout_s: int = 120):
    """Join the process group torchrun describes (no-op for one process).
    Returns the torch.distributed module or None."""
    ws, _, _ = _dist()
    if ws <= 1:
        return None
    import datetime

    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return dist


def max_over_ranks(value: float, pg, device="cpu") -> float:
    """Max of a per-rank scalar (timings are the slowest rank's)."""
    if pg is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def step_launches(B: int, H: int, nb: int) -> int:
    """Kernel launches of one step: reorder, attention and unreorder once each,
    and sba_build_mask's pooling, head scan and finalize once plus one score and
    one cut launch per chunk of heads (the library forms the fp64 pooled scores
    of as many heads at a time as 48 MiB hold, at least one)."""
    per_head = nb * nb * 8
    heads = max(1, max(per_head, 48 << 20) // per_head)
    chunks = -(-(B * H) // min(heads, B * H))
    return 3 + 3 + 2 * chunks


def whole_job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """Weak scaling: every rank processes its own replica; the job's rate is
    all ranks' FLOPs over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def _cpu_cores():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    threads = n
    try:
        from threadpoolctl import threadpool_info
        info = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            threads = max(info)
    except Exception:
        pass
    return n, threads


def cpu_oracle_sample(wl, q, k, v, heads=(0,), blocks_per_head=None, seed=0):
    """Time the fp64 oracle (reorder, routing, attention) on a bounded sample:
    the given heads in full (routing) and `blocks_per_head` query blocks of
    each (attention; all blocks when None). Returns (selected tile FLOPs,
    seconds, description)."""
    import numpy as np

    import oracle
    g = oracle.Geom(wl.T, wl.Hh, wl.W, *wl.cube)
    tp = wl.top_p_per_head()
    flops = 0.0
    secs = 0.0
    rng = np.random.default_rng(seed)
    for h in heads:
        Q, K, V = (x[:, h:h + 1].double().cpu().numpy() for x in (q, k, v))
        t0 = time.perf_counter()
        qt, kt, vt = oracle.reorder(Q, g), oracle.reorder(K, g), oracle.reorder(V, g)
        m = oracle.build_mask(qt, kt, g, [tp[h]], wl.top_k)
        if blocks_per_head is None:
            blocks = [(0, 0, i) for i in range(g.nb)]
        else:
            blocks = [(0, 0, int(i)) for i in rng.choice(g.nb, size=blocks_per_head, replace=False)]
        oracle.attention(qt, kt, vt, g, m["row_ptr"], m["col_idx"], blocks=blocks)
        secs += time.perf_counter() - t0
        flops += sum(int(m["row_cnt"][i]) for (_, _, i) in blocks) * 4.0 * g.bs * g.bs * wl.d
    nb = len(blocks)
    desc = (f"{len(heads)} head(s) of {wl.H}: reorder + routing of the whole head, attention on "
            f"{nb} of {g.nb} query blocks; fp64 numpy")
    return flops, secs, desc


def run_reference(args):
    ws, rank, local = _dist()
    if rank != 0:
        return 0
    import datagen
    wl = datagen.WORKLOADS[args.workload]
    q, k, v = datagen.generate(wl, seed=0, device="cpu")
    cores, threads = _cpu_cores()
    times, flops_tot = [], 0.0
    desc = ""
    for s in range(args.warmup + args.steps):
        f, sec, desc = cpu_oracle_sample(wl, q, k, v, heads=(s % wl.H,), blocks_per_head=8, seed=s)
        if s >= args.warmup:
            times.append(sec)
            flops_tot += f
    tot = sum(times)
    value = flops_tot / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def sm_idle_fraction(tr, nsm: int) -> float:
    """SM idle / tail fraction from per-row (start, end, smid) stamps:
    1 - sum over SMs of the time the SM had at least one row in flight /
    (SMs x makespan). Rows that overlap on one SM (the attention kernel runs
    two at once per CTA) count once."""
    import numpy as np
    tr = np.asarray(tr, dtype=np.int64).reshape(-1, 3)
    t0, t1 = int(tr[:, 0].min()), int(tr[:, 1].max())
    busy = 0
    for sm in np.unique(tr[:, 2]):
        iv = tr[tr[:, 2] == sm][:, :2]
        iv = iv[np.argsort(iv[:, 0], kind="stable")]
        cur_s, cur_e = int(iv[0, 0]), int(iv[0, 1])
        for s, e in iv[1:]:
            if s > cur_e:
                busy += cur_e - cur_s
                cur_s, cur_e = int(s), int(e)
            else:
                cur_e = max(cur_e, int(e))
        busy += cur_e - cur_s
    return 1.0 - busy / (nsm * float(t1 - t0))


def sched_report(dev, name="stress", reps=3):
    """SM idle / tail fraction of sba_attention on the heterogeneous-load
    workload, persistent longest-first vs a grid in head-major order (two rows
    per CTA), from per-row %globaltimer stamps (see sm_idle_fraction). Also
    the per-head spread of selected blocks."""
    import torch

    import block_sparse_attention_sba_b200 as sba
    import datagen
    wl = datagen.WORKLOADS[name]
    q, k, v = datagen.generate(wl, seed=0, device=dev)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube, order=wl.order)
    sa = sba.SparseAttention(plan, device=dev)
    h = plan.handle
    sba.sba_reorder(h, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace)
    sba.sba_build_mask(h, sa.qt, sa.kt, wl.top_p_per_head(), wl.top_k, sa.bitmask, sa.row_cnt,
                       sa.row_ptr, sa.col_idx, sa.work_order, sa.workspace)
    R = plan.info.rows
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    trace = torch.zeros(R * 3, dtype=torch.int64, device=dev)
    out = {"workload": name}
    for label, mode in (("lpt_persistent", sba.SBA_SCHED_LPT), ("head_major_grid", sba.SBA_SCHED_HEAD_MAJOR)):
        best = None
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sba.sba_attention(h, sa.qt, sa.kt, sa.vt, sa.row_ptr, sa.col_idx, sa.work_order, sa.ot,
                              sa.lse, mode, trace, sa.workspace)
            e1.record()
            torch.cuda.synchronize(dev)
            tr = trace.view(R, 3).cpu()
            span = float(int(tr[:, 1].max()) - int(tr[:, 0].min()))
            res = {"ms": e0.elapsed_time(e1), "idle_frac": sm_idle_fraction(tr.numpy(), nsm),
                   "makespan_ms": span * 1e-6, "sms_used": int(torch.unique(tr[:, 2]).numel())}
            if best is None or res["ms"] < best["ms"]:
                best = res
        out[label] = best
    cnt = sa.row_cnt.view(wl.B * wl.H, plan.info.nb).sum(dim=1).float()
    out["per_head_blocks_max_over_min"] = float(cnt.max() / cnt.min())
    out["density"] = float(sa.row_cnt.sum()) / (R * plan.info.nb)
    return out


def run_ours(args):
    import torch

    import block_sparse_attention_sba_b200 as sba
    import datagen

    ws, rank, local = _dist()
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = dist_init("nccl", dev)
    wl = datagen.WORKLOADS[args.workload]
    gen_dev = dev if args.gen_device == "gpu" else "cpu"
    q, k, v = datagen.generate(wl, seed=0, device=gen_dev, out_device=dev)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube, order=wl.order)
    sa = sba.SparseAttention(plan, device=dev)
    h = plan.handle
    o = torch.empty_like(q)
    top_p = wl.top_p_per_head()
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        sba.sba_reorder(h, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace, stream)
        if ev:
            ev[1].record(stream)
        sba.sba_build_mask(h, sa.qt, sa.kt, top_p, wl.top_k, sa.bitmask, sa.row_cnt, sa.row_ptr,
                           sa.col_idx, sa.work_order, sa.workspace, stream)
        if ev:
            ev[2].record(stream)
        sba.sba_attention(h, sa.qt, sa.kt, sa.vt, sa.row_ptr, sa.col_idx, sa.work_order, sa.ot,
                          sa.lse, sba.SBA_SCHED_LPT, None, sa.workspace, stream)
        if ev:
            ev[3].record(stream)
        sba.sba_unreorder(h, sa.ot, o, sa.workspace, stream)
        if ev:
            ev[4].record(stream)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    status = sa.check(stream)
    if status != 0:
        print(json.dumps({"error": f"device status {sba.sba_status_string(status)}"}))
        return 1

    gpu_id = str(local)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id)
    time.sleep(0.3)  # let the sampler start before the timed region
    for s in range(args.steps):
        flush.zero_()
        step(evs[s])
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    clocks = sampler.stop()
    per_call = {"reorder": [], "build_mask": [], "attention": [], "unreorder": []}
    step_ms = []
    for e in evs:
        per_call["reorder"].append(e[0].elapsed_time(e[1]))
        per_call["build_mask"].append(e[1].elapsed_time(e[2]))
        per_call["attention"].append(e[2].elapsed_time(e[3]))
        per_call["unreorder"].append(e[3].elapsed_time(e[4]))
        step_ms.append(e[0].elapsed_time(e[4]))
    mean_step = max_over_ranks(sum(step_ms) / len(step_ms), pg, dev)
    status = sa.check(stream)

    # selected-block FLOPs of one step
    rc = sa.row_cnt.cpu().tolist()
    cols = sa.col_idx[: int(sa.row_ptr[-1].item())].cpu().tolist()
    rp = sa.row_ptr.cpu().tolist()
    bs = plan.info.bs
    nnz = rp[-1]
    f_tile = 4.0 * bs * bs * wl.d * nnz
    lens = _block_lens(wl)
    nb = plan.info.nb
    f_valid = 0.0
    f_exec = 0.0
    for r in range(len(rc)):
        li = lens[r % nb]
        sel = cols[rp[r]:rp[r + 1]]
        f_valid += 4.0 * wl.d * li * sum(lens[j] for j in sel)
        # the kernel runs every query slot of the tile (M = 128) against the
        # key block's real length rounded up to 16 (N of S, K of P.V)
        f_exec += 4.0 * wl.d * bs * sum(-(-lens[j] // 16) * 16 for j in sel)
    density = nnz / (len(rc) * nb)

    peak, peak_sus, hbm, peak_kind = _peaks()
    attn_ms = statistics.mean(per_call["attention"])
    achieved = f_tile / (attn_ms * 1e-3) / 1e12
    traffic = _traffic_from_profile(os.path.join(ROOT, "block_sparse_attention_sba_b200", "csrc",
                                                 "attn_sm100.cu"))
    value = whole_job_tflops(f_tile, ws, mean_step)
    ms_calls = {k: round(statistics.mean(vv), 4) for k, vv in per_call.items()}
    overhead = (ms_calls["reorder"] + ms_calls["build_mask"] + ms_calls["unreorder"]) / ms_calls["attention"]

    # end to end through the public API with pinned host buffers: each step
    # copies its q, k, v in and its output back out. Copies run on two copy
    # streams (host->device, device->host) against the compute stream with two
    # device buffer sets, so step s+1's inputs and step s-1's output move while
    # step s computes.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        bufs = [tuple(torch.empty_like(x) for x in (q, k, v, o)) for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        n_e2e = max(4, min(args.steps, 12))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)

        def h2d(i):
            b = bufs[i % 2]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_done[i % 2])  # step i-2 no longer reads this set
                b[0].copy_(hq, non_blocking=True)
                b[1].copy_(hk, non_blocking=True)
                b[2].copy_(hv, non_blocking=True)
                ev_in[i % 2].record(h2d_s)

        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        e0.record(h2d_s)
        h2d(0)
        for i in range(n_e2e):
            b = bufs[i % 2]
            if i + 1 < n_e2e:
                h2d(i + 1)
            stream.wait_event(ev_in[i % 2])
            if i >= 2:
                stream.wait_event(ev_out[i % 2])  # step i-2's output has left this set
            sa(b[0], b[1], b[2], top_p, wl.top_k, o=b[3], stream=stream)
            ev_done[i % 2].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[i % 2])
                ho.copy_(b[3], non_blocking=True)
                ev_out[i % 2].record(d2h_s)
        e1.record(d2h_s)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, pg, dev)
        h2d_bytes = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
        e2e = {"value": whole_job_tflops(f_tile, ws, e2e_ms), "unit": UNIT,
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d_bytes,
               "d2h_bytes_per_step": ho.numel() * ho.element_size(),
               "steps": n_e2e, "copies": "overlapped with compute (two copy streams, two buffer sets)",
               "ratio_to_device_step": e2e_ms / mean_step}

    # the low-bit P.V path (E4M3 probabilities and values) on the same inputs:
    # informational, not the headline (reduced precision)
    lowbit = None
    if not args.no_lowbit and wl.dtype == "bf16" and wl.d == 128 and plan.info.bs == 128:
        ref_ot = sa.ot.float().clone()
        sa.lowbit(q, k, v, top_p, wl.top_k, o=o, stream=stream)
        torch.cuda.synchronize(dev)
        got = sa.ot.float()
        rel = float((got - ref_ot).norm() / ref_ot.norm())
        h = plan.handle
        t_s, t_a = [], []
        for _ in range(6):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            flush.zero_()
            ev[0].record(stream)
            sba.sba_smooth_v(h, sa.vt, sa.vq, sa.vmean, sa.vexp, sa.workspace, stream)
            ev[1].record(stream)
            sba.sba_attention_lowbit(h, sa.qt, sa.kt, sa.vq, sa.vmean, sa.vexp, sa.row_ptr,
                                     sa.col_idx, sa.work_order, sa.ot, sa.lse, None, sa.workspace,
                                     stream)
            ev[2].record(stream)
            torch.cuda.synchronize(dev)
            t_s.append(ev[0].elapsed_time(ev[1]))
            t_a.append(ev[1].elapsed_time(ev[2]))
        ms_a = statistics.mean(t_a[2:])
        lowbit = {"ms_smooth_v": round(statistics.mean(t_s[2:]), 4), "ms_attention": round(ms_a, 4),
                  "tflops_tile": f_tile / (ms_a * 1e-3) / 1e12,
                  "rel_l2_vs_bf16_output": rel,
                  "kernel": "attn_tc_kernel<128,128,1> (E4M3 P.V)"}

    sched = None
    if not args.no_sched_report:
        sched = sched_report(dev, args.sched_workload, args.sched_reps)

    # the same layer at lower Top-p (sparser routing): per-call ms, density,
    # overhead and attention TFLOPS (a report, not the headline)
    sweep = None
    if not args.no_sweep and wl.name == "wan":
        sweep = []
        for p_sw in (0.4, 0.5, 0.7):
            tp = [p_sw] * wl.H
            t = {"reorder": [], "build_mask": [], "attention": [], "unreorder": []}
            for it in range(3 + 5):
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
                flush.zero_()
                ev[0].record(stream)
                sba.sba_reorder(h, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace, stream)
                ev[1].record(stream)
                sba.sba_build_mask(h, sa.qt, sa.kt, tp, wl.top_k, sa.bitmask, sa.row_cnt, sa.row_ptr,
                                   sa.col_idx, sa.work_order, sa.workspace, stream)
                ev[2].record(stream)
                sba.sba_attention(h, sa.qt, sa.kt, sa.vt, sa.row_ptr, sa.col_idx, sa.work_order, sa.ot,
                                  sa.lse, sba.SBA_SCHED_LPT, None, sa.workspace, stream)
                ev[3].record(stream)
                sba.sba_unreorder(h, sa.ot, o, sa.workspace, stream)
                ev[4].record(stream)
                torch.cuda.synchronize(dev)
                if it >= 3:
                    for kk, (a0, a1) in zip(t, [(0, 1), (1, 2), (2, 3), (3, 4)]):
                        t[kk].append(ev[a0].elapsed_time(ev[a1]))
            nnz_sw = int(sa.row_ptr[-1].item())
            ms_sw = {kk: round(statistics.mean(vv), 4) for kk, vv in t.items()}
            sweep.append({"top_p": p_sw, "density": nnz_sw / (len(rc) * nb), "ms_per_call": ms_sw,
                          "overhead_frac": (ms_sw["reorder"] + ms_sw["build_mask"] + ms_sw["unreorder"])
                          / ms_sw["attention"],
                          "attention_tflops_tile": 4.0 * bs * bs * wl.d * nnz_sw
                          / (ms_sw["attention"] * 1e-3) / 1e12})
        assert sa.check(stream) == 0

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cores, threads = _cpu_cores()
        f, sec, desc = cpu_oracle_sample(wl, q, k, v, heads=(0,), blocks_per_head=None)
        cpu = {"value": f / sec / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc + f"; {sec:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": mean_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": _config(wl),
            "routing": {"density": round(density, 4), "nnz_blocks": nnz, "sched": "lpt-persistent"},
            "ms_per_call": ms_calls,
            "attention": {"tflops_tile": achieved,
                          "tflops_valid": f_valid / (attn_ms * 1e-3) / 1e12,
                          "tflops_executed": f_exec / (attn_ms * 1e-3) / 1e12,
                          "valid_over_executed": f_valid / f_exec,
                          "frac_of_peak": achieved / peak, "peak_kind": peak_kind,
                          "frac_of_sustained_peak": achieved / peak_sus if peak_sus else None},
            "overhead_frac": overhead,
            "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel<128,128>",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_flops_per_launch": f_tile},
            "scheduler": sched, "lowbit": lowbit, "sparsity_sweep": sweep,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": step_launches(wl.B, wl.H, nb) * args.steps,
            "clocks": clocks, "device_status": sba.sba_status_string(status),
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def _alg_bytes(wl, info):
    """Algorithmic HBM bytes of reorder (q,k,v), mask (reads qt, kt) and unreorder."""
    e = 4 if wl.dtype == "f32" else 2
    bh = wl.B * wl.H
    row = wl.d * e
    reorder = 3 * bh * (wl.N + info.Npad) * row
    mask = 2 * bh * info.Npad * row
    unreorder = bh * (info.Npad + wl.N) * row
    return reorder, mask, unreorder


def report_all(args):
    """One JSON line per workload: per-call ms, effective TFLOPS (tile and
    real-token FLOPs), fraction of the measured bf16 peak, HBM fractions of
    the three bandwidth-bound calls, density and SM idle for both schedules."""
    import torch

    import block_sparse_attention_sba_b200 as sba
    import datagen
    dev = torch.device("cuda", 0)
    peak, peak_sus, hbm, kind = _peaks()
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for name in ["tiny", "small", "wan", "hunyuan", "stress", "wan_hilbert"]:
        wl = (datagen.with_order(datagen.WORKLOADS["wan"], "hilbert") if name == "wan_hilbert"
              else datagen.WORKLOADS[name])
        q, k, v = datagen.generate(wl, seed=0, device=dev)
        plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube, order=wl.order)
        sa = sba.SparseAttention(plan, device=dev)
        h = plan.handle
        o = torch.empty_like(q)
        tp = wl.top_p_per_head()
        R = plan.info.rows
        trace = torch.zeros(R * 3, dtype=torch.int64, device=dev)
        calls = {"reorder": [], "build_mask": [], "attention": [], "unreorder": []}
        steps = 10
        for it in range(3 + steps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            flush.zero_()
            ev[0].record()
            sba.sba_reorder(h, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace)
            ev[1].record()
            sba.sba_build_mask(h, sa.qt, sa.kt, tp, wl.top_k, sa.bitmask, sa.row_cnt, sa.row_ptr,
                               sa.col_idx, sa.work_order, sa.workspace)
            ev[2].record()
            sba.sba_attention(h, sa.qt, sa.kt, sa.vt, sa.row_ptr, sa.col_idx, sa.work_order, sa.ot,
                              sa.lse, sba.SBA_SCHED_LPT, None, sa.workspace)
            ev[3].record()
            sba.sba_unreorder(h, sa.ot, o, sa.workspace)
            ev[4].record()
            torch.cuda.synchronize(dev)
            if it >= 3:
                for i, key in enumerate(calls):
                    calls[key].append(ev[i].elapsed_time(ev[i + 1]))
        ms = {key: statistics.mean(val) for key, val in calls.items()}
        nnz = int(sa.row_ptr[-1].item())
        rc = sa.row_cnt.cpu().tolist()
        rp = sa.row_ptr.cpu().tolist()
        cols = sa.col_idx[:nnz].cpu().tolist()
        lens = _block_lens(wl)
        nb = plan.info.nb
        f_tile = 4.0 * plan.info.bs ** 2 * wl.d * nnz
        f_valid = sum(4.0 * wl.d * lens[r % nb] * sum(lens[j] for j in cols[rp[r]:rp[r + 1]])
                      for r in range(R))
        idle = {}
        for label, mode in (("lpt", sba.SBA_SCHED_LPT), ("head_major", sba.SBA_SCHED_HEAD_MAJOR)):
            sba.sba_attention(h, sa.qt, sa.kt, sa.vt, sa.row_ptr, sa.col_idx, sa.work_order, sa.ot,
                              sa.lse, mode, trace, sa.workspace)
            torch.cuda.synchronize(dev)
            tr = trace.view(R, 3).cpu()
            idle[label] = sm_idle_fraction(tr.numpy(), nsm)
        rb, mb, ub = _alg_bytes(wl, plan.info)
        att_s = ms["attention"] * 1e-3
        line = {"workload": name, "dtype": wl.dtype, "ms": {k2: round(v2, 4) for k2, v2 in ms.items()},
                "tflops_tile": f_tile / att_s / 1e12, "tflops_valid": f_valid / att_s / 1e12,
                "frac_bf16_peak": f_tile / att_s / 1e12 / peak,
                "hbm_frac": {"reorder": rb / (ms["reorder"] * 1e-3) / 1e9 / hbm,
                             "build_mask": mb / (ms["build_mask"] * 1e-3) / 1e9 / hbm,
                             "unreorder": ub / (ms["unreorder"] * 1e-3) / 1e9 / hbm},
                "overhead_frac": (ms["reorder"] + ms["build_mask"] + ms["unreorder"]) / ms["attention"],
                "density": nnz / (R * nb), "sm_idle": idle,
                "per_head_blocks_max_over_min": float(
                    sa.row_cnt.view(wl.B * wl.H, nb).sum(1).max() / sa.row_cnt.view(wl.B * wl.H, nb).sum(1).min()),
                "status": sba.sba_status_string(sa.check())}
        print(json.dumps(line), flush=True)
        del q, k, v, sa, o, trace
        torch.cuda.empty_cache()
    return 0


def main():
    args = _args()
    if args.report_all:
        return report_all(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
