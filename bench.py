"""Benchmark of the HARD-KV decode step (one attention layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path (append, condense on block steps, score +
calibration + top-p, regularize fused with attention, combine) over one batch of
synthetic input, replayed from the same starting cache state so every timed step is
the workload's single decode step. Each step is one CUDA-graph replay timed with CUDA
events on the launching stream; L2 is flushed before every timed step, outside the
timed events: a 2 x L2 buffer is written and then read back, so no line of the
previous step survives and the flush's own dirty lines are written back before the
timed region starts (the L2 is left holding clean lines of the flush buffer). `e2e`
repeats the measurement through the host-buffer C entry point
(hardkv_decode_step_host: pinned H2D of q / k_new / v_new, the step, D2H of the output). With --gpus N (torchrun) every rank runs an independent replica of
the workload on its own GPU (no collective in the step) and the step time is the max
over ranks.

`--impl reference` times the fp64 CPU oracle as it stands, on this host's cores, on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode tokens/s at batch×ctx; HBM GB/s as % of B200 peak"
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0
STAGES = ("append", "condense", "score", "topp", "attend")
# --path unfused: the step as its standalone calls; "select" is one call (score + top-p)
UNFUSED_STAGES = ("append", "condense", "select", "regularize", "attend")
KERNEL_OF_STAGE = {"append": "append_kernel", "condense": "condense_kernel",
                   "score": "score_tma_kernel", "topp": "topp_kernel",
                   "regularize": "compact_kernel", "attend": "attend_ws_kernel"}


# ----------------------------------------------------------------------------- helpers

def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def csrc_digest() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "attention_kv_head_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str, path: str = "fused"):
    """DRAM bytes per launch from a committed ncu capture of the current sources (of the
    same workload and the same path: fused step or standalone calls)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(kernel)
        if (e and e.get("csrc_sha") == csrc_digest() and e.get("workload") == workload
                and e.get("path", "fused") == path):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons (NVML) while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period, self.samples = index, period_s, []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        busy = [m for m, r in self.samples if not (r & 0x1)] or [m for m, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_max(x: float, world: int, device=None) -> float:
    """Max of a float over ranks (identity when not distributed)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_tokens_per_s(world: int, batch: int, max_step_ms: float) -> float:
    """Whole-job throughput: every rank decodes one token for each of its `batch`
    sequences per step; the job's step time is the slowest rank's."""
    return world * batch / (max_step_ms * 1e-3)


# ----------------------------------------------------------------------------- bytes

def step_bytes(w, st: dict, fused: bool = True) -> dict:
    """Bytes one decode step must move (reads + writes), per stage, from the device state
    after the step: `st` holds len / d_lo / s_lo / moved [B], n_kept / sp_mode [B,H],
    live [B,H] (kept rows whose position is still Sparse) and `reselect` [B] (sequences
    that scored and selected in this step). fused = False: the step as its standalone
    calls (stages append, condense, select, regularize, attend; unfused_bytes).

      append    k_new, v_new read; their ring rows written
      condense  per unit of a moved sequence (MERGE): the block's K/V and the C slots'
                K/V read, the merged slots written back (the survey's (Blk + 2C) 2 d e)
      score     per reselecting unit: its L candidate keys and G queries read, L fp32
                scores written
      topp      per reselecting unit: L scores read, the mask words and the Cap-long
                flattened index written
      attend    per unit: kept rows (gathered from the ring and, under Rewrite Cache,
                written to the compact layout in a reselecting step; otherwise read from
                the compact layout or the ring), their index, the Dense and Condensed
                rows, the Condensed weights, q and the fp32 output"""
    if not fused:
        return unfused_bytes(w, st)
    e = 2 if w.dtype == "bf16" else 4
    d, H, G, C = w.head_dim, w.n_kv_heads, w.group, w.condensed_slots
    row = 2 * d * e                                             # one K row + one V row
    Ls = (st["d_lo"] - st["s_lo"]).astype(np.int64)            # per sequence
    dense = (st["len"] - st["d_lo"]).astype(np.int64)
    resel = st["reselect"].astype(bool)
    moved = st["moved"].astype(bool)
    n = st["n_kept"].astype(np.int64)
    live = st["live"].astype(np.int64)
    rw = st["sp_mode"].astype(bool)
    U = w.batch * H
    q_bytes = w.batch * w.n_q_heads * d * e
    Lsel = int(Ls[resel].sum()) * H
    kept_sel = int(n[resel].sum())
    gather_rw = int((n * (resel[:, None] & rw)).sum())          # gathered + written
    gather_ld = int((n * (resel[:, None] & ~rw)).sum())         # gathered, not written
    later = int((live * ~resel[:, None]).sum())                 # read again, either layout
    by = {
        "append": 2 * U * d * e * 2,
        "condense": (int(moved.sum()) * H * (w.block + 2 * C) * row
                     if w.condense_mode == 1 else 0),
        "score": Lsel * d * e + int(resel.sum()) * H * G * d * e + Lsel * 4,
        "topp": Lsel * 4 + int(((Ls[resel] + 31) // 32).sum()) * H * 4
                + int(resel.sum()) * H * w.sparse_cap * 4,
        "attend": 2 * gather_rw * row + gather_ld * row + later * row + int(n.sum()) * 4
                  + (int(dense.sum()) * H + U * C) * row + U * C * 4 + q_bytes
                  + w.batch * w.n_q_heads * d * 4,
    }
    by["total"] = sum(by.values())
    by["sum_kept"] = kept_sel
    by["kept_fraction"] = kept_sel / max(Lsel, 1)
    return by


def unfused_bytes(w, st: dict) -> dict:
    """step_bytes of the step as its standalone calls: the selection writes only the mask
    (the index comes from the compaction), the compaction reads each reselecting unit's
    mask and writes its Cap-long index and, under Rewrite Cache, reads its kept rows
    from the ring and writes them to the compact layout, and the attention then reads
    every kept row once (compact rows, or ring rows through the index)."""
    e = 2 if w.dtype == "bf16" else 4
    d, H, G, C = w.head_dim, w.n_kv_heads, w.group, w.condensed_slots
    row = 2 * d * e
    Ls = (st["d_lo"] - st["s_lo"]).astype(np.int64)
    dense = (st["len"] - st["d_lo"]).astype(np.int64)
    resel = st["reselect"].astype(bool)
    moved = st["moved"].astype(bool)
    n = st["n_kept"].astype(np.int64)
    live = st["live"].astype(np.int64)
    rw = st["sp_mode"].astype(bool)
    U = w.batch * H
    Lsel = int(Ls[resel].sum()) * H
    words = int(((Ls[resel] + 31) // 32).sum()) * H * 4
    kept_sel = int(n[resel].sum())
    rewritten = int((n * (resel[:, None] & rw)).sum())
    by = {
        "append": 2 * U * d * e * 2,
        "condense": (int(moved.sum()) * H * (w.block + 2 * C) * row
                     if w.condense_mode == 1 else 0),
        "select": Lsel * d * e + int(resel.sum()) * H * G * d * e + Lsel * 4   # score
                  + Lsel * 4 + words,                                            # top-p
        "regularize": words + int(resel.sum()) * H * w.sparse_cap * 4 + 2 * rewritten * row,
        "attend": (kept_sel + int((live * ~resel[:, None]).sum())) * row + int(n.sum()) * 4
                  + (int(dense.sum()) * H + U * C) * row + U * C * 4
                  + w.batch * w.n_q_heads * d * e + w.batch * w.n_q_heads * d * 4,
    }
    by["total"] = sum(by.values())
    by["sum_kept"] = kept_sel
    by["kept_fraction"] = kept_sel / max(Lsel, 1)
    return by


def sum_bytes(per_step: list) -> dict:
    keys = [k for k in per_step[0] if k != "kept_fraction"]
    out = {k: sum(b[k] for b in per_step) for k in keys}
    sel_L = sum(b["sum_kept"] / b["kept_fraction"] for b in per_step if b["kept_fraction"] > 0)
    out["kept_fraction"] = out["sum_kept"] / sel_L if sel_L else 0.0
    return out


# ----------------------------------------------------------------------------- GPU arm

# Tensors of the cache state a replay starts from (the fused step changes all of them).
STATE_TENSORS = ("len", "d_lo", "s_lo", "moved", "n_kept", "sp_mode", "sp_idx", "k_cd", "v_cd",
                 "w_cd", "k_sp", "v_sp", "k_pool", "v_pool", "blk_tab", "blk_cnt", "free_list",
                 "ret_list", "pool_ctl")


def run_gpu(args, world, rank, local) -> dict:
    import torch

    from attention_kv_head_b200 import binding as Bn
    from attention_kv_head_b200 import build as Bd
    from attention_kv_head_b200 import synth
    from attention_kv_head_b200.cache import DecodeCache

    Bd.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload].with_(seed=rank)
    if args.p is not None:
        w = w.with_(p=args.p)
    st = synth.initial_state(w)
    # --paged: the compact rows in one pool of 16-row blocks with per-head block tables,
    # sized so that no head can run short (B*H*ceil(Cap/16) blocks)
    pool = w.batch * w.n_kv_heads * (-(-w.sparse_cap // Bn.PAGE_ROWS)) if args.paged else None
    dc = DecodeCache.from_state(st, device=dev, pool_blocks=pool)
    p = synth.p_values(w)[0]
    N = args.window or w.select_every                 # decode steps per timed replay
    on_move = w.select_every > 1                      # sequences reselect on their block move
    first = args.first_step if args.first_step >= 0 else (1 if on_move else 0)
    sel = {}
    if args.rule == "topk":
        k_sel = args.top_k
        if k_sel <= 0:   # the fixed budget that keeps as many rows as calibrated top-p
            q0, _ = synth.queries(w, 0)
            k0, _, v0, _ = synth.step_kv(w, st.lens, 0)
            probe = DecodeCache.from_state(st, device=dev)
            o0 = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dev)
            probe.step(probe.to_dev(q0), probe.to_dev(k0), probe.to_dev(v0), o0, p)
            k_sel = max(1, int(round(float(probe.n_kept.float().mean()))))
            del probe
        sel.update(rule=Bn.RULE_TOPK, top_k=k_sel)
    if args.calibration == "entropy":
        sel.update(calibration=Bn.CAL_ENTROPY)
    if args.layout != "rewrite":
        sel["layout"] = Bn.LayoutPolicy(
            Bn.LAYOUT_SPARSE_LOAD if args.layout == "sparse" else Bn.LAYOUT_MTI, -1,
            args.l_lower, args.l_upper, args.gather_surcharge)
    inputs = []
    for t in range(first, first + N):
        qraw, _ = synth.queries(w, t)
        kr, _, vr, _ = synth.step_kv(w, st.lens, t)
        inputs.append(tuple(dc.to_dev(x) for x in (qraw, kr, vr)))
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dev)
    mask = dc.new_mask()
    mode = Bn.SELECT_MOVED if on_move else Bn.SELECT_ALL
    stream = torch.cuda.Stream(device=dev)
    # untimed steps before the window (the first selects every sequence, so a workload
    # that reselects on block moves starts the window with every head holding a selection)
    for t in range(first):
        qs, _ = synth.queries(w, t)
        ks, _, vs, _ = synth.step_kv(w, st.lens, t)
        with torch.cuda.stream(stream):
            dc.step(dc.to_dev(qs), dc.to_dev(ks), dc.to_dev(vs), out, p, mask=mask, stream=stream,
                    select_mode=Bn.SELECT_ALL if t == 0 else mode, **sel)
        stream.synchronize()
    snap = {n_: getattr(dc, n_).clone() for n_ in STATE_TENSORS if getattr(dc, n_) is not None}

    def restore():
        for n_, t_ in snap.items():
            getattr(dc, n_).copy_(t_)

    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        flush.zero_()                      # write 2 x L2 ...
        flush.view(torch.int32).sum()      # ... then read it back: clean lines only

    # external: recorded during graph capture (by the library, or by unfused_step) they
    # become event-record nodes that keep their timestamps
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(Bn.STEP_EVENTS)]
           for _ in range(N)]
    # the timed graph records one event before the window's first kernel and one after
    # its last (graph-launch latency stays outside the timed region)
    ends = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    edge = [[ends[0] if (t == 0 and i == 0) else
             ends[1] if (t == N - 1 and i == Bn.STEP_EVENTS - 1) else None
             for i in range(Bn.STEP_EVENTS)] for t in range(N)]

    fused = args.path == "fused"
    stages = STAGES if fused else UNFUSED_STAGES

    def select_call(q):
        """The selection as one standalone call (score + calibration + top-p or top-k)."""
        if "top_k" in sel:
            dc.score_topk(q, sel["top_k"], mask, select_mode=mode, stream=stream)
        elif sel.get("calibration") == Bn.CAL_ENTROPY:
            dc.score_calibrate_entropy_topp(q, p, mask, select_mode=mode, stream=stream)
        else:
            dc.score_calibrate_topp(q, p, mask, select_mode=mode, stream=stream)

    def unfused_step(q, k, v, ev):
        """One decode step as the standalone calls; ev[i] (or None) recorded before call i
        and ev[5] after the last, like the fused step's stage events."""
        def rec(i):
            if ev is not None and ev[i] is not None:
                ev[i].record(stream)
        rec(0)
        dc.append(k, v, stream=stream)
        rec(1)
        dc.condense(stream=stream)
        rec(2)
        select_call(q)
        rec(3)
        dc.regularize(mask, select_mode=mode, stream=stream, layout=sel.get("layout"))
        rec(4)
        dc.decode_attn(q, out, stream=stream)
        rec(5)

    def window(events=None):
        for t, (q, k, v) in enumerate(inputs):
            if fused:
                dc.step(q, k, v, out, p, mask=mask, select_mode=mode, stream=stream,
                        events=events[t] if events else None, **sel)
            else:
                unfused_step(q, k, v, events[t] if events else None)

    # algorithmic bytes of every step of the window, from the device state after it
    per_step = []
    pool_held = 0   # paged tier: most blocks the heads held after any step of the window
    with torch.cuda.stream(stream):
        for row in evs + [ends]:
            for e_ in row:
                e_.record(stream)                  # create the CUDA events
        restore()
        for t, (q, k, v) in enumerate(inputs):
            if fused:
                dc.step(q, k, v, out, p, mask=mask, select_mode=mode, stream=stream, **sel)
            else:
                unfused_step(q, k, v, None)
            stream.synchronize()
            cur = {n_: getattr(dc, n_).cpu().numpy() for n_ in ("len", "d_lo", "s_lo", "moved", "n_kept",
                                                               "sp_mode", "sp_idx")}
            cur["reselect"] = cur["moved"] if on_move else np.ones(w.batch, bool)
            cur["live"] = ((cur["sp_idx"] >= cur["s_lo"][:, None, None]) &
                           (np.arange(w.sparse_cap)[None, None, :] < cur["n_kept"][:, :, None])).sum(-1)
            per_step.append(step_bytes(w, cur, fused=fused))
            if dc.blk_cnt is not None:
                pool_held = max(pool_held, int(dc.blk_cnt.sum().item()))
        by = sum_bytes(per_step)
        for _ in range(2):                         # eager warm-up (sets kernel attributes)
            restore()
            window(events=evs)
    stream.synchronize()
    # `g` is the timed window (event nodes only at its two ends); `gp` the same window
    # with event nodes between the stages (an event node between two kernels adds ~2.6 us
    # and breaks their launch overlap, so those stay out of the timed graph)
    g = torch.cuda.CUDAGraph()
    restore()
    with torch.cuda.graph(g, stream=stream):
        window(events=edge)
    gp = torch.cuda.CUDAGraph()
    restore()
    with torch.cuda.graph(gp, stream=stream):
        window(events=evs)
    kernels_per_step = 4 + (1 if w.condense_mode == synth.MERGE else 0)
    if not fused:   # + the compaction (and, on the paged tier, the pool merge and allocation)
        kernels_per_step += 1 + (2 if args.paged else 0)

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)

    def one(graph):
        """Replays `graph` from the starting state after an L2 flush; returns (ms between
        the graph's own first and last event nodes, ms around the replay call)."""
        with torch.cuda.stream(stream):
            restore()
            flush_l2()
            t0.record(stream)
            graph.replay()
            t1.record(stream)
        stream.synchronize()
        return ends[0].elapsed_time(ends[1]), t0.elapsed_time(t1)

    for _ in range(args.warmup):
        one(g)
        one(gp)
    win_ms, outer_ms, stage_ms = [], [], []
    dist_barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            a_, b_ = one(g)
            win_ms.append(a_)
            outer_ms.append(b_)
        for _ in range(args.steps):  # stage durations from the event-node replay
            one(gp)
            stage_ms.append([sum(evs[t][i].elapsed_time(evs[t][i + 1]) for t in range(N))
                             for i in range(len(stages))])
    torch.cuda.synchronize()
    dist_barrier(world)
    mean_ms = float(np.mean(win_ms)) / N              # per decode step
    max_ms = dist_max(mean_ms, world, dev)
    stage_mean = {s: float(np.mean([x[i] for x in stage_ms])) / N for i, s in enumerate(stages)}

    # e2e through the host-buffer entry point (every step's inputs copied in, output out)
    host_in = [tuple(t.cpu().pin_memory() for t in x) for x in inputs]
    oh = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        with torch.cuda.stream(stream):
            restore()
            flush_l2()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for t, (qh, kh, vh) in enumerate(host_in):
                if fused:
                    dc.step_host(qh, kh, vh, oh, p, mask=mask, select_mode=mode, stream=stream,
                                 **sel)
                else:   # the standalone calls take device buffers: copies in, output out
                    q, k, v = inputs[t]
                    q.copy_(qh, non_blocking=True)
                    k.copy_(kh, non_blocking=True)
                    v.copy_(vh, non_blocking=True)
                    unfused_step(q, k, v, None)
                    oh.copy_(out, non_blocking=True)
            e1.record(stream)
        stream.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1) / N)
    e2e_mean = dist_max(float(np.mean(e2e_ms)), world, dev)
    status = dc.read_status()
    q, k, _ = inputs[0]
    del g, gp
    return dict(w=w, mean_ms=mean_ms, max_ms=max_ms, bytes=by, stages=stage_mean, window=N,
                outer_ms=float(np.mean(outer_ms)) / N, first=first,
                clocks=clk.summary(), e2e_ms=e2e_mean, kernels_per_step=kernels_per_step,
                h2d=int(q.numel() * q.element_size() + 2 * k.numel() * k.element_size()),
                d2h=int(out.numel() * 4), status=status, p50_ms=float(np.median(win_ms)) / N,
                select=sel, pool=None if pool is None else dict(
                    pool_blocks=int(pool), blocks_held_max=pool_held,
                    bytes_held_max=pool_held * Bn.PAGE_ROWS * w.head_dim * dc.k_pool.element_size() * 2,
                    contiguous_bytes=w.batch * w.n_kv_heads * w.sparse_cap * w.head_dim *
                    dc.k_pool.element_size() * 2))


# ----------------------------------------------------------------------------- oracle

def _oracle_unit_inputs(w, unit_ids):
    """Exact per-unit inputs of the workload's first decode step for the given units."""
    from attention_kv_head_b200 import synth
    lens = synth.seq_lengths(w)
    _, q_ex = synth.queries(w, 0)
    _, k_ex, _, v_ex = synth.step_kv(w, lens, 0)
    G = w.group
    out = []
    for u in unit_ids:
        b, h = divmod(u, w.n_kv_heads)
        L0 = int(lens[b]) - 1
        _, ke, _, ve = synth.unit_kv(w, b, h, 0, L0)
        out.append((b, h, L0, ke, ve, q_ex[b, h * G:(h + 1) * G], k_ex[b, h], v_ex[b, h]))
    return out


def _oracle_worker(task):
    """One pool process: time whole (sequence, KV-head) unit steps of the oracle on its
    share of the units until `budget_s` of oracle time has run."""
    name, seed, unit_ids, budget_s = task
    from attention_kv_head_b200 import synth
    from oracle import hardkv_oracle as O
    w = synth.WORKLOADS[name].with_(seed=seed)
    p = synth.p_values(w)[0]
    prm = O.Params(w.head_dim, w.group, w.dense_window, w.condensed_slots, w.block,
                   w.sparse_cap, w.n_sink, w.dtype, w.condense_mode)
    C = w.condensed_slots
    units = _oracle_unit_inputs(w, unit_ids)
    done, elapsed = 0, 0.0
    while elapsed < budget_s:
        for (b, h, L0, ke, ve, qg, kx, vx) in units:
            un = O.Unit(prm, ke, ve, ke[:C], ve[:C], np.ones(C), L0, L0 + 1 - w.dense_window,
                        C, L0 + 2)
            t = time.perf_counter()
            un.step(qg, kx, vx, 1.0, p)
            elapsed += time.perf_counter() - t
            done += 1
            if elapsed >= budget_s:
                break
    return done, elapsed


class OraclePool:
    """The fp64 oracle as it stands, run over the workload's independent (sequence,
    KV-head) units by a pool of single-threaded processes, one per host core this
    process may use (spawned, so it is safe after CUDA has been initialised)."""

    def __init__(self, w):
        import multiprocessing as mp
        self.w = w
        self.workers = max(1, min(len(os.sched_getaffinity(0)), w.units))
        saved = {k: os.environ.get(k) for k in _BLAS_VARS}
        for k in _BLAS_VARS:
            os.environ[k] = "1"          # one BLAS thread per process: cores = processes
        try:
            self.pool = mp.get_context("spawn").Pool(self.workers)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.shares = [list(range(i, w.units, self.workers)) for i in range(self.workers)]

    def time(self, budget_s: float) -> dict:
        w = self.w
        res = self.pool.map(_oracle_worker, [(w.name, w.seed, sh, budget_s) for sh in self.shares])
        done = sum(d for d, _ in res)
        rate = sum(d / e for d, e in res if e > 0)      # unit steps per second, all processes
        step_s = w.units / rate
        return {"value": w.batch / step_s, "unit": "tokens/s", "cores": self.workers,
                "kind": "oracle", "seconds": round(max(e for _, e in res), 3),
                "sample": f"{done} (sequence, KV-head) unit steps of the {w.name} decode step "
                          f"({w.units} units per step) run by {self.workers} single-threaded "
                          f"processes for {budget_s:.1f} s each; step time = units per step / "
                          f"summed unit-step rate"}

    def close(self):
        self.pool.close()
        self.pool.join()


_BLAS_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def oracle_timing(w, budget_s: float) -> dict:
    """Time the oracle on the workload's first decode step for about `budget_s`."""
    pool = OraclePool(w)
    try:
        return pool.time(budget_s)
    finally:
        pool.close()


# ----------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="llama8b_8k")
    ap.add_argument("--impl", default="hardkv", choices=["hardkv", "reference"])
    ap.add_argument("--oracle-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--p", type=float, default=None, help="top-p mass (default: the workload's)")
    ap.add_argument("--window", type=int, default=0,
                    help="decode steps per timed replay (default: the reselection period)")
    ap.add_argument("--first-step", type=int, default=-1,
                    help="decode steps run untimed before the window (default: 1 for a "
                         "workload that reselects on block moves, else 0)")
    ap.add_argument("--rule", default="topp", choices=["topp", "topk"])
    ap.add_argument("--top-k", type=int, default=0,
                    help="top-k budget (0: the calibrated top-p step's mean kept count)")
    ap.add_argument("--calibration", default="tau", choices=["tau", "entropy"])
    ap.add_argument("--layout", default="rewrite", choices=["rewrite", "sparse", "mti"])
    ap.add_argument("--paged", action="store_true",
                    help="compact rows in the paged tier (block pool + per-head tables)")
    ap.add_argument("--path", default="fused", choices=["fused", "unfused"],
                    help="the fused step (hardkv_decode_step), or the same step as its "
                         "standalone calls: append, condense, selection, regularize, attention")
    ap.add_argument("--l-lower", type=int, default=64)
    ap.add_argument("--l-upper", type=int, default=1 << 30)
    ap.add_argument("--gather-surcharge", type=float, default=0.5)
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_info()
    from attention_kv_head_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.p is not None:
        w = w.with_(p=args.p)
    config = {"workload": w.name, "batch": w.batch, "context": w.context,
              "len_range": w.len_range, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
              "head_dim": w.head_dim, "dense_window": w.dense_window,
              "condensed_slots": w.condensed_slots, "sparse_cap": w.sparse_cap,
              "p": synth.p_values(w)[0], "condense": "merge" if w.condense_mode else "evict",
              "reselect": "every step" if w.select_every == 1 else "on each block move",
              "selection": args.rule + ("" if args.rule == "topp" else f" k={args.top_k or 'auto'}"),
              "calibration": args.calibration, "layout": args.layout,
              "compact_tier": "paged (16-row blocks)" if args.paged else "contiguous",
              "path": "fused step" if args.path == "fused" else "standalone calls",
              "l2": "flushed before every timed step: 2 x L2 written, then read back",
              "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        per_step = max(0.2, min(10.0, 60.0 / max(args.steps + args.warmup, 1)))
        vals, cb = [], None
        pool = OraclePool(w)
        try:
            for i in range(args.warmup + args.steps):
                cb = pool.time(per_step)
                if i >= args.warmup:
                    vals.append(cb["value"])
        finally:
            pool.close()
        v = float(np.mean(vals))
        cb["value"] = v
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * w.batch / v, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": cb,
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    r = run_gpu(args, world, rank, local)
    peaks = measured_peaks()
    N = r["window"]
    by = {k: (v / N if k not in ("kept_fraction",) else v) for k, v in r["bytes"].items()}
    config["decode_steps_per_replay"] = N
    config["first_timed_step"] = r["first"]
    if r["select"].get("top_k"):
        config["selection"] = f"topk k={r['select']['top_k']}"
    # dominant kernel by time (per decode step)
    stages = STAGES if args.path == "fused" else UNFUSED_STAGES
    dom = max(("score", "topp", "attend") if args.path == "fused" else ("regularize", "attend"),
              key=lambda s: r["stages"][s])
    dom_us = r["stages"][dom] * 1e3
    achieved = by[dom] / (dom_us * 1e-6) / 1e9
    traffic = ncu_traffic(KERNEL_OF_STAGE[dom], w.name, args.path)
    step_gbs = by["total"] / (r["mean_ms"] * 1e-3) / 1e9
    value = job_tokens_per_s(world, w.batch, r["max_ms"])
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["max_ms"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
        if w.dtype == "bf16" else "f32", "data": "synthetic", "config": config,
        "e2e": {"value": job_tokens_per_s(world, w.batch, r["e2e_ms"]), "unit": "tokens/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "ms_per_step": r["e2e_ms"],
                "api": "hardkv_decode_step_host" if args.path == "fused" else
                       "pinned-host copies in, the standalone calls, the output copied out"},
        "roofline": {"bound": "hbm", "kernel": KERNEL_OF_STAGE[dom], "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": traffic, "alg_bytes_per_launch": by[dom],
                     "launch_us": dom_us, "peak_source": peaks["source"],
                     "timing": "CUDA events around the kernel in a replay of the step graph"},
        "step_hbm": {"alg_bytes": by["total"], "gbs": step_gbs,
                     "frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS,
                     "frac_of_copy_peak": step_gbs / peaks["hbm_gbs"],
                     "copy_peak_gbs": peaks["hbm_gbs"], "copy_peak_source": peaks["source"],
                     "target_frac_of_8tbs": 0.70,
                     "meets_target": step_gbs / NOMINAL_HBM_GBS >= 0.70,
                     "kept_fraction": by["kept_fraction"], "sum_kept": by["sum_kept"],
                     "p50_ms": r["p50_ms"]},
        "timing": "CUDA events recorded by the step graph before its first and after its "
                  "last kernel, on the launching stream; ms_per_step_with_graph_launch adds "
                  "the graph launch (events around the replay call)",
        "ms_per_step_with_graph_launch": r["outer_ms"],
        "stages_us": {s: round(v_ * 1e3, 2) for s, v_ in r["stages"].items()},
        "stage_alg_bytes": {s: int(by[s]) for s in stages},
        "gpu_launches": r["kernels_per_step"] * args.steps * N,
        "clocks": r["clocks"],
        "device_status": [int(x) for x in r["status"]],
        **({"compact_tier_memory": r["pool"]} if r.get("pool") else {}),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_timing(w, args.oracle_seconds)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
