#!/usr/bin/env python
"""Draft blocks/s of one draft cycle on B200: conv2tap + LM-head top-16 +
path selection + verification.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole path over one batch of B blocks: the two-tap
conv on [B, P, d], the fused LM head + log-softmax + top-16 on [B*L, d] x
[V, d], pair scores + max-sum walk, greedy verification against the target's
tokens.  Inputs are seeded synthetic arrays of the workload's shapes and
distributions (block_draft_synth); W alone is larger than L2, so steps do not
reuse each other's data through L2.

The printed line is the headline workload (default: throughput, 256 blocks of
16 positions, d = 4096, V = 129,280 -- the largest of the five); with one GPU
the same run also times every other workload for its own K steps and reports
each under "workloads", with its own roofline, stage times, clocks and
end-to-end figure.

Multi-GPU: one process per GPU.  `--gpus N` outside torchrun starts N ranks
itself through torch.distributed.run on 127.0.0.1; under torchrun WORLD_SIZE
must equal N.  Blocks are independent, so each rank runs its own batch with
replicated weights and no data-path collective (weak scaling).  The timed
region is bracketed by a barrier and a device synchronize; the elapsed device
time is the max over ranks.

`--impl reference` times the CPU oracle (float64 numpy) on the host's cores on
a bounded sample of the same workload; it is a deliberately slow baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
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

import block_draft_synth as syn  # noqa: E402

METRIC = "draft blocks/sec (LM-head+top16+select+verify) on 1 B200; % of roofline"
UNIT = "blocks/s"
DEFAULT_WORKLOAD = "throughput"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ------------------------------------------------------------------ helpers --

def dist_env():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def rank_workload(w: syn.Workload, rank: int) -> syn.Workload:
    """Per-rank batch: the same weights, different blocks (hidden states,
    targets, conv inputs are drawn from a rank-specific seed)."""
    import dataclasses
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 7919 * rank)


def reduce_max(value: float, world: int) -> float:
    """Max of a host float over all ranks (plumbing, not the data path)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(blocks_per_rank: int, world: int, ms_max: float, steps: int) -> float:
    """Whole-job blocks/s: blocks all ranks processed / the slowest rank's time."""
    return blocks_per_rank * world * steps / (ms_max / 1e3)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS}, "fallback"


def lmhead_algorithmic(w: syn.Workload):
    """Algorithmic bytes and FLOPs of one LM-head top-16 launch: W and H read
    once, the candidate lists and lse written once; 2*M*d*V FLOPs."""
    bytes_ = 2 * w.V * w.d + 2 * w.M * w.d + w.M * (16 * 8 + 4)
    flops = 2.0 * w.M * w.d * w.V
    return bytes_, flops


def kernel_source_hash():
    h = hashlib.sha256()
    for name in ("lmhead_topk.cu", "common.cuh"):
        with open(os.path.join(ROOT, "block_draft_selection_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the LM-head kernel from the committed ncu
    summary for this workload, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"lmhead_topk_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_workload"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for bit, name in self.REASONS.items():
            if mask & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------- GPU arm ----

class Step:
    """One draft cycle on device-resident buffers, through the C ABI.

    cycle "greedy": conv, LM head top-16, max-sum selection + greedy
    verification (the path the metric names).  cycle "sample": conv, LM head
    top-16, a sampled walk from the last verified token (T = 1) and
    rejection-sampling verification against the target's logits (resident
    on the device, as a target model leaves them)."""

    TEMPERATURE = 1.0

    def __init__(self, w: syn.Workload, rank: int, device, cycle: str = "greedy", conv: str = "static"):
        import torch
        import block_draft_selection_b200 as bds
        self.bds, self.torch, self.w = bds, torch, w
        wr = rank_workload(w, rank)
        dev = device
        self.W = bds.bf16_tensor(syn.lm_head(w), dev)
        E, M = syn.selector_tables(w)
        self.E, self.Msel = bds.bf16_tensor(E, dev), bds.bf16_tensor(M, dev)
        a0, a1 = syn.conv_taps(w)
        self.a0, self.a1 = bds.bf16_tensor(a0, dev), bds.bf16_tensor(a1, dev)
        H = syn.hidden(wr)
        x, prev = syn.conv_input(wr)
        self.H = bds.bf16_tensor(H, dev)
        self.x, self.prev = bds.bf16_tensor(x, dev), bds.bf16_tensor(prev, dev)
        # target tokens: the greedy choice of the same head on the noised hidden
        # states (computed once with the library's own LM head, outside timing)
        Hn = bds.bf16_tensor(syn.target_hidden(wr, H), dev)
        _, tix, _ = bds.dflash_lmhead_topk(Hn, self.W)
        self.target = tix[:, 0].contiguous().view(w.B, w.L + 1)
        self.ws = bds.workspace(w.M, w.V, w.d, dev)
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
        self.y = torch.empty_like(self.x)
        self.lp, self.ix, self.lse = e((w.M, 16), torch.float32), e((w.M, 16), torch.int32), e(w.M, torch.float32)
        self.tok, self.slot = e((w.B, w.L), torch.int32), e((w.B, w.L), torch.int32)
        self.score, self.acc, self.nxt = e(w.B, torch.float32), e(w.B, torch.int32), e(w.B, torch.int32)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.side = torch.cuda.Stream(device=dev)     # timing events hang off the kernel chain here
        self.marked = False
        self.cycle, self.conv = cycle, conv
        if conv == "dynamic":
            self.Wc = bds.bf16_tensor(syn.conv_correction(w), dev)
            self.cws = torch.empty(max(1, bds.dflash_conv2tap_dynamic_workspace(w.B, w.P, w.d)),
                                   dtype=torch.uint8, device=dev)
        if cycle == "ctx":
            # the pages' context-gated scorer: tied embeddings (the head), e = 256;
            # the token tables A, B for the whole vocabulary are weights: built once
            Pab, Pg = syn.ctx_scorer_weights(w, 256)
            self.Pab, self.Pg = bds.bf16_tensor(Pab, dev), bds.bf16_tensor(Pg, dev)
            self.anchor = torch.from_numpy(syn.anchors(w.B, w.V, wr.seed)).to(dev)
            self.tab = bds.dflash_ctx_table(self.W, self.Pab)
            self.gate = e((w.M, 256), torch.float32)
            self.gate_stream = torch.cuda.Stream(device=dev)
        if cycle == "sample":
            # the target's logits at the L drafted positions and the bonus
            # position (the library's plain GEMM on the noised hidden states)
            self.z_target = bds.dflash_gemm_bf16(Hn, self.W)
            self.anchor = torch.from_numpy(syn.anchors(w.B, w.V, wr.seed)).to(dev)
            u = lambda shape, name: torch.from_numpy(syn.uniforms(shape, wr.seed, name)).to(dev)
            self.u_walk, self.u_acc, self.u_res = u((w.B, w.L), "u_walk"), u((w.B, w.L), "u_accept"), u((w.B,), "u_resample")
            self.q = e((w.B, w.L, 16), torch.float32)
            self.rws = torch.empty(max(16, bds.dflash_verify_rejection_workspace(w.B, w.L, w.V)), dtype=torch.uint8,
                                   device=dev)

    # conv, LM-head GEMM+epilogue, LM-head merge, select+verify
    LAUNCHES_PER_STEP = 4
    # sample cycle: conv, LM head (2), walk, rejection verification (2)
    LAUNCHES_PER_STEP_SAMPLE = 6
    # ctx cycle: conv, LM head (2), gate GEMM (its zeroing, when K is split, is
    # a memset node, not a kernel), scores + walk
    LAUNCHES_PER_STEP_CTX = 5

    def launches(self):
        n = {"sample": self.LAUNCHES_PER_STEP_SAMPLE, "ctx": self.LAUNCHES_PER_STEP_CTX}.get(
            self.cycle, self.LAUNCHES_PER_STEP)
        return n + (1 if self.conv == "dynamic" else 0)   # the dynamic conv adds its correction GEMM

    def mark(self, ev):
        """Record `ev` when everything enqueued so far on the current stream
        has completed, on a side stream: the event hangs off the kernel chain
        instead of sitting in it, so consecutive kernels keep their
        programmatic (early) launch.  Inside graph capture the side stream
        must be joined back before the capture ends (see join_marks)."""
        import torch
        cur = torch.cuda.current_stream()
        self.side.wait_stream(cur)
        with torch.cuda.stream(self.side):
            ev.record()
        self.marked = True

    def join_marks(self):
        import torch
        if self.marked:
            torch.cuda.current_stream().wait_stream(self.side)
            self.marked = False

    def run(self, marks=None, side=False):
        """One cycle.  `marks`: optional {stage name: (event, event)} recorded
        around that stage's call.  side=False: the events sit in the kernel
        chain (the bracketed stage's first kernel then starts only after the
        start event, without the programmatic early launch); side=True: they
        hang off the chain on a side branch (see mark), so the kernels keep
        their early launch -- accurate for long stages, while two side
        events are never less than a few microseconds apart.  "event_pair"
        brackets nothing (the cost of the two event nodes) and
        "lmhead_select" brackets the LM head and the selection together."""
        bds = self.bds
        marks = marks or {}
        put = self.mark if side else (lambda e: e.record())

        def stage(name, fn):
            ev = marks.get(name)
            if ev:
                put(ev[0])
            fn()
            if ev:
                put(ev[1])

        stage("event_pair", lambda: None)    # calibration: two event nodes, nothing between
        if self.cycle == "ctx":
            # the gate needs only H: it runs on a forked stream beside the conv
            # and the LM head, and the walk waits for it
            cur = self.torch.cuda.current_stream()
            self.gate_stream.wait_stream(cur)
            with self.torch.cuda.stream(self.gate_stream):
                bds.dflash_ctx_gate(self.H, self.Pg, gate=self.gate)
        if self.conv == "dynamic":
            stage("conv2tap", lambda: bds.dflash_conv2tap_dynamic(self.x, self.a0, self.a1, self.Wc, self.prev,
                                                                  y=self.y, ws=self.cws))
        else:
            stage("conv2tap", lambda: bds.dflash_conv2tap(self.x, self.a0, self.a1, self.prev, y=self.y))
        span = marks.get("lmhead_select")
        if span:
            put(span[0])
        stage("lmhead_topk", lambda: bds.dflash_lmhead_topk(
            self.H, self.W, topk_logp=self.lp, topk_idx=self.ix, lse=self.lse, ws=self.ws, dev_status=self.status))
        if self.cycle == "sample":
            def walk_verify():
                bds.dflash_path_walk(self.lp, self.ix, self.E, self.Msel, self.anchor, self.w.B, self.w.L,
                                     uniforms=self.u_walk, temperature=self.TEMPERATURE, path_tok=self.tok,
                                     path_slot=self.slot, path_score=self.score, path_q=self.q,
                                     dev_status=self.status)
                bds.dflash_verify_rejection(self.z_target, self.TEMPERATURE, self.tok, self.slot, self.ix, self.q,
                                            self.u_acc, self.u_res, accept_len=self.acc, next_token=self.nxt,
                                            ws=self.rws, dev_status=self.status)
            stage("select_verify", walk_verify)
        elif self.cycle == "ctx":
            def ctx_select_verify():
                self.torch.cuda.current_stream().wait_stream(self.gate_stream)
                bds.dflash_ctx_walk(self.lp, self.ix, self.anchor, self.tab, self.gate, self.w.B, self.w.L,
                                    self.w.V, walk="maxsum", target=self.target, path_tok=self.tok,
                                    path_slot=self.slot, path_score=self.score, accept_len=self.acc,
                                    next_token=self.nxt, dev_status=self.status)
            stage("select_verify", ctx_select_verify)
        else:
            stage("select_verify", lambda: bds.dflash_select_verify(
                self.lp, self.ix, self.E, self.Msel, self.target, self.w.B, self.w.L, path_tok=self.tok,
                path_slot=self.slot, path_score=self.score, accept_len=self.acc, next_token=self.nxt,
                dev_status=self.status))
        if span:
            put(span[1])


def _graph_steps(step, n_steps, plan, side=False):
    """Capture n_steps cycles into one CUDA graph.  plan(k) names the stage
    (or a tuple of stages) whose call cycle k brackets with a pair of
    external timing events (event nodes; in the kernel chain, or on a side
    branch with side=True), or None.  Returns (graph, [(stage name, (start,
    end))])."""
    import torch
    ev = lambda: (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
    def names(k):
        n = plan(k)
        return () if not n else ((n,) if isinstance(n, str) else tuple(n))
    marks = [{n: ev() for n in names(k)} or None for k in range(n_steps)]
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step.run()
    side.synchronize()
    with torch.cuda.graph(g, stream=side):
        for k in range(n_steps):
            step.run(marks[k], side=side)
        step.join_marks()          # a timing side branch rejoins once, at the end
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    return g, [(name, pair) for m in marks if m for name, pair in m.items()]


def _chunk(steps, cap=32):
    """Largest divisor of `steps` not above `cap`: cycles per captured graph."""
    return max(c for c in range(1, min(cap, steps) + 1) if steps % c == 0)


# LM-head launch durations sampled inside the timed region (at least).
LM_SAMPLES = 20
# Samples of each bracket in the graph that measures what the selection adds
# to a pipelined cycle (the difference of two medians of event spans a few
# microseconds apart needs more than the roofline's mean).
PIPE_SAMPLES = 40

# Stage breakdown: one extra graph after the timed region in which cycle k
# brackets stage BREAKDOWN[k % 5]; every stage gets BREAKDOWN_SAMPLES samples.
BREAKDOWN = ("event_pair", "conv2tap", "lmhead_topk", "select_verify", "lmhead_select")
BREAKDOWN_SAMPLES = 24


def _summ(xs):
    xs = sorted(xs)
    return {"mean": statistics.mean(xs), "median": statistics.median(xs), "min": xs[0], "max": xs[-1],
            "n": len(xs)} if xs else None


def _release():
    import gc
    import torch
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _calibrated_steps(step, target_s: float, floor: int, cap: int = 20000) -> int:
    """Cycles that make a timed region of about target_s seconds (at least
    `floor`), from one replay of an 8-cycle graph; a multiple of 32 when
    that many."""
    import torch
    g, _ = _graph_steps(step, 8, lambda k: None)
    g.replay()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(3):
        g.replay()
    t1.record()
    torch.cuda.synchronize()
    per = t0.elapsed_time(t1) / 1e3 / 24
    del g
    n = int(min(cap, max(floor, target_s / max(per, 1e-9))))
    return n - n % 32 if n >= 64 else n


def measure(args, w: syn.Workload, steps, warmup: int, rank: int, world: int, device):
    """Time `steps` cycles of workload w (steps None: calibrated to about
    args.sub_seconds, at least args.steps) and return the workload's result:
    blocks/s, the LM head's roofline from the timed region, the stage
    breakdown, clocks and the end-to-end figure."""
    import torch
    import block_draft_selection_b200 as bds

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    step = Step(w, rank, device, args.cycle, args.conv)
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    if steps is None:
        steps = _calibrated_steps(step, args.sub_seconds, args.steps)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # timed region: cycles replayed from up to 64 distinct captured graphs, a
    # few evenly spaced cycles of each bracketing their LM-head call, so the
    # roofline's launch duration has at least LM_SAMPLES samples from the
    # timed region (every cycle when there are no more steps than that) while
    # most cycles keep their kernel-to-kernel launch overlap
    if args.eager:
        chunk, graphs = 1, []
        marks = [{"lmhead_topk": (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))}
                 for _ in range(steps)]
    else:
        chunk = _chunk(steps)
        n_rep = steps // chunk
        n_graphs = min(64, n_rep)
        per_graph = min(chunk, -(-LM_SAMPLES // n_graphs))
        spacing = chunk // per_graph
        # evenly spaced and centred: with one bracket per graph it sits in the
        # middle cycle (the last cycle of a graph measured about 10 us slower
        # at qwen3-4b-bs1 than the same stage anywhere else)
        timed = {spacing // 2 + j * spacing for j in range(per_graph)}
        graphs = [_graph_steps(step, chunk, lambda k: "lmhead_topk" if k in timed else None, side=True)
                  for _ in range(n_graphs)]
        for g, _ in graphs:
            g.replay()              # one untimed replay of each captured graph
    barrier()
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t0.record()
        if args.eager:
            for k in range(steps):
                step.run(marks[k], side=True)
            step.join_marks()
        else:
            for rep in range(n_rep):
                graphs[rep % len(graphs)][0].replay()
        t1.record()
        torch.cuda.synchronize()
    barrier()
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} during the timed region ({w.name})")
    ms = t0.elapsed_time(t1)
    # LM-head launch durations of the timed region: every cycle of the eager
    # loop, or every cycle of each graph's last replay
    if args.eager:
        lm_samples = [m["lmhead_topk"][0].elapsed_time(m["lmhead_topk"][1]) for m in marks]
    else:
        lm_samples = [a.elapsed_time(b) for _, gm in graphs for _, (a, b) in gm]
    ms_max = reduce_max(ms, world)
    value = aggregate(w.B, world, ms_max, steps)
    del graphs

    # what the selection adds to a pipelined cycle (after the timed region):
    # one graph whose cycles alternate side-branch brackets of the LM head
    # alone and of the LM head with the selection after it, every kernel
    # keeping its programmatic launch; the difference of the medians.  (Two
    # brackets in one cycle would fork the chain between the LM head and the
    # selection, which delays the selection.)
    pg, pm = _graph_steps(step, 2 * PIPE_SAMPLES, lambda k: ("lmhead_topk", "lmhead_select")[k % 2], side=True)
    pg.replay()
    torch.cuda.synchronize()
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} in the pipelined brackets ({w.name})")
    lmp = [a.elapsed_time(b) for n, (a, b) in pm if n == "lmhead_topk"]
    lsp = [a.elapsed_time(b) for n, (a, b) in pm if n == "lmhead_select"]
    del pg, pm
    sel_pipe_ms = max(0.0, statistics.median(lsp) - statistics.median(lmp))

    # stage breakdown (after the timed region, same clocks regime): cycle k of
    # one graph brackets stage BREAKDOWN[k % 5].  This graph is captured
    # without programmatic launch: with it, a kernel may start before the
    # event node in front of it, and a bracket of a few microseconds then
    # misses part of its stage.  Each stage here runs serialised -- its own
    # launch plus its execution -- an upper bound on what it adds to a
    # pipelined cycle.
    pdl_before = os.environ.get("DFLASH_PDL")
    os.environ["DFLASH_PDL"] = "0"
    try:
        sg, sm = _graph_steps(step, len(BREAKDOWN) * BREAKDOWN_SAMPLES, lambda k: BREAKDOWN[k % len(BREAKDOWN)])
    finally:
        if pdl_before is None:
            del os.environ["DFLASH_PDL"]
        else:
            os.environ["DFLASH_PDL"] = pdl_before
    sg.replay()
    torch.cuda.synchronize()
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} in the stage breakdown ({w.name})")
    samples = {n: [] for n in BREAKDOWN}
    for name, (a, b) in sm:
        samples[name].append(a.elapsed_time(b))
    del sg, sm
    med = lambda n: statistics.median(samples[n])
    ev_ms = med("event_pair")
    # in-chain brackets: net of the cost of the two event nodes (measured alone)
    stage_ms = {n: max(0.0, med(n) - ev_ms) for n in ("conv2tap", "lmhead_topk", "select_verify")}
    # what the selection stage adds to a cycle: (LM head + selection bracketed
    # together) - (LM head bracketed alone); both gross, the event cost cancels
    sel_added_ms = max(0.0, med("lmhead_select") - med("lmhead_topk"))
    cyc_ms = ms_max / steps


    # end-to-end leg: the library's DraftCycle, one graph launch per step that
    # copies the step's inputs from pinned host memory, runs the cycle and
    # copies the results back; the host waits for them every step
    if args.cycle == "greedy" and args.conv == "static":
        cyc = bds.DraftCycle(step.W, step.E, step.Msel, step.a0, step.a1, w.B, w.L, w.P)
        cyc.host_in["H"].copy_(step.H)
        cyc.host_in["x"].copy_(step.x)
        cyc.host_in["prev"].copy_(step.prev)
        cyc.host_in["target"].copy_(step.target)
        for _ in range(max(3, warmup)):
            cyc.run()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            cyc.run()               # raises if a kernel of the step reports a device error
        e1.record()
        torch.cuda.synchronize()
        barrier()
        e_ms = reduce_max(e0.elapsed_time(e1), world)
        h2d, d2h = cyc.io_bytes()
        e2e = {"value": aggregate(w.B, world, e_ms, steps), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
               "path": "DraftCycle.run(): one graph launch per step: pinned H2D of H + targets + zeroed status, "
                       "LM head, select/verify, D2H of status + results; beside it on a second stream H2D of the "
                       "conv input, conv, D2H of its output; host sync"}
        del cyc
        # the same steps through DraftPipeline: two independent batches in
        # flight on two streams, every step's inputs copied in and its
        # results read back on the host (serving independent groups of
        # blocks; the dependent loop is the e2e above)
        pipe = bds.DraftPipeline(step.W, step.E, step.Msel, step.a0, step.a1, w.B, w.L, w.P)
        for c in pipe.cycles:
            c.host_in["H"].copy_(step.H)
            c.host_in["x"].copy_(step.x)
            c.host_in["prev"].copy_(step.prev)
            c.host_in["target"].copy_(step.target)
        for _ in range(max(3, warmup)):
            pipe.host_in()
            pipe.launch()
        pipe.drain()
        barrier()
        cur = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s_ in pipe.streams:
            s_.wait_stream(cur)
        for _ in range(steps):
            pipe.host_in()          # waits for this cycle's previous step and reads its results
            pipe.launch()
        pipe.drain()
        for s_ in pipe.streams:
            cur.wait_stream(s_)
        e1.record()
        torch.cuda.synchronize()
        barrier()
        p_ms = reduce_max(e0.elapsed_time(e1), world)
        e2e["overlapped"] = {"value": aggregate(w.B, world, p_ms, steps), "unit": UNIT, "steps": steps,
                             "path": "DraftPipeline: the same graph as above on two DraftCycles, stepped "
                                     "alternately on two streams; each step's inputs copied from pinned host "
                                     "memory and its results read back on the host"}
        del pipe
    else:
        e2e = {"value": None, "unit": UNIT, "h2d_bytes_per_step": None, "d2h_bytes_per_step": None,
               "path": "measured for the greedy cycle with static taps only (the metric's path)"}

    peaks, peaks_kind = load_peaks()
    alg_bytes, alg_flops = lmhead_algorithmic(w)
    lm_ms = statistics.mean(lm_samples)
    t_lm = lm_ms / 1e3
    hbm_t = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    tc_t = alg_flops / (peaks["bf16_tflops"] * 1e12)
    if hbm_t >= tc_t:
        roof = {"bound": "hbm", "achieved": alg_bytes / t_lm / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        pk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": alg_flops / t_lm / 1e12, "peak": pk, "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if roof["bound"] == "tensor":
        # timed inside long runs of back-to-back cycles: the sustained peak is
        # the denominator; the burst-peak fraction is given beside it
        roof["peak_kind"] = "bf16_tflops_sustained"
        roof["frac_of_burst"] = roof["achieved"] / peaks["bf16_tflops"]
    roof["traffic"] = profiled_traffic(w.name)
    roof["peak_source"] = peaks_kind
    roof["kernel"] = "dflash_lmhead_topk (GEMM+epilogue and merge kernels)"
    roof["algorithmic_per_launch"] = alg_bytes if roof["bound"] == "hbm" else alg_flops
    roof["launch_ms"] = lm_ms
    roof["launch_ms_samples"] = _summ(lm_samples)
    roof["timing"] = ("mean CUDA-event duration of the LM-head call (GEMM+epilogue kernel and merge kernel), from "
                      "the completion of the kernel before it to the completion of its merge kernel; events recorded "
                      "on a side branch of the graph so the kernels keep their programmatic launch; evenly spaced "
                      "cycles of every timed graph: at least %d samples (every cycle when the run has no more "
                      "steps), over the timed region" % LM_SAMPLES)
    stages = {**{n: 1e3 * stage_ms[n] for n in stage_ms},
              "select_verify_share": stage_ms["select_verify"] / cyc_ms,
              "select_verify_added": 1e3 * sel_added_ms,
              "select_verify_added_share": sel_added_ms / cyc_ms,
              "select_verify_pipelined": 1e3 * sel_pipe_ms,
              "select_verify_pipelined_share": sel_pipe_ms / cyc_ms,
              "pipelined_samples": {"lmhead_topk": len(lmp), "lmhead_select": len(lsp)},
              "event_pair_overhead": 1e3 * ev_ms,
              "samples": {n: len(samples[n]) for n in BREAKDOWN},
              "raw_us": {n: {k: (1e3 * v if k != "n" else v) for k, v in _summ(samples[n]).items()}
                         for n in BREAKDOWN},
              "note": ("medians over one extra graph after the timed region, captured without programmatic "
                       "launch, whose cycle k brackets stage k mod 5 (%d samples per stage) with event nodes "
                       "in the kernel chain, net of the two event nodes (measured alone): each stage's time is "
                       "its own launch plus its execution, serialised -- an upper bound on what it adds to the "
                       "pipelined cycles of the timed region; select_verify_added = (LM head + selection "
                       "bracketed together) - (LM head bracketed alone). select_verify_pipelined: the same "
                       "difference of medians from a second extra graph whose cycles alternate the two brackets "
                       "on side branches of the kernel chain, every kernel keeping its programmatic launch as in "
                       "the timed region: what the selection adds to the timed cycles" % BREAKDOWN_SAMPLES)}
    config = {"workload": w.name + {"greedy": "", "sample": "+sampled-walk(T=1)",
                                    "ctx": "+context-gated-scorer"}[args.cycle]
                          + ("+dynamic-conv" if args.conv == "dynamic" else ""),
              "blocks_per_gpu": w.B, "L": w.L, "M": w.M, "d": w.d, "V": w.V,
              "K": 16, "r": w.r, "conv": [w.B, w.P, w.d], "conv_taps": args.conv, "cycle": args.cycle,
              "parallelism": f"dp{world} (blocks)",
              "launch": "eager" if args.eager else f"cuda graphs of {chunk} cycles, PDL between kernels",
              "l2": "inputs larger than L2 (W is %.0f MB > 126 MB)" % (2 * w.V * w.d / 1e6)}
    launches = step.launches() * steps
    del step
    _release()
    return {"value": value, "unit": UNIT, "steps": steps, "warmup": warmup, "ms_per_step": cyc_ms,
            "config": config, "e2e": e2e, "gpu_launches": launches, "roofline": roof,
            "stages_us": stages, "clocks": clk.summary()}


def gpu_arm(args, w: syn.Workload):
    import torch
    rank, local_rank, world = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    head = measure(args, w, args.steps, args.warmup, rank, world, device)
    subs = {}
    if world == 1 and args.sub_workloads:
        for name in args.sub_workloads:
            if name != w.name:
                subs[name] = measure(args, syn.workload(name), None, args.warmup, rank, world, device)
    out = None
    if rank == 0:
        out = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded block_draft_synth; random-init weights of the workload's shapes)",
            "config": head["config"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
            "roofline": head["roofline"], "stages_us": head["stages_us"], "clocks": head["clocks"],
        }
        if subs:
            out["workloads"] = subs
            out["workloads_note"] = ("the other workloads, each timed in this run for its own steps "
                                     "(calibrated to about %.2f s, at least --steps), same warm-up; the headline "
                                     "above is the largest workload" % args.sub_seconds)
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return out


# --------------------------------------------------------------- CPU oracle --

class OracleSample:
    """The CPU oracle, as it stands, on a bounded sample of the workload.

    One sample step runs the oracle's conv on the full conv input, its LM head
    + top-16 on a slice of the vocabulary (rows [v0, v0+Vs) of W, rotating
    over steps), and its path selection + verification on the slice's lists.
    The LM-head part is the only one whose work depends on V, and it grows in
    proportion to V, so a full cycle is estimated as
    t_cycle = (V / Vs) * t_lmhead_slice + t_rest."""

    def __init__(self, w: syn.Workload):
        import oracle
        self.o, self.w = oracle, w
        self.H, self.W = syn.hidden(w), syn.lm_head(w)
        self.E, self.M = syn.selector_tables(w)
        self.x, self.prev = syn.conv_input(w)
        self.a0, self.a1 = syn.conv_taps(w)
        self.target = np.random.default_rng(0).integers(0, w.V, size=(w.B, w.L + 1))
        self.v0 = 0

    def step(self, Vs: int):
        o, w = self.o, self.w
        Vs = max(16, min(Vs, w.V))
        if self.v0 + Vs > w.V:
            self.v0 = 0
        sl = slice(self.v0, self.v0 + Vs)
        self.v0 += Vs
        t0 = time.perf_counter()
        lp, ix, _ = o.lmhead_topk(self.H, self.W[sl], 16)
        t1 = time.perf_counter()
        o.conv2tap(self.x, self.prev, self.a0, self.a1)
        sel = o.path_select(lp, ix, self.E[sl], self.M, w.B, w.L)
        o.verify(sel["path_tok"], self.target)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1, Vs

    def estimate(self, recs):
        """blocks/s from recorded (t_lm, t_rest, Vs) steps."""
        w = self.w
        t_cycle = statistics.mean(t_lm * (w.V / vs) for t_lm, _, vs in recs) + statistics.mean(r for _, r, _ in recs)
        return w.B / t_cycle, t_cycle


def _threads_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def _size_slice(smp: OracleSample, per_step_s: float) -> int:
    """Vocabulary slice whose sample step takes about per_step_s seconds."""
    w = smp.w
    Vs = min(w.V, 4096)
    t_lm, t_rest, _ = smp.step(Vs)
    per_row = t_lm / Vs
    return int(max(256, min(w.V, (per_step_s - t_rest) / max(per_row, 1e-12))))


def cpu_baseline(w: syn.Workload, seconds: float):
    """The oracle timed for about `seconds` of host CPU work on a bounded sample."""
    smp = OracleSample(w)
    Vs = _size_slice(smp, per_step_s=max(0.05, seconds / 8))
    recs, t_start = [], time.perf_counter()
    while time.perf_counter() - t_start < seconds or len(recs) < 2:
        recs.append(smp.step(Vs))
    value, t_cycle = smp.estimate(recs)
    return {"value": value, "unit": UNIT, "cores": _threads_used(), "kind": "oracle",
            "sample": (f"{len(recs)} oracle steps on workload {w.name}: conv + selection + verification of "
                       f"all {w.B} block(s) per step, LM head on a {Vs}-row vocabulary slice (of {w.V}); "
                       f"cycle time estimated as (V/slice)*t_lmhead + t_rest = {t_cycle:.3f} s"),
            "host_cores_available": len(os.sched_getaffinity(0))}


def reference_arm(args, w: syn.Workload):
    rank, _, world = dist_env()
    if rank != 0:
        return None
    smp = OracleSample(w)
    budget = float(args.ref_budget_s)
    Vs = _size_slice(smp, per_step_s=max(0.01, budget / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        smp.step(Vs)
    recs = [smp.step(Vs) for _ in range(args.steps)]
    value, t_cycle = smp.estimate(recs)
    cb = {"value": value, "unit": UNIT, "cores": _threads_used(), "kind": "oracle",
          "sample": (f"each step: oracle conv + selection + verification of all {w.B} block(s), LM head on a "
                     f"{Vs}-row slice of the {w.V}-row vocabulary; blocks/s from "
                     f"(V/slice)*t_lmhead + t_rest = {t_cycle:.3f} s per cycle"),
          "host_cores_available": len(os.sched_getaffinity(0))}
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_cycle,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded block_draft_synth)",
            "config": {"workload": w.name, "blocks_per_gpu": w.B, "L": w.L, "M": w.M, "d": w.d, "V": w.V,
                       "K": 16, "r": w.r, "conv": [w.B, w.P, w.d], "parallelism": "host cores"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def relaunch(n: int, argv) -> int:
    """Run this script as n ranks through torch.distributed.run on 127.0.0.1
    (one process per GPU) and return its exit code; rank 0 prints the line."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__), *argv]
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "1"))
    return subprocess.run(cmd, env=env).returncode


def launch_selftest(args):
    """Checks the N-rank launch itself on CPU (gloo): every rank joins, the
    ranks agree on the world size, and a max over ranks reaches rank 0.  No
    GPU, no kernel, no metric."""
    import datetime
    import torch
    import torch.distributed as dist
    rank, _, world = dist_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    seen = [None] * world
    dist.all_gather_object(seen, rank)
    t = torch.tensor([float(rank + 1)], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return None
    return {"launch_selftest": True, "n_gpus": world, "ranks": seen, "max_over_ranks": float(t.item())}


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    names = [x.name for x in syn.WORKLOADS]
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=names)
    ap.add_argument("--sub-workloads", default=",".join(names),
                    help="comma-separated workloads also timed (one GPU only) and reported under 'workloads'; "
                         "'' for none (the headline workload is skipped here)")
    ap.add_argument("--sub-seconds", type=float, default=0.3,
                    help="timed seconds each extra workload aims at (at least --steps steps)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch each cycle eagerly instead of a CUDA graph")
    ap.add_argument("--cycle", default="greedy", choices=["greedy", "sample", "ctx"],
                    help="greedy: max-sum selection + greedy verification (the metric's path); sample: "
                         "sampled walk from the last verified token + rejection-sampling verification; ctx: "
                         "the pages' context-gated scorer, max-sum from the last verified token + greedy "
                         "verification")
    ap.add_argument("--conv", default="static", choices=["static", "dynamic"],
                    help="static base taps (the metric's path) or taps with the per-16-channel correction")
    ap.add_argument("--ref-budget-s", type=float, default=120.0,
                    help="host seconds the --impl reference run aims to take")
    ap.add_argument("--launch-selftest", action="store_true",
                    help="check the N-rank launch on CPU (gloo) and print the ranks seen; runs no kernel")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    args.sub_workloads = [x for x in args.sub_workloads.split(",") if x]
    for x in args.sub_workloads:
        if x not in names:
            ap.error(f"unknown workload {x!r} in --sub-workloads")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch(args.gpus, argv))
    _, _, world = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    w = syn.workload(args.workload)
    if args.launch_selftest:
        out = launch_selftest(args)
    elif args.impl == "reference":
        out = reference_arm(args, w)
    else:
        out = gpu_arm(args, w)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
