#!/usr/bin/env python3
"""Benchmark of the hybrid compressed-attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all] [--impl reference]

Workloads (synthetic, seeded): csa_decode_1m_incremental (the headline),
csa_decode_64k, hca_decode_1m, csa_prefill_128k, tiny_prefill.  The default
(`all`) times K steps of the headline, then up to 20 steps of every other
workload, and prints the headline's figures at the top level of the line and
every workload's under "workloads".  A step is one pass of the whole path for
one batch: decode -> append 4 tokens (pool one entry + 4 window tokens), indexer
+ top-k, attention; HCA decode -> append 128 tokens (one entry + window) then
dense attention; prefill -> pool the whole sequence, index + select every
position, attend.

Prints ONE JSON line (rank 0).  With N > 1 every rank runs its own independent
sequences (weak scaling, no collective on the data path); times are the max
over ranks.  `--gpus N` without torchrun starts the N ranks itself.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA decode tokens/s and prefill queries/s on 1 B200; % of HBM BW / MMA peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# cycles of the device sleep that queues each separately timed call
SLEEP_CYCLES = 2_000_000


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------------------
# algorithmic work per step (bytes that must move, flops that must be done)
# ---------------------------------------------------------------------------


def op_work(wl):
    """Algorithmic bytes / flops of each library call of one step."""
    B, D, H, m, K, W = wl.B, wl.D, wl.H, wl.m, wl.K, wl.W
    ent = D + 4                        # E4M3 codes + fp32 scale
    w = {}
    if wl.kind in ("decode", "decode_incremental", "hca_decode"):
        n_new = 4 if wl.kind != "hca_decode" else m
        N = wl.N
        raw = B * n_new * D * 8
        # entries and window in one pass over the new tokens (x and z once)
        w["compress"] = dict(bytes=raw + B * (n_new // m) * ent + B * n_new * ent, flops=0)
        if wl.kind == "hca_decode":
            items = N + W
            w["hca_attend"] = dict(bytes=B * items * ent + 2 * B * H * D * 2 + B * H * 4,
                                   flops=4.0 * B * H * items * D)
        else:
            keys = B * N * (wl.dI // 2)
            w["index_topk"] = dict(bytes=keys + B * wl.HI * (wl.dI // 2 + 4) + B * K * 8,
                                   flops=2.0 * B * N * wl.HI * wl.dI)
            items = K + W
            w["attend"] = dict(bytes=B * items * ent + 2 * B * H * D * 2 + B * K * 4 + B * H * 4,
                               flops=4.0 * B * H * items * D)
            # the fused step moves exactly what the four calls move (the
            # selection is handed over on chip instead of through memory)
            w["decode_step"] = dict(bytes=sum(v["bytes"] for v in w.values()),
                                    flops=sum(v["flops"] for v in w.values()), aggregate=True)
    else:   # prefill
        T, N = wl.T, wl.N
        w["compress"] = dict(bytes=B * T * D * 8 + B * N * ent + B * T * ent, flops=0)
        pairs = B * sum_visible(T, m, N)
        w["index_topk"] = dict(bytes=B * N * (wl.dI // 2) + B * T * (wl.HI * (wl.dI // 2 + 4) + K * 8),
                               flops=2.0 * pairs * wl.HI * wl.dI)
        att = B * sum_attended(T, m, N, K, W)
        w["attend"] = dict(bytes=att * ent + 2 * B * T * H * D * 2 + B * T * K * 4,
                           flops=4.0 * att * H * D)
    return w


def sum_visible(T, m, N):
    t = np.arange(T, dtype=np.int64)
    return int(np.minimum((t + 1) // m, N).sum())


def sum_attended(T, m, N, K, W):
    t = np.arange(T, dtype=np.int64)
    return int((np.minimum(np.minimum((t + 1) // m, N), K) + np.minimum(W, t + 1)).sum())


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(rows), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------


class Runner:
    """One workload's device state.  `calls(i)` lists the library calls of step i
    as (name, launch) pairs; a step is replayed as one CUDA graph."""

    def __init__(self, wl, seed, device, fused=True):
        import torch

        import synth
        from compressed_sparse_attention_16_b200 import Dims, pipeline

        self.torch = torch
        self.wl = wl
        self.dev = device
        torch.cuda.set_device(device)
        self.graphs = {}
        self._side = None
        self.decode = wl.kind in ("decode", "decode_incremental", "hca_decode")
        if self.decode:
            self.n_new = wl.m if wl.kind == "hca_decode" else 4
            self.n_steps = max(wl.steps, 1) + 256 if wl.kind == "decode_incremental" else 1
            self.T0 = wl.T if wl.kind == "decode_incremental" else wl.T - self.n_new
            Ttot = self.T0 + self.n_new * self.n_steps
            self.x, self.z = synth.tokens(wl.B, Ttot, wl.D, seed, device=device)
            dense = wl.kind == "hca_decode"
            cap = Ttot // wl.m
            self.state = pipeline.DecodeState(wl.B, wl.D, wl.H, wl.m, wl.W, entry_cap=cap, K=max(wl.K, 1),
                                              HI=max(wl.HI, 1), dI=max(wl.dI, 32), dense=dense)
            if not dense:
                self.ind = synth.indexer_inputs(wl.B, 1, cap, wl.HI, wl.dI, seed, device=device)
                self.state.kI.copy_(self.ind.kI)
                # each step's new tokens as contiguous [B, n_new, D] blocks (the fused step's input)
                steps_x = self.x[:, self.T0:self.T0 + self.n_new * self.n_steps]
                steps_z = self.z[:, self.T0:self.T0 + self.n_new * self.n_steps]
                self.x_steps = steps_x.reshape(wl.B, self.n_steps, self.n_new, wl.D).transpose(0, 1).contiguous()
                self.z_steps = steps_z.reshape(wl.B, self.n_steps, self.n_new, wl.D).transpose(0, 1).contiguous()
            self.q = synth.queries(wl.B, 1, wl.H, wl.D, wl.q_scale, seed, device=device)
            self.state.prefill_context(self.x, self.z, self.T0)
            # per-step query positions (graph-static)
            pos = self.T0 + self.n_new * (torch.arange(self.n_steps, device=device) + 1) - 1
            self.q_pos_all = pos.to(torch.int32)[:, None, None].repeat(1, wl.B, 1).contiguous()
            self.units_per_step = wl.B
            self.unit = "tokens/s"
            self.Dims = Dims
            # workspaces sized for the largest step, allocated before any capture
            import compressed_sparse_attention_16_b200 as csa
            self.fused = False
            for j in (0, self.n_steps - 1):
                d = self._dims(j)
                if wl.kind == "hca_decode":
                    self._ws(csa.attend_workspace(d, True), "_ws_hca")
                else:
                    self._ws(csa.index_topk_workspace(d), "_ws_index")
                    self._ws(csa.attend_workspace(d), "_ws_attend")
                    nb = csa.decode_step_workspace(d, self.n_new) if fused else 0
                    if nb:
                        self.fused = True
                        if getattr(self, "_ws_step", None) is None or self._ws_step.numel() < nb:
                            # zero-filled once: the fused step keeps its barrier words consistent
                            self._ws_step = torch.zeros(nb + 4096, dtype=torch.uint8, device=device)
        else:
            self.x, self.z = synth.tokens(wl.B, wl.T, wl.D, seed, device=device)
            self.q = synth.queries(wl.B, wl.T, wl.H, wl.D, wl.q_scale, seed, device=device)
            self.ind = synth.indexer_inputs(wl.B, wl.T, wl.N, wl.HI, wl.dI, seed, device=device)
            self._prefill_buffers()
            self.units_per_step = wl.B * wl.T
            self.unit = "queries/s"
        torch.cuda.synchronize()

    def _prefill_buffers(self):
        import compressed_sparse_attention_16_b200 as csa
        torch, wl, dev = self.torch, self.wl, self.dev
        B, T, D, H, N, K = wl.B, wl.T, wl.D, wl.H, wl.N, wl.K
        self.codes = torch.empty((B, N, D), dtype=torch.uint8, device=dev)
        self.scales = torch.empty((B, N), dtype=torch.float32, device=dev)
        self.wcodes = torch.empty((B, T, D), dtype=torch.uint8, device=dev)
        self.wscales = torch.empty((B, T), dtype=torch.float32, device=dev)
        self.q_pos = torch.arange(T, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
        self.dims = csa.Dims(B=B, Tq=T, H=H, D=D, HI=wl.HI, dI=wl.dI, K=K, W=wl.W, m=wl.m, n_entries=N,
                             entry_cap=N, win_cap=T)
        self.idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
        self.score = torch.empty((B, T, K), dtype=torch.float32, device=dev)
        self.out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
        nb = csa.index_topk_workspace(self.dims)
        self.ws_i = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
        nb = csa.attend_workspace(self.dims)
        self.ws_a = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None

    def _ws(self, nbytes, key):
        cur = getattr(self, key, None)
        if nbytes and (cur is None or cur.numel() < nbytes):
            if self.torch.cuda.is_current_stream_capturing():
                raise RuntimeError("workspace growth during graph capture")
            cur = self.torch.empty(int(nbytes * 1.25) + 4096, dtype=self.torch.uint8, device=self.dev)
            setattr(self, key, cur)
        return cur if nbytes else None

    def _dims(self, j):
        wl, st = self.wl, self.state
        t0 = self.T0 + self.n_new * j
        return self.Dims(B=wl.B, Tq=1, H=wl.H, D=wl.D, HI=st.HI, dI=st.dI, K=st.K, W=wl.W, m=wl.m,
                         n_entries=(t0 + self.n_new) // wl.m, entry_cap=st.entry_cap, win_cap=st.win_cap)

    def step_index(self, i):
        return i % self.n_steps if self.wl.kind == "decode_incremental" else 0

    def calls(self, i, inputs=None):
        """(name, launch) pairs of step i.  `inputs` (optional) supplies contiguous
        device buffers x, z [B, n_new, D], q, qI, w instead of the resident ones."""
        import compressed_sparse_attention_16_b200 as csa
        wl = self.wl
        if not self.decode:
            x = self.x if inputs is None else inputs["x"]
            z = self.z if inputs is None else inputs["z"]
            q = self.q if inputs is None else inputs["q"]
            return [
                ("compress", lambda: csa.compress_ew(x, z, wl.m, self.codes, self.scales, self.wcodes, self.wscales)),
                ("index_topk", lambda: csa.index_topk(self.ind.qI, self.ind.w, self.ind.kI, self.q_pos, self.dims,
                                                      self.idx, self.score, workspace=self.ws_i)),
                ("attend", lambda: csa.attend(q, self.codes, self.scales, self.idx, self.wcodes, self.wscales,
                                              self.q_pos, self.dims, self.out, self.lse, workspace=self.ws_a)),
            ]
        st = self.state
        j = self.step_index(i)
        t0 = self.T0 + self.n_new * j
        d = self._dims(j)
        q_pos = self.q_pos_all[j]
        if inputs is None:
            src, first = (self.x, self.z), t0
        else:
            src, first = (inputs["x"], inputs["z"]), 0
        q = self.q if inputs is None else inputs["q"]
        out = [
            ("compress", lambda: csa.compress_ew(src[0], src[1], wl.m, st.codes, st.scales, st.win_codes, st.win_scales,
                                                 dst_first=t0 // wl.m, win_first=t0, win_ring_cap=st.win_cap,
                                                 T=self.n_new, first_token=first)),
        ]
        if wl.kind == "hca_decode":
            ws = self._ws(csa.attend_workspace(d, True), "_ws_hca")
            out.append(("hca_attend", lambda: csa.hca_attend(q, st.codes, st.scales, st.win_codes, st.win_scales,
                                                             q_pos, d, st.out, st.lse, workspace=ws)))
        elif self.fused:
            qI = self.ind.qI if inputs is None else inputs["qI"]
            w = self.ind.w if inputs is None else inputs["w"]
            xs = self.x_steps[j] if inputs is None else inputs["x"]
            zs = self.z_steps[j] if inputs is None else inputs["z"]
            ws = self._ws_step
            return [("decode_step", lambda: csa.decode_step(xs, zs, None, q, qI, w, q_pos, st.codes, st.scales, st.kI,
                                                            st.win_codes, st.win_scales, d, st.idx, st.score, st.out,
                                                            st.lse, ws))]
        else:
            qI = self.ind.qI if inputs is None else inputs["qI"]
            w = self.ind.w if inputs is None else inputs["w"]
            wsi = self._ws(csa.index_topk_workspace(d), "_ws_index")
            wsa = self._ws(csa.attend_workspace(d), "_ws_attend")
            out.append(("index_topk", lambda: csa.index_topk(qI, w, st.kI, q_pos, d, st.idx, st.score, workspace=wsi)))
            out.append(("attend", lambda: csa.attend(q, st.codes, st.scales, st.idx, st.win_codes, st.win_scales,
                                                     q_pos, d, st.out, st.lse, workspace=wsa)))
        return out

    def output(self):
        return self.state.out if self.decode else self.out

    def run(self, i, inputs=None):
        for _, fn in self.calls(i, inputs):
            fn()

    def _capture_step(self, calls):
        """Issue one step's calls as a fork/join: the appends (compress) feed
        only the attention, so they run on a side stream beside the indexer
        (CSA) or beside each other (HCA); the attention waits for both."""
        torch = self.torch
        if len(calls) == 1:               # the fused decode step: one launch
            calls[0][1]()
            return
        if self._side is None:
            self._side = torch.cuda.Stream(device=self.dev)
        side, main = self._side, torch.cuda.current_stream(self.dev)
        appends = [fn for name, fn in calls if name.startswith("compress")]
        index = [fn for name, fn in calls if name == "index_topk"]
        final = [fn for name, fn in calls if not name.startswith("compress") and name != "index_topk"]
        side.wait_stream(main)
        with torch.cuda.stream(side):
            for fn in (appends if index else appends[1:]):
                fn()
        for fn in (index if index else appends[:1]):
            fn()
        main.wait_stream(side)
        for fn in final:
            fn()

    def graph(self, i, inputs=None, key=None):
        """CUDA graph of step i (captured once)."""
        import compressed_sparse_attention_16_b200 as csa
        torch = self.torch
        key = (self.step_index(i), key)
        g = self.graphs.get(key)
        if g is None:
            calls = self.calls(i, inputs)
            if not getattr(self, "_warmed", False):
                for _, fn in calls:             # first launches set kernel attributes
                    fn()
                torch.cuda.synchronize()
                self._warmed = True
            g = torch.cuda.CUDAGraph()
            n0 = csa.launch_count()
            with torch.cuda.graph(g):
                self._capture_step(calls)
            g.kernels = csa.launch_count() - n0
            self.graphs[key] = g
        return g


def max_over_ranks(ms, world, device):
    """The job's duration: the maximum of one per-rank duration over all ranks
    (an all-reduce on the default process group when world > 1)."""
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank, ms):
    """Whole-job units per second: every rank processes its own units (weak
    scaling) in at most `ms` milliseconds."""
    return world * units_per_rank / (ms / 1e3)


def l2_flush(buf):
    """Evict the L2 between timed steps: write a buffer larger than the L2, then
    read it back, so the write-backs of the dirty lines also happen here and
    not inside the next timed region."""
    import torch
    buf.fill_(1)
    buf.view(torch.int64).sum()


HEADLINE = "csa_decode_1m_incremental"
# every configuration of the library's workload set, headline first
ALL_WORKLOADS = (HEADLINE, "csa_decode_64k", "hca_decode_1m", "csa_prefill_128k", "tiny_prefill")
# timed steps and CPU-baseline budget of the workloads after the headline
SECONDARY_STEPS = 20
SECONDARY_CPU_BUDGET_S = 6.0
HBM_NOMINAL_GBS = 8000.0


def init_ranks():
    """(world, rank, local rank, device); joins the NCCL group when world > 1."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    return world, rank, local, dev


def measure(args, wl, steps, world, rank, local, dev, peaks, peaks_src, cpu_budget):
    """Time `steps` steps of one workload on every rank; rank 0 gets the
    workload's record (the other ranks None)."""
    import torch
    import torch.distributed as dist

    if args.decode_path == "auto":
        from compressed_sparse_attention_16_b200.pipeline import prefer_fused_step
        fused = prefer_fused_step(wl.B, dev)
    else:
        fused = args.decode_path == "fused"
    r = Runner(wl, seed=rank, device=dev, fused=fused)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    use_graph = r.decode and not args.no_graph

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    # warm-up (also captures the graphs of the steps to be timed)
    for i in range(args.warmup):
        if use_graph:
            r.graph(i).replay()
        else:
            r.run(i)
    if use_graph:
        for i in range(args.warmup, args.warmup + steps):
            r.graph(i)
    barrier()

    clocks = ClockSampler(local)
    clocks.start()
    step_events = []
    launches = 0
    wall0 = time.perf_counter()
    for i in range(args.warmup, args.warmup + steps):
        l2_flush(flush)                     # evict L2 between timed steps (outside the events)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if use_graph:
            g = r.graph(i)
            e0.record()
            g.replay()
            e1.record()
            launches += g.kernels
        else:
            n0 = launch_count()
            e0.record()
            r.run(i)
            e1.record()
            launches += launch_count() - n0
        step_events.append((e0, e1))
    barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in step_events), world, dev)
    ms_per_step = step_ms / steps
    value = job_throughput(world, r.units_per_step, ms_per_step)

    # per-call device time: each call alone, cold L2, queued behind a bounded
    # sleep (~1 ms, longer than the binding's host-side launch work, so the
    # events bracket device time only)
    per_call = {}
    for i in range(args.warmup, args.warmup + min(steps, 5)):
        for name, fn in r.calls(i):
            l2_flush(flush)
            torch.cuda._sleep(SLEEP_CYCLES)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            per_call.setdefault(name, []).append((a, b))
    torch.cuda.synchronize()
    call_ms = {k: float(np.mean([a.elapsed_time(b) for a, b in v])) for k, v in per_call.items()}

    e2e = e2e_leg(r, args, world, dev, use_graph, steps)
    fused = getattr(r, "fused", False)
    r.graphs.clear()
    del r, flush
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    work = op_work(wl)
    dom = max(call_ms, key=lambda k: call_ms[k])
    rec = {
        "value": value, "unit": "queries/s" if wl.kind == "prefill" else "tokens/s",
        "ms_per_step": ms_per_step, "steps": steps,
        "config": workload_config(wl, world, use_graph, fused),
        "roofline": roofline(dom, work[dom], call_ms[dom], peaks, peaks_src, wl),
        "step_hbm": step_hbm(work, ms_per_step, peaks),
        "per_call_ms": call_ms,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
        "wall_s_timed_region": wall,
    }
    if world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(wl, budget_s=cpu_budget)
    return rec


def workload_config(wl, world, use_graph, fused=False):
    return {"workload": wl.name, "B": wl.B, "T": wl.T, "m": wl.m, "K": wl.K, "W": wl.W,
            "H": wl.H, "D": wl.D, "HI": wl.HI, "dI": wl.dI,
            "l2": "flushed between timed steps (256 MiB write then read, outside the step events)",
            "launch": ("one CUDA graph per step" if use_graph else "direct C-ABI calls")
            + (" of one csa_decode_step launch" if fused else ""),
            "parallelism": f"dp{world} (independent sequences per GPU)"}


def step_hbm(work, ms, peaks):
    """Algorithmic bytes of the whole step over its time, against the measured
    copy bandwidth and the 8 TB/s nominal figure."""
    nbytes = sum(w["bytes"] for w in work.values() if not w.get("aggregate"))
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"algorithmic_bytes": nbytes, "achieved_gbs": gbs, "frac_measured": gbs / peaks["hbm_gbs"],
            "frac_8tbs": gbs / HBM_NOMINAL_GBS}


def gpu_arm(args, names):
    import torch.distributed as dist

    import synth

    world, rank, local, dev = init_ranks()
    peaks, peaks_src = load_peaks()
    recs = {}
    for k, name in enumerate(names):
        wl = synth.WORKLOADS[name]
        steps = args.steps if k == 0 else min(args.steps, SECONDARY_STEPS)
        budget = args.cpu_budget if k == 0 else min(args.cpu_budget, SECONDARY_CPU_BUDGET_S)
        recs[name] = measure(args, wl, steps, world, rank, local, dev, peaks, peaks_src, budget)
    line = None
    if rank == 0:
        head = recs[names[0]]
        line = {
            "metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": head["steps"], "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) tokens/logits, E2M1 indexer codes, bf16 queries)",
            "config": head["config"],
        }
        for key in ("roofline", "step_hbm", "per_call_ms", "e2e", "gpu_launches", "clocks",
                    "wall_s_timed_region", "cpu_baseline"):
            if key in head:
                line[key] = head[key]
        if len(names) > 1:
            line["workloads"] = {n: recs[n] for n in names}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def relaunch_with_ranks(n):
    """`bench.py --gpus N` started without torchrun: run the same command as N
    ranks on this node (one per GPU) and return their exit status."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def launch_count():
    import compressed_sparse_attention_16_b200 as csa
    return csa.launch_count()


def e2e_leg(r, args, world, dev, use_graph, steps):
    """The same step through the public API: pinned host inputs copied in and the
    attention output copied back, all inside the timed region."""
    import torch
    wl = r.wl
    if r.decode:
        t0 = r.T0
        host = {"x": r.x[:, t0:t0 + r.n_new].contiguous().cpu().pin_memory(),
                "z": r.z[:, t0:t0 + r.n_new].contiguous().cpu().pin_memory(),
                "q": r.q.cpu().pin_memory()}
        if wl.kind != "hca_decode":
            host["qI"] = r.ind.qI.cpu().pin_memory()
            host["w"] = r.ind.w.cpu().pin_memory()
    else:
        host = {"x": r.x.cpu().pin_memory(), "z": r.z.cpu().pin_memory(), "q": r.q.cpu().pin_memory()}
    out_dev = r.output()
    out_host = torch.empty(out_dev.shape, dtype=out_dev.dtype).pin_memory()
    dbuf = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()
    step = args.warmup
    g = r.graph(step, inputs=dbuf, key="e2e") if use_graph else None
    times = []
    for i in range(max(1, min(steps, 10)) + 2):
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for k in host:
            dbuf[k].copy_(host[k], non_blocking=True)
        if g is not None:
            g.replay()
        else:
            r.run(step, inputs=dbuf)
        out_host.copy_(out_dev, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    ms = max_over_ranks(np.mean(times), world, dev)
    return {"value": job_throughput(world, r.units_per_step, ms), "unit": r.unit,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms}


def roofline(name, work, ms, peaks, src, wl):
    """Roofline of the step's dominant call: tensor-bound for the attention of
    prefill and HCA decode (FLOPs against the measured bf16 peak), HBM-bound
    otherwise (algorithmic bytes against the measured copy bandwidth, and
    against the 8 TB/s nominal figure)."""
    sec = ms / 1e3
    traffic = kernel_traffic(name, wl.name)
    gbs = work["bytes"] / sec / 1e9
    if work["flops"] and wl.kind in ("prefill", "hca_decode") and name.endswith("attend"):
        achieved = work["flops"] / sec / 1e12
        peak = peaks["bf16_tflops"]
        return {"bound": "tensor", "kernel": name, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": f"bf16_tflops ({src})", "traffic": traffic,
                "algorithmic_flops": work["flops"], "algorithmic_bytes": work["bytes"], "ms": ms,
                "hbm_gbs": gbs, "hbm_frac_measured": gbs / peaks["hbm_gbs"], "hbm_frac_8tbs": gbs / HBM_NOMINAL_GBS}
    peak = peaks["hbm_gbs"]
    out = {"bound": "hbm", "kernel": name, "achieved": gbs, "peak": peak, "unit": "GB/s",
           "frac": gbs / peak, "frac_8tbs": gbs / HBM_NOMINAL_GBS, "peak_source": f"hbm_gbs ({src})",
           "traffic": traffic, "algorithmic_bytes": work["bytes"], "algorithmic_flops": work["flops"], "ms": ms}
    if work["flops"]:
        tf = work["flops"] / sec / 1e12
        out.update({"tflops": tf, "bf16_frac": tf / peaks["bf16_tflops"]})
    return out


def kernel_traffic(call, workload):
    """DRAM bytes per launch of a call from the committed ncu summary, or None
    when absent or when the kernel's sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(workload, {}).get(call)
    if not rec:
        return None
    if rec.get("source_sha") != source_sha(rec.get("kernel", "")):
        return None
    return rec.get("dram_bytes")


# the source files each profiled kernel is built from (its own file and the
# shared device headers)
KERNEL_SOURCES = {
    "attend_tc_kernel": ["attend_tc.cu"],
    "attend_prefill_kernel": ["attend_prefill.cu"],
    "index_decode_kernel<4>": ["indexer.cu"],
    "index_prefill_kernel<4>": ["index_prefill.cu"],
    "decode_step_kernel<4>": ["decode_step.cu"],
}
SHARED_SOURCES = ["common.cuh", "tc.cuh"]


def source_sha(kernel):
    """Hash of the sources a kernel is built from; unknown kernels hash every
    file of the CUDA sources."""
    csrc = os.path.join(ROOT, "compressed_sparse_attention_16_b200", "csrc")
    files = KERNEL_SOURCES.get(kernel)
    files = sorted(files + SHARED_SOURCES) if files else sorted(os.listdir(csrc))
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------


class OracleStep:
    """The oracle's version of one step on a bounded sample of the workload.

    Decode samples keep the full context length: the cache before the step
    holds random finite E4M3 entries (dequantised by the oracle), and only the
    window tokens and the appended tokens are raw values, so that building the
    sample stays cheap; the timed step is the oracle's whole step (pool the
    new tokens, score every visible entry, select, attend)."""

    def __init__(self, wl, seed=0, max_seqs=2, max_rows=64):
        import torch

        import synth
        from oracle import csa as ocsa
        self.o = ocsa
        self.wl = wl
        self.kind = wl.kind
        if wl.kind == "hca_decode":
            # 1 sequence with a 1/8-length context (1,024 entries)
            self.B = 1
            T = wl.T // 8
        elif wl.kind in ("decode", "decode_incremental"):
            self.B = min(wl.B, max_seqs)
            T = wl.T
        else:
            self.B = wl.B
            T = wl.T
        g = torch.Generator().manual_seed(seed)
        self.T = T
        n_new = wl.m if wl.kind == "hca_decode" else 4
        self.n_new = n_new
        D = wl.D
        if wl.kind == "prefill":
            self.x = torch.randn((self.B, T, D), generator=g).numpy()
            self.z = torch.randn((self.B, T, D), generator=g).numpy()
            self.rows = np.unique(np.linspace(0, T - 1, min(max_rows, T)).astype(np.int64))
            self.q = synth.queries(self.B, len(self.rows), wl.H, D, wl.q_scale, seed).view(torch.int16).numpy().view(np.uint16)
            self.ind = synth.indexer_inputs(self.B, len(self.rows), wl.N, wl.HI, wl.dI, seed)
            return
        # raw tokens of positions [base, T + n_new): the window before the step and the new tokens
        self.base = max(0, T - wl.W)
        self.x = torch.randn((self.B, T + n_new - self.base, D), generator=g).numpy()
        self.z = torch.randn((self.B, T + n_new - self.base, D), generator=g).numpy()
        self.q = synth.queries(self.B, 1, wl.H, D, wl.q_scale, seed).view(torch.int16).numpy().view(np.uint16)
        N = (T + n_new) // wl.m
        self.ind = synth.indexer_inputs(self.B, 1, N, max(wl.HI, 1), max(wl.dI, 32), seed) if wl.HI else None
        n0 = T // wl.m
        codes, scales = synth.e4m3_cache(self.B, n0, D, seed)
        self.entries = np.zeros((self.B, n0 + 1, D))
        self.entries[:, :n0] = ocsa.dequantize(codes.numpy(), scales.numpy())
        self.win = np.zeros((self.B, T + n_new - self.base, D))
        self.win[:, :T - self.base] = ocsa.window_token_values(self.x[:, :T - self.base])

    def units(self):
        return self.B * (len(self.rows) if self.kind == "prefill" else 1)

    def run(self):
        o, wl = self.o, self.wl
        if self.kind == "prefill":
            T, m = self.T, wl.m
            c, s = o.quantize_entries(o.compress(self.x[:, :T], self.z[:, :T], m))
            ent = o.dequantize(c, s)
            win = o.window_token_values(self.x[:, :T])
            s64 = o.indexer_scores64(self.ind.qI.numpy(), self.ind.w.numpy(), self.ind.kI.numpy())
            pos = self.rows[None].repeat(self.B, 0)
            idx, _ = o.topk(s64, o.n_visible(pos, m, wl.N), wl.K)
            return o.attend(self.q, ent, idx, lambda b, p: win[b, p], pos, wl.W)
        T, n_new, m, base = self.T, self.n_new, wl.m, self.base
        lo, hi = T - base, T + n_new - base
        new = o.compress(self.x[:, lo:hi], self.z[:, lo:hi], m)
        c, s = o.quantize_entries(new)
        self.entries[:, T // m] = o.dequantize(c, s)[:, 0]
        self.win[:, lo:hi] = o.window_token_values(self.x[:, lo:hi])
        t = T + n_new - 1
        pos = np.full((self.B, 1), t)
        n_ent = (T + n_new) // m
        win = lambda b, p: self.win[b, p - base]
        if self.kind == "hca_decode":
            return o.hca_attend(self.q, self.entries, win, pos, m, wl.W)
        s64 = o.indexer_scores64(self.ind.qI.numpy(), self.ind.w.numpy(), self.ind.kI[:, :n_ent].numpy())
        idx, _ = o.topk(s64, o.n_visible(pos, m, n_ent), wl.K)
        return o.attend(self.q, self.entries, idx, win, pos, wl.W)

    def describe(self):
        wl = self.wl
        if self.kind == "prefill":
            return (f"{self.B} sequence(s) of {self.T} tokens: whole-sequence pooling, then indexer, top-k and "
                    f"attention for {len(self.rows)} evenly spaced query rows")
        if self.kind == "hca_decode":
            return (f"1 sequence, context {self.T} tokens (1/8 of the workload's; {self.T // wl.m} entries): "
                    "append 128 tokens + dense attention")
        return (f"{self.B} of {wl.B} sequences, full {self.T}-token context (cache of random finite E4M3 "
                "entries): append 4 tokens + index + top-k + attend")


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s=15.0):
    st = OracleStep(wl, max_rows=64 if budget_s >= 15.0 else 16)
    st.run()                          # warm (allocations, BLAS threads)
    t0 = time.perf_counter()
    n = 0
    while True:
        st.run()
        n += 1
        if time.perf_counter() - t0 > budget_s or n >= 50:
            break
    dt = (time.perf_counter() - t0) / n
    out = {"value": st.units() / dt, "unit": "tokens/s" if wl.kind != "prefill" else "queries/s",
           "cores": cpu_cores(), "kind": "oracle", "sample": st.describe(), "sec_per_sample": dt}
    if wl.kind == "prefill":
        # the rate of the sampled rows, extrapolated to every row of the workload
        out["extrapolated"] = True
        out["extrapolated_full_step_s"] = wl.B * wl.T / out["value"]
    return out


def reference_arm(args, wl, others=()):
    """The oracle timed on the host cores (rank 0 only): `args.steps` steps of
    the bounded sample of `wl`, plus one step of each workload in `others`."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None

    def run(w, steps, warmup):
        st = OracleStep(w)
        for _ in range(warmup):
            st.run()
        t0 = time.perf_counter()
        for _ in range(steps):
            st.run()
        dt = (time.perf_counter() - t0) / steps
        return st, dt

    st, dt = run(wl, args.steps, args.warmup)
    unit = "tokens/s" if wl.kind != "prefill" else "queries/s"
    value = st.units() / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "m": wl.m, "K": wl.K, "W": wl.W,
                       "H": wl.H, "D": wl.D},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cpu_cores(), "kind": "oracle",
                             "sample": st.describe()},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if others:
        line["workloads"] = {}
        for w in others:
            so, d = run(w, 1, 0)
            u = "tokens/s" if w.kind != "prefill" else "queries/s"
            line["workloads"][w.name] = {"value": so.units() / d, "unit": u, "ms_per_step": d * 1e3,
                                         "sample": so.describe(), "cores": cpu_cores()}
    return line


def kernel_case(args, wl):
    """One library call of the workload, alone, on inputs of the workload's
    shape (no raw-token context): a small, repeatable target for profilers.
    Cases: index_topk, attend, hca_attend, compress_entry."""
    import torch

    import compressed_sparse_attention_16_b200 as csa
    import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, D, H, m, K, W = wl.B, wl.D, wl.H, wl.m, max(wl.K, 1), wl.W
    decode = wl.kind != "prefill"
    Tq = 1 if decode else (args.rows or wl.T)
    N = wl.N
    # prefill: the last Tq positions of the sequence (the heaviest rows)
    q_pos = (torch.full((B, 1), wl.T - 1, dtype=torch.int32, device=dev) if decode
             else (wl.T - Tq + torch.arange(Tq, dtype=torch.int32, device=dev)).repeat(B, 1).contiguous())
    d = csa.Dims(B=B, Tq=Tq, H=H, D=D, HI=max(wl.HI, 1), dI=max(wl.dI, 32), K=K, W=W, m=m, n_entries=N,
                 entry_cap=N, win_cap=W if decode else wl.T)
    case = args.kernel_case
    if case == "index_topk":
        ind = synth.indexer_inputs(B, Tq, N, wl.HI, wl.dI, 0, device=dev)
        idx = torch.empty((B, Tq, K), dtype=torch.int32, device=dev)
        sc = torch.empty((B, Tq, K), device=dev)
        ws = torch.empty(max(1, csa.index_topk_workspace(d)), dtype=torch.uint8, device=dev)
        fn = lambda: csa.index_topk(ind.qI, ind.w, ind.kI, q_pos, d, idx, sc, workspace=ws)
    elif case in ("attend", "hca_attend"):
        codes, scales = synth.e4m3_cache(B, N, D, 0, device=dev)
        wcodes, wscales = synth.e4m3_cache(B, d.win_cap, D, 0, device=dev, tag="win")
        q = synth.queries(B, Tq, H, D, wl.q_scale, 0, device=dev)
        out = torch.empty((B, Tq, H, D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, Tq, H), device=dev)
        dense = case == "hca_attend"
        ws = torch.empty(max(1, csa.attend_workspace(d, dense)), dtype=torch.uint8, device=dev)
        if dense:
            fn = lambda: csa.hca_attend(q, codes, scales, wcodes, wscales, q_pos, d, out, lse, workspace=ws)
        else:
            # K distinct entries per row: a random offset plus a fixed random pattern of distinct steps
            g = torch.Generator(device=dev).manual_seed(0)
            base = torch.randperm(N, generator=g, device=dev)[:K]
            shift = torch.randint(0, N, (B * Tq, 1), generator=g, device=dev)
            idx = ((base[None] + shift) % N).to(torch.int32).view(B, Tq, K).contiguous()
            fn = lambda: csa.attend(q, codes, scales, idx, wcodes, wscales, q_pos, d, out, lse, workspace=ws)
    elif case == "compress_entry":
        n_tok = wl.m if wl.kind == "hca_decode" else (4 if decode else wl.T)
        x, z = synth.tokens(B, n_tok, D, 0, device=dev)
        codes = torch.empty((B, max(1, n_tok // m), D), dtype=torch.uint8, device=dev)
        scales = torch.empty((B, max(1, n_tok // m)), device=dev)
        fn = lambda: csa.compress(x, z, m, codes, scales)
    elif case == "quantize_mxfp4":
        # fp32 indexer queries of the workload (B * Tq * HI rows of dI values) to MXFP4
        rows = B * Tq * max(wl.HI, 1)
        cols = max(wl.dI, 32)
        g = torch.Generator(device=dev).manual_seed(0)
        xq = torch.randn((rows, cols), generator=g, device=dev)
        qcodes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
        qscales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)
        case_bytes = rows * cols * 4 + rows * cols // 2 + rows * cols // 32
        fn = lambda: csa.quantize_mxfp4(xq, qcodes, qscales)
    else:
        raise SystemExit(f"unknown kernel case {case}")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        l2_flush(flush)
        torch.cuda._sleep(SLEEP_CYCLES)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        times.append((a, b))
    torch.cuda.synchronize()
    csa.sync_status()
    ms = [a.elapsed_time(b) for a, b in times]
    line = {"kernel_case": case, "workload": wl.name, "ms_mean": float(np.mean(ms)),
            "ms_min": float(np.min(ms)), "calls": args.steps,
            "device_bytes": int(torch.cuda.max_memory_allocated(dev))}
    if case == "quantize_mxfp4":
        peaks, src = load_peaks()
        gbs = case_bytes / (float(np.mean(ms)) / 1e3) / 1e9
        line.update({"algorithmic_bytes": int(case_bytes), "achieved_gbs": gbs,
                     "frac_of_hbm": gbs / peaks["hbm_gbs"], "peak_source": src})
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all",
                    help="one workload, or 'all' (the 1M-context incremental decode first, then every "
                         "other configuration)")
    ap.add_argument("--impl", default="csa", choices=["csa", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch decode steps without CUDA graphs")
    ap.add_argument("--decode-path", default="auto", choices=["auto", "separate", "fused"],
                    help="CSA decode steps as the separate calls (compress, index_topk, attend), as one "
                         "csa_decode_step launch, or (auto) whichever pipeline.prefer_fused_step picks")
    ap.add_argument("--rows", type=int, default=0, help="kernel-case: query rows of a prefill workload")
    ap.add_argument("--kernel-case", default=None,
                    help="run one library call (index_topk, attend, hca_attend, compress_entry, "
                         "quantize_mxfp4, decode_step) alone on inputs of the workload's shape; for profilers")
    args = ap.parse_args()
    import synth
    world_env = os.environ.get("WORLD_SIZE")
    if args.gpus > 1 and world_env is None:
        sys.exit(relaunch_with_ranks(args.gpus))
    if world_env is not None and int(world_env) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world_env}")
    names = ALL_WORKLOADS if args.workload == "all" else (args.workload,)
    for n in names:
        if n not in synth.WORKLOADS:
            sys.exit(f"bench.py: unknown workload {n}")
    if args.kernel_case:
        kernel_case(args, synth.WORKLOADS[names[0]])
        return
    if args.impl == "reference":
        line = reference_arm(args, synth.WORKLOADS[names[0]], [synth.WORKLOADS[n] for n in names[1:]])
    else:
        if args.warmup < 3:
            args.warmup = 3
        line = gpu_arm(args, names)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
