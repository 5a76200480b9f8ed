#!/usr/bin/env python3
"""Benchmark of the hybrid compressed-attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Workloads (synthetic, seeded): csa_decode_64k (default), csa_decode_1m_incremental,
hca_decode_1m, csa_prefill_128k, tiny_prefill.  A step is one pass of the whole path
for one batch: decode -> append 4 tokens (pool one entry + 4 window tokens), indexer +
top-k, attention; HCA decode -> append 128 tokens (one entry + window) then dense
attention; prefill -> pool the whole sequence, index + select every position, attend.

Prints ONE JSON line (rank 0).  With N > 1 (torchrun) every rank runs its own
independent sequences (weak scaling, no collective on the data path); times are the
max over ranks.
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
        w["compress_entry"] = dict(bytes=raw + B * (n_new // m) * ent, flops=0)
        w["compress_window"] = dict(bytes=raw + B * n_new * ent, flops=0)
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
    else:   # prefill
        T, N = wl.T, wl.N
        w["compress_entry"] = dict(bytes=B * T * D * 8 + B * N * ent, flops=0)
        w["compress_window"] = dict(bytes=B * T * D * 8 + B * T * ent, flops=0)
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
    """Holds one workload's device state and runs steps of it."""

    def __init__(self, wl, seed, device):
        import torch

        import synth
        from compressed_sparse_attention_16_b200 import pipeline

        self.torch = torch
        self.wl = wl
        self.dev = device
        torch.cuda.set_device(device)
        self.calls = {}
        if wl.kind in ("decode", "decode_incremental", "hca_decode"):
            self.n_new = 4 if wl.kind != "hca_decode" else wl.m
            steps_cap = max(wl.steps, 1) + 1024 if wl.kind == "decode_incremental" else 1
            self.T0 = wl.T if wl.kind == "decode_incremental" else wl.T - self.n_new
            Ttot = self.T0 + self.n_new * steps_cap
            self.x, self.z = synth.tokens(wl.B, Ttot, wl.D, seed, device=device)
            dense = wl.kind == "hca_decode"
            cap = Ttot // wl.m
            self.state = pipeline.DecodeState(wl.B, wl.D, wl.H, wl.m, wl.W, entry_cap=cap, K=max(wl.K, 1),
                                              HI=max(wl.HI, 1), dI=max(wl.dI, 32), dense=dense)
            if not dense:
                self.ind = synth.indexer_inputs(wl.B, 1, cap, wl.HI, wl.dI, seed, device=device)
                self.state.kI.copy_(self.ind.kI)
            self.q = synth.queries(wl.B, 1, wl.H, wl.D, wl.q_scale, seed, device=device)
            self.state.prefill_context(self.x, self.z, self.T0)
            self.step_i = 0
            self.units_per_step = wl.B
            self.unit = "tokens/s"
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

    # -- one step, each library call bracketed by events when `ev` is given ----
    def _call(self, name, ev, fn):
        if ev is None:
            fn()
            return
        e0 = self.torch.cuda.Event(enable_timing=True)
        e1 = self.torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ev.append((name, e0, e1))

    def _decode_t0(self):
        if self.wl.kind == "decode_incremental":
            return self.T0 + self.n_new * self.step_i
        return self.T0            # decode / hca_decode: the same last block every step

    def step(self, ev=None, inputs=None):
        """One step on the current stream; q_pos was set by prepare_step()."""
        import compressed_sparse_attention_16_b200 as csa
        wl = self.wl
        if wl.kind in ("decode", "decode_incremental", "hca_decode"):
            st = self.state
            t0 = self._decode_t0()
            st.n_tokens = t0
            xs = (self.x[:, t0:t0 + self.n_new] if inputs is None else inputs["x"]).contiguous()
            zs = (self.z[:, t0:t0 + self.n_new] if inputs is None else inputs["z"]).contiguous()
            q = self.q if inputs is None else inputs["q"]
            first = st.n_entries
            self._call("compress_entry", ev, lambda: csa.compress(xs, zs, wl.m, st.codes, st.scales, dst_first=first))
            self._call("compress_window", ev, lambda: csa.compress(xs, zs, 1, st.win_codes, st.win_scales,
                                                                    dst_first=t0, ring_cap=st.win_cap))
            st.n_tokens = t0 + self.n_new
            if wl.kind == "decode_incremental":
                self.step_i += 1
            d = st.dims()
            if wl.kind == "hca_decode":
                self._call("hca_attend", ev, lambda: csa.hca_attend(q, st.codes, st.scales, st.win_codes,
                                                                    st.win_scales, st.q_pos, d, st.out, st.lse,
                                                                    workspace=self._ws(d, "attend_dense")))
            else:
                qI = self.ind.qI if inputs is None else inputs["qI"]
                w = self.ind.w if inputs is None else inputs["w"]
                self._call("index_topk", ev, lambda: csa.index_topk(qI, w, st.kI, st.q_pos, d, st.idx, st.score,
                                                                    workspace=self._ws(d, "index")))
                self._call("attend", ev, lambda: csa.attend(q, st.codes, st.scales, st.idx, st.win_codes,
                                                            st.win_scales, st.q_pos, d, st.out, st.lse,
                                                            workspace=self._ws(d, "attend")))
            return st.out
        x = self.x if inputs is None else inputs["x"]
        z = self.z if inputs is None else inputs["z"]
        q = self.q if inputs is None else inputs["q"]
        self._call("compress_entry", ev, lambda: csa.compress(x, z, wl.m, self.codes, self.scales))
        self._call("compress_window", ev, lambda: csa.compress(x, z, 1, self.wcodes, self.wscales))
        self._call("index_topk", ev, lambda: csa.index_topk(self.ind.qI, self.ind.w, self.ind.kI, self.q_pos,
                                                            self.dims, self.idx, self.score, workspace=self.ws_i))
        self._call("attend", ev, lambda: csa.attend(q, self.codes, self.scales, self.idx, self.wcodes,
                                                    self.wscales, self.q_pos, self.dims, self.out, self.lse,
                                                    workspace=self.ws_a))
        return self.out

    def _ws(self, d, kind):
        import compressed_sparse_attention_16_b200 as csa
        nb = csa.index_topk_workspace(d) if kind == "index" else csa.attend_workspace(d, kind == "attend_dense")
        key = "_ws_" + kind
        cur = getattr(self, key, None)
        if nb and (cur is None or cur.numel() < nb):
            cur = self.torch.empty(int(nb * 1.05) + 256, dtype=self.torch.uint8, device=self.dev)
            setattr(self, key, cur)
        return cur if nb else None

    def prepare_step(self):
        """Set the decode query position for the next step (a device write issued
        before the step's events)."""
        if self.wl.kind in ("decode", "decode_incremental", "hca_decode"):
            self.state.q_pos.fill_(self._decode_t0() + self.n_new - 1)


def gpu_arm(args, wl):
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
    peaks, peaks_src = load_peaks()
    r = Runner(wl, seed=rank, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        r.prepare_step()
        r.step()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    evs = []
    step_events = []
    launches0 = launch_count()
    wall0 = time.perf_counter()
    for _ in range(args.steps):
        flush.fill_(1)                      # evict L2 between timed steps
        r.prepare_step()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ev = []
        e0.record()
        r.step(ev)
        e1.record()
        step_events.append((e0, e1))
        evs.append(ev)
    barrier()
    wall = time.perf_counter() - wall0
    launches = launch_count() - launches0
    clk = clocks.stop()
    step_ms = float(sum(a.elapsed_time(b) for a, b in step_events))
    per_call = {}
    for ev in evs:
        for name, a, b in ev:
            per_call.setdefault(name, []).append(a.elapsed_time(b))
    t = torch.tensor([step_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    step_ms = float(t.item())
    ms_per_step = step_ms / args.steps
    value = world * r.units_per_step / (ms_per_step / 1e3)

    # e2e: pinned host inputs -> device, step, result -> host, all timed
    e2e = e2e_leg(r, args, world, dev)

    line = None
    if rank == 0:
        work = op_work(wl)
        call_ms = {k: float(np.mean(v)) for k, v in per_call.items()}
        dom = max(call_ms, key=lambda k: call_ms[k])
        roof = roofline(dom, work[dom], call_ms[dom], peaks, peaks_src, wl)
        line = {
            "metric": METRIC, "value": value, "unit": r.unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
            "data": "synthetic (seeded N(0,1) tokens/logits, E2M1 indexer codes, bf16 queries)",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "m": wl.m, "K": wl.K, "W": wl.W,
                       "H": wl.H, "D": wl.D, "HI": wl.HI, "dI": wl.dI,
                       "l2": "flushed between timed steps (256 MiB write, outside the step events)",
                       "parallelism": f"dp{world} (independent sequences per GPU)"},
            "roofline": roof,
            "per_call_ms": call_ms,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "wall_s_timed_region": wall,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def launch_count():
    import compressed_sparse_attention_16_b200 as csa
    return csa.launch_count()


def e2e_leg(r, args, world, dev):
    """Same step through the public API with pinned host inputs copied in and the
    attention output copied back inside the timed region."""
    import torch
    wl = r.wl
    if wl.kind in ("decode", "decode_incremental", "hca_decode"):
        st = r.state
        t0 = r.T0
        host = {"x": r.x[:, t0:t0 + r.n_new].contiguous().cpu().pin_memory(),
                "z": r.z[:, t0:t0 + r.n_new].contiguous().cpu().pin_memory(),
                "q": r.q.cpu().pin_memory()}
        if wl.kind != "hca_decode":
            host["qI"] = r.ind.qI.cpu().pin_memory()
            host["w"] = r.ind.w.cpu().pin_memory()
        out_host = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    else:
        host = {"x": r.x.cpu().pin_memory(), "z": r.z.cpu().pin_memory(), "q": r.q.cpu().pin_memory()}
        out_host = torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory()
    dbuf = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()
    saved_i = getattr(r, "step_i", None)
    n = max(1, min(args.steps, 10))
    times = []
    for i in range(n + 2):
        if saved_i is not None and wl.kind == "decode_incremental":
            r.step_i = saved_i
        r.prepare_step()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for k in host:
            dbuf[k].copy_(host[k], non_blocking=True)
        out = r.step(inputs=dbuf)
        out_host.copy_(out, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    ms = float(np.mean(times))
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    return {"value": world * r.units_per_step / (ms / 1e3), "unit": r.unit,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms}


def roofline(name, work, ms, peaks, src, wl):
    sec = ms / 1e3
    traffic = kernel_traffic(name, wl.name)
    if work["flops"] and wl.kind in ("prefill", "hca_decode") and name.endswith("attend"):
        achieved = work["flops"] / sec / 1e12
        peak = peaks["bf16_tflops"]
        return {"bound": "tensor", "kernel": name, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": f"bf16_tflops ({src})", "traffic": traffic,
                "algorithmic_flops": work["flops"], "algorithmic_bytes": work["bytes"], "ms": ms}
    achieved = work["bytes"] / sec / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": f"hbm_gbs ({src})", "traffic": traffic,
            "algorithmic_bytes": work["bytes"], "algorithmic_flops": work["flops"], "ms": ms}


def kernel_traffic(call, workload):
    """DRAM bytes per launch of a call from the committed ncu summary, or None
    when absent or when the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(workload, {}).get(call)
    if not rec:
        return None
    if rec.get("source_sha") != source_sha():
        return None
    return rec.get("dram_bytes")


def source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "compressed_sparse_attention_16_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------


class OracleStep:
    """The oracle's version of one step on a bounded sample of the workload."""

    def __init__(self, wl, seed=0, max_seqs=2, max_rows=64):
        import torch

        import synth
        from oracle import csa as ocsa
        self.o = ocsa
        self.wl = wl
        self.kind = wl.kind
        if wl.kind == "hca_decode":
            # 1 sequence with a 1/8-length context (1,024 entries): the oracle builds
            # its cache outside the timed step
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
        self.x = torch.randn((self.B, T + n_new, D), generator=g).numpy()
        self.z = torch.randn((self.B, T + n_new, D), generator=g).numpy()
        if wl.kind == "prefill":
            self.rows = np.unique(np.linspace(0, T - 1, min(max_rows, T)).astype(np.int64))
            self.q = synth.queries(self.B, len(self.rows), wl.H, D, wl.q_scale, seed).view(torch.int16).numpy().view(np.uint16)
            ind = synth.indexer_inputs(self.B, len(self.rows), wl.N, wl.HI, wl.dI, seed)
        else:
            self.q = synth.queries(self.B, 1, wl.H, D, wl.q_scale, seed).view(torch.int16).numpy().view(np.uint16)
            N = (T + n_new) // wl.m
            ind = synth.indexer_inputs(self.B, 1, N, max(wl.HI, 1), max(wl.dI, 32), seed) if wl.HI else None
        self.ind = ind
        if wl.kind != "prefill":
            # the cache state before the step (built once, untimed)
            n0 = T // wl.m
            c, s = ocsa.quantize_entries(ocsa.compress(self.x[:, :T], self.z[:, :T], wl.m))
            self.entries = np.zeros((self.B, n0 + 1, D))
            self.entries[:, :n0] = ocsa.dequantize(c, s)
            self.win = np.zeros((self.B, T + n_new, D))
            lo = max(0, T - wl.W)
            self.win[:, lo:T] = ocsa.window_token_values(self.x[:, lo:T])

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
        T, n_new, m = self.T, self.n_new, wl.m
        new = o.compress(self.x[:, T:T + n_new], self.z[:, T:T + n_new], m)
        c, s = o.quantize_entries(new)
        self.entries[:, T // m] = o.dequantize(c, s)[:, 0]
        self.win[:, T:T + n_new] = o.window_token_values(self.x[:, T:T + n_new])
        t = T + n_new - 1
        pos = np.full((self.B, 1), t)
        n_ent = (T + n_new) // m
        if self.kind == "hca_decode":
            return o.hca_attend(self.q, self.entries, lambda b, p: self.win[b, p], pos, m, wl.W)
        s64 = o.indexer_scores64(self.ind.qI.numpy(), self.ind.w.numpy(), self.ind.kI[:, :n_ent].numpy())
        idx, _ = o.topk(s64, o.n_visible(pos, m, n_ent), wl.K)
        return o.attend(self.q, self.entries, idx, lambda b, p: self.win[b, p], pos, wl.W)

    def describe(self):
        wl = self.wl
        if self.kind == "prefill":
            return (f"{self.B} sequence(s) of {self.T} tokens: whole-sequence pooling, then indexer, top-k and "
                    f"attention for {len(self.rows)} evenly spaced query rows")
        if self.kind == "hca_decode":
            return (f"1 sequence, context {self.T} tokens (1/8 of the workload's; {self.T // wl.m} entries): "
                    "append 128 tokens + dense attention")
        return f"{self.B} of {wl.B} sequences, full {self.T}-token context: append 4 tokens + index + top-k + attend"


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s=15.0):
    st = OracleStep(wl)
    st.run()                          # warm (allocations, BLAS threads)
    t0 = time.perf_counter()
    n = 0
    while True:
        st.run()
        n += 1
        if time.perf_counter() - t0 > budget_s or n >= 50:
            break
    dt = (time.perf_counter() - t0) / n
    return {"value": st.units() / dt, "unit": "tokens/s" if wl.kind != "prefill" else "queries/s",
            "cores": cpu_cores(), "kind": "oracle", "sample": st.describe(), "sec_per_sample": dt}


def reference_arm(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    st = OracleStep(wl)
    for _ in range(args.warmup):
        st.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        st.run()
    dt = (time.perf_counter() - t0) / args.steps
    unit = "tokens/s" if wl.kind != "prefill" else "queries/s"
    value = st.units() / dt
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "m": wl.m, "K": wl.K, "W": wl.W,
                       "H": wl.H, "D": wl.D},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cpu_cores(), "kind": "oracle",
                             "sample": st.describe()},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="csa_decode_64k")
    ap.add_argument("--impl", default="csa", choices=["csa", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    import synth
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        line = reference_arm(args, wl)
    else:
        if args.warmup < 3:
            args.warmup = 3
        line = gpu_arm(args, wl)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
