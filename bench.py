#!/usr/bin/env python
"""AQUA decode benchmark on B200: decode queries/s and HBM GB/s (fraction of the
measured B200 copy bandwidth) on a Llama-3.1-8B-shaped attention layer.

A step is one pass of the decode hot path over one batch: the new tokens' key
projection + append, query projection + magnitude top-k, and the
sparse-dimension split-K attention with its combine -- one aqua_decode_attn
call carrying the step's k_new/v_new (two kernel launches).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl aqua|reference]

Multi-GPU runs (torchrun) are independent replicas: every rank runs the same
workload on its own GPU with no collective on the data path (weak scaling);
the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "AQUA decode queries/s and HBM GB/s (% of B200 peak) at Llama-8B shape"
UNIT = "queries/s"
WORKLOADS = {
    # Llama-3.1-8B attention layer, bf16 cache, one new token per step
    "llama3.1-8b-decode": dict(B=8, Hq=32, Hkv=8, T=8192, k=96, kv="bf16", d_store=128),
    # long context, split-K over tokens
    "long-context-decode": dict(B=1, Hq=32, Hkv=8, T=131072, k=96, kv="bf16", d_store=128),
    # tiny f32 case (launch-bound)
    "tiny-f32-decode": dict(B=1, Hq=4, Hkv=1, T=1024, k=96, kv="f32", d_store=128),
    # AQUA-Memory at the Llama decode shape: the first 96 projected key AND value
    # dimensions stored, k = 64 chosen within the keys' 96
    "aqua-memory-decode": dict(B=8, Hq=32, Hkv=8, T=8192, k=64, kv="bf16", d_store=96, dv_store=96),
}
DEFAULT_WORKLOAD = "llama3.1-8b-decode"
# chunked causal prefill: a 4096-token prompt in 512-token chunks (Llama-3.1-8B heads)
PREFILL = dict(B=1, Hq=32, Hkv=8, L_total=4096, chunk=512, k=96)
# the same prompt on a truncated cache (AQUA-Memory: the first m projected key
# dimensions stored), k chosen within them
PREFILL_TRUNC = dict(PREFILL, d_store=96, k=64)
# truncated cache (first m projected dims stored), k within them, H2O budget of
# `recent` newest + heavy hitters; absolute length runs from `budget` to T_end
H2O_WL = dict(B=32, Hq=32, Hkv=8, m=96, k=64, budget=2048, recent=256, T_end=32768)
# break-even sweep over the context length and k at the Llama decode shape (one
# cache built at the largest T; shorter contexts rewind the lengths)
T_SWEEP = dict(B=8, Hq=32, Hkv=8, kv="bf16", d_store=128, Ts=(2048, 8192, 32768), ks=(128, 96, 64, 32))
T_SWEEP_FULL_TS = (512, 1024, 2048, 4096, 8192, 16384, 32768)
L2_BYTES = 126e6
FALLBACK_HBM_GBS = 6650.0


def profile_traffic(kernel: str, source: str):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    traffic record (profiles/ncu_traffic.json, one entry per kernel with the
    sha256 of the source it was captured from), or None when the kernel's
    source changed since that capture."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))[kernel]
        digest = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()
        if rec.get("source_sha256") != digest:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, 1590.0, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons during the timed region: an NVML thread
    polling every 2 ms (read-only queries), else nvidia-smi at its shortest loop."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import threading
        self.proc = None
        self.sm, self.smax, self.reasons = [], [], set()
        self.stop_evt = threading.Event()
        self.thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(ident)
            self.nv = pynvml
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "10"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def _poll(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                self.smax.append(float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS:
                    if r & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            self.stop_evt.wait(0.002)

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=2)
            return {"sm_mhz": statistics.median(self.sm) if self.sm else None,
                    "sm_max_mhz": max(self.smax) if self.smax else None,
                    "reasons": sorted(self.reasons), "samples": len(self.sm), "source": "nvml"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "no clock source"}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.strip().splitlines():
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi"}


# ----------------------------------------------------------------------------- distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Maximum of x over the ranks (the timing of a multi-GPU run is the slowest
    rank's).  The reduction tensor lives where the process group's backend
    works: on the GPU for nccl, on the host for gloo."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank processes its own replica of
    the workload (weak scaling), timed by the slowest rank."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


# ----------------------------------------------------------------------------- AQUA arm
class DecodeBench:
    def __init__(self, wl: dict, steps: int, warmup: int, P=None):
        """P: optional projection [Hkv, d, d] (f32, on the device); by default the
        offline step computes it from the calibration matrix on the GPU."""
        import torch
        import sparse_dimension_attention_b200 as aq
        from sparse_dimension_attention_b200 import build
        build.build()
        self.aq, self.torch = aq, torch
        self.wl = wl
        B, Hq, Hkv, T, kv = wl["B"], wl["Hq"], wl["Hkv"], wl["T"], wl["kv"]
        self.dt = torch.bfloat16 if kv == "bf16" else torch.float32
        self.esize = 2 if kv == "bf16" else 4
        n_steps = max(steps, warmup, 1) + 1
        self.n_in = n_steps
        if P is not None:
            self.P = P[:Hkv].contiguous()
        else:
            # offline step: P from the calibration matrix, on the GPU
            X = torch.from_numpy(synth.calibration_matrix()).cuda()
            P1 = torch.empty((128, 128), dtype=torch.float32, device="cuda")
            sig = torch.empty((128,), dtype=torch.float32, device="cuda")
            ws = torch.empty(aq.aqua_calibrate_workspace_size(X.shape[0], 128), dtype=torch.uint8, device="cuda")
            aq.aqua_calibrate(X, P1, sig, ws)
            self.P = P1.unsqueeze(0).expand(Hkv, 128, 128).contiguous()
        # history of T-1 tokens so the first step attends T
        inp = synth.decode_inputs(B, Hq, Hkv, T - 1, bf16=(kv == "bf16"), steps=n_steps)
        self.T0 = T - 1
        self.cache = aq.AquaCache(B, Hkv, T + n_steps + 64, d_store=wl["d_store"], dtype=self.dt,
                                  dv_store=wl.get("dv_store"))
        self.vcols = wl.get("dv_store") or 128          # stored value dims
        chunk = 4096
        for s in range(0, T - 1, chunk):
            e = min(T - 1, s + chunk)
            kt = torch.from_numpy(np.ascontiguousarray(inp["k_hist"][:, s:e])).to(self.dt).cuda()
            vt = torch.from_numpy(np.ascontiguousarray(inp["v_hist"][:, s:e])).to(self.dt).cuda()
            aq.aqua_project_keys(self.cache.desc, kt, vt, self.P, e - s)
        torch.cuda.synchronize()
        del inp["k_hist"], inp["v_hist"]
        self.q_h = torch.from_numpy(inp["q"]).to(self.dt).pin_memory()                       # [S, B, Hq, d]
        self.k_h = torch.from_numpy(inp["k_new"]).to(self.dt).pin_memory()                   # [S, B, Hkv, d]
        self.v_h = torch.from_numpy(inp["v_new"]).to(self.dt).pin_memory()
        # the same inputs packed per step (q | k_new | v_new) for one host->device copy per step
        self.in_h = torch.cat([self.q_h.reshape(n_steps, -1), self.k_h.reshape(n_steps, -1),
                               self.v_h.reshape(n_steps, -1)], dim=1).pin_memory()
        self.q_d = self.q_h.cuda()
        self.k_d = self.k_h.cuda()
        self.v_d = self.v_h.cuda()
        self.out = torch.empty((B, Hq, 128), dtype=self.dt, device="cuda")
        self.out_h = torch.empty((B, Hq, 128), dtype=self.dt).pin_memory()
        self.ws = torch.zeros(aq.aqua_decode_workspace_size(self.cache.desc, Hq), dtype=torch.uint8, device="cuda")
        self.sel = torch.empty((B, Hq, 128), dtype=torch.int32, device="cuda")

    def rewind(self):
        self.cache.len.fill_(self.T0)
        self.cache.n_abs.fill_(self.T0)
        self.cache.desc.max_len = self.T0

    def step(self, s: int, k: int, sel=None):
        aq, wl = self.aq, self.wl
        aq.aqua_decode_attn(self.cache.desc, self.q_d[s], self.P, wl["Hq"], k, self.out, self.ws,
                            k_new=self.k_d[s], v_new=self.v_d[s], sel_out=sel)

    def step_unfused(self, s: int, k: int):
        aq, wl = self.aq, self.wl
        aq.aqua_project_keys(self.cache.desc, self.k_d[s][:, None], self.v_d[s][:, None], self.P, 1)
        aq.aqua_decode_attn(self.cache.desc, self.q_d[s], self.P, wl["Hq"], k, self.out, self.ws)

    def union_sizes(self, k: int, n: int):
        """|U| per (b, g) for the first n steps' queries (selection depends on q and P only)."""
        torch, wl = self.torch, self.wl
        G = wl["Hq"] // wl["Hkv"]
        sizes = []
        for s in range(n):
            self.rewind()
            sel = torch.empty((wl["B"], wl["Hq"], k), dtype=torch.int32, device="cuda")
            self.step(s, k, sel)
            m = torch.zeros((wl["B"], wl["Hq"], 128), dtype=torch.bool, device="cuda")
            m.scatter_(2, sel.long(), True)
            u = m.view(wl["B"], wl["Hkv"], G, 128).any(2).sum(-1)          # [B, Hkv]
            sizes.append(u.cpu().numpy())
        self.rewind()
        return np.stack(sizes)                                               # [n, B, Hkv]

    def bytes_decode(self, usz: np.ndarray, T: int) -> float:
        """Algorithmic HBM bytes of one aqua_decode_attn call at T tokens per sequence:
        union rows of K~ and stored V rows (per (b, g) and token), q read, output write."""
        wl, e = self.wl, self.esize
        d = 128
        return float(T * np.sum(e * usz + e * self.vcols) + wl["B"] * wl["Hq"] * d * e * 2)

    def bytes_append(self) -> float:
        wl, e = self.wl, self.esize
        # read k, v; write the k~ column and the (projected) value row
        return float(wl["B"] * wl["Hkv"] * (128 * e * 2 + wl["d_store"] * e + self.vcols * e))

    def bytes_attend(self, usz: np.ndarray, T: int) -> float:
        """Algorithmic HBM bytes of the attention kernel alone: union rows of K~
        and stored V rows per (b, g) and token, and the output write."""
        wl, e = self.wl, self.esize
        return float(T * np.sum(e * usz + e * self.vcols) + wl["B"] * wl["Hq"] * 128 * e)

    def kernel_times(self, K: int, k: int):
        """Each kernel of the decode step timed alone with CUDA events on the
        launching stream: K steps issued as aqua_decode_select (projection
        kernel with the fused append) and aqua_decode_attend (attention
        kernel), with an event before, between and after.  An event between
        the two launches serialises the attention kernel behind the projection
        kernel (no programmatic overlap), so each interval is one kernel's
        duration.  A sleep kernel in front keeps the GPU busy while the host
        enqueues all K steps, so no interval includes host launch gaps.
        Returns the mean select and attend durations in ms."""
        torch, aq, wl = self.torch, self.aq, self.wl
        st = torch.cuda.current_stream()
        self.rewind()
        for s in range(3):                                   # warm (first launches configure the kernels)
            aq.aqua_decode_select(self.cache.desc, self.q_d[s], self.P, wl["Hq"], k, self.ws,
                                  k_new=self.k_d[s], v_new=self.v_d[s])
            aq.aqua_decode_attend(self.cache.desc, wl["Hq"], self.out, self.ws, appended=True, P=self.P)
        torch.cuda.synchronize()
        self.rewind()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        torch.cuda._sleep(int(2e6 + K * 1e5))                # ~1 ms + 50 us per step of GPU time
        for s in range(K):
            i = s % self.n_in
            ev[s][0].record(st)
            aq.aqua_decode_select(self.cache.desc, self.q_d[i], self.P, wl["Hq"], k, self.ws,
                                  k_new=self.k_d[i], v_new=self.v_d[i])
            ev[s][1].record(st)
            aq.aqua_decode_attend(self.cache.desc, wl["Hq"], self.out, self.ws, appended=True, P=self.P)
            ev[s][2].record(st)
        torch.cuda.synchronize()
        sel = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
        att = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
        self.rewind()
        return sel, att

    def timed_unfused(self, K: int, W: int, k: int):
        """The same steps as two public calls (aqua_project_keys, then aqua_decode_attn)."""
        torch = self.torch
        self.rewind()
        for s in range(W):
            self.step_unfused(s % self.n_in, k)
        torch.cuda.synchronize()
        self.rewind()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s in range(K):
            self.step_unfused(s % self.n_in, k)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    def timed(self, K: int, W: int, k: int, world: int, clocks: bool, graph: bool = True):
        """K decode steps after W warm-up steps.  With graph=True the K steps are
        captured once into a CUDA graph and timed as one replay (the way a serving
        loop issues them); otherwise each step is issued from Python."""
        torch = self.torch
        st = torch.cuda.current_stream()
        self.rewind()
        for s in range(W):
            self.step(s % self.n_in, k)
        torch.cuda.synchronize()
        self.rewind()
        g = None
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for s in range(K):
                    self.step(s % self.n_in, k)
            torch.cuda.synchronize()
            self.rewind()
            g.replay()          # one untimed replay (uploads the graph)
            torch.cuda.synchronize()
            self.rewind()
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
        if sampler:
            time.sleep(0.05)
        barrier(world)
        torch.cuda.synchronize()
        if g is not None:
            # keep the GPU busy while the host submits the replay, so that the
            # interval holds the K steps' device time, not the submission latency
            torch.cuda._sleep(int(1e6))
        e0.record(st)
        if g is not None:
            g.replay()
        else:
            for s in range(K):
                self.step(s % self.n_in, k)
        e1.record(st)
        torch.cuda.synchronize()
        barrier(world)
        clk = sampler.stop() if sampler else None
        total_ms = e0.elapsed_time(e1)
        del g
        return total_ms, [total_ms / K] * K, clk

    def e2e(self, K: int, k: int):
        """Same steps through the public API from pinned host memory: per step one
        H2D copy of the step's packed inputs (q, k_new, v_new) and one D2H copy
        of the step's output are part of the timed region (captured with the
        calls into one CUDA graph).  Both copies run on a second stream with
        double buffers: the input copy of step s + 1 overlaps step s's kernels
        (it waits until step s - 1, the last user of its buffer, is done), and
        the output copy of step s overlaps step s + 1."""
        torch = self.torch
        st = torch.cuda.current_stream()
        cs = torch.cuda.Stream()
        wl = self.wl
        nq, nk = self.q_d[0].numel(), self.k_d[0].numel()
        in_d = [torch.empty_like(self.in_h[0], device="cuda") for _ in range(2)]
        views = [(x[:nq].view(self.q_d[0].shape), x[nq:nq + nk].view(self.k_d[0].shape),
                  x[nq + nk:].view(self.v_d[0].shape)) for x in in_d]
        outs = [self.out, torch.empty_like(self.out)]
        outs_h = [self.out_h, torch.empty_like(self.out_h).pin_memory()]

        def run(n):
            done = [torch.cuda.Event() for _ in range(n)]
            loaded = [torch.cuda.Event() for _ in range(n)]
            copied = [torch.cuda.Event() for _ in range(n)]
            cs.wait_stream(st)

            def load(s):
                with torch.cuda.stream(cs):
                    if s >= 2:
                        cs.wait_event(done[s - 2])            # step s - 2 no longer reads this buffer
                    in_d[s % 2].copy_(self.in_h[s % self.n_in], non_blocking=True)
                    loaded[s].record(cs)

            load(0)
            for s in range(n):
                if s + 1 < n:
                    load(s + 1)
                st.wait_event(loaded[s])
                if s >= 2:
                    st.wait_event(copied[s - 2])              # the output buffer's previous copy is out
                qd, kd, vd = views[s % 2]
                self.aq.aqua_decode_attn(self.cache.desc, qd, self.P, wl["Hq"], k, outs[s % 2], self.ws,
                                         k_new=kd, v_new=vd)
                done[s].record(st)
                with torch.cuda.stream(cs):
                    cs.wait_event(done[s])
                    outs_h[s % 2].copy_(outs[s % 2], non_blocking=True)
                    copied[s].record(cs)
            st.wait_stream(cs)

        self.rewind()
        run(3)
        torch.cuda.synchronize()
        self.rewind()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run(K)
        torch.cuda.synchronize()
        self.rewind()
        g.replay()
        torch.cuda.synchronize()
        self.rewind()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(1e6))                  # the host submits the replay while the GPU sleeps
        e0.record(st)
        g.replay()
        e1.record(st)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        del g
        h2d = self.in_h[0].numel() * self.esize
        d2h = self.out.numel() * self.esize
        return ms, h2d, d2h


class PrefillBench:
    """A prompt pass = for every chunk: aqua_project_keys (append the chunk's keys
    and values), then aqua_prefill_attn (selection + tcgen05 attention).  With
    d_store < d the cache keeps the first d_store projected key dimensions."""

    def __init__(self, wl: dict, P):
        import torch
        import sparse_dimension_attention_b200 as aq
        self.aq, self.torch, self.wl, self.P = aq, torch, wl, P[:wl["Hkv"]].contiguous()
        self.d_store = wl.get("d_store", 128)
        inp = synth.prefill_inputs(wl["L_total"], wl["Hq"], wl["Hkv"], bf16=True, B=wl["B"])
        bf = torch.bfloat16
        self.q = torch.from_numpy(inp["q"]).to(bf).cuda()          # [B, L, Hq, d]
        self.k = torch.from_numpy(inp["k"]).to(bf).cuda()          # [B, L, Hkv, d]
        self.v = torch.from_numpy(inp["v"]).to(bf).cuda()
        self.cache = aq.AquaCache(wl["B"], wl["Hkv"], wl["L_total"] + 128, d_store=self.d_store)
        self.out = torch.empty((wl["B"], wl["chunk"], wl["Hq"], 128), dtype=bf, device="cuda")
        self.ws = torch.empty(aq.aqua_prefill_workspace_size(self.cache.desc, wl["Hq"], wl["chunk"]),
                              dtype=torch.uint8, device="cuda")
        self.n_chunks = wl["L_total"] // wl["chunk"]

    def one_pass(self, k: int, ev=None):
        aq, wl, C = self.aq, self.wl, self.wl["chunk"]
        self.cache.reset()
        for c in range(self.n_chunks):
            s = c * C
            aq.aqua_project_keys(self.cache.desc, self.k[:, s:s + C], self.v[:, s:s + C], self.P, C)
            if ev is not None:
                ev[c][0].record()
            aq.aqua_prefill_attn(self.cache.desc, self.q[:, s:s + C], s, C, self.P, wl["Hq"], k, self.out, self.ws)
            if ev is not None:
                ev[c][1].record()

    def flops(self, pos0: int, k: int):
        """(algorithmic, dense causal, tensor-core issued) flops of one
        aqua_prefill_attn chunk call.  Algorithmic: 2 k flops for the scores on
        the k selected dimensions and 2 d for p.v, per visible (row, token)
        pair and query head.  Dense causal: 4 d per pair and head (standard
        attention).  Issued: the kernel's MMAs, bf16 high + low parts of the
        masked query (contraction d_store) and of P, over every 128-token tile
        each 128-row CTA visits."""
        wl, C, d = self.wl, self.wl["chunk"], 128
        G = wl["Hq"] // wl["Hkv"]
        pairs = C * pos0 + C * (C + 1) // 2
        alg = pairs * wl["Hq"] * (2.0 * k + 2.0 * d)
        dense = pairs * wl["Hq"] * 4.0 * d
        rpb = 128 // G
        tiles = sum(-(-(pos0 + min(C, (qb + 1) * rpb)) // 128) for qb in range(-(-C // rpb)))
        issued = tiles * wl["Hkv"] * wl["B"] * (2 * 2.0 * 128 * 128 * self.d_store + 2 * 2.0 * 128 * 128 * d)
        return alg, dense, issued

    def timed(self, K: int, W: int, k: int):
        """Eager passes with CUDA events around every attention call.  A sleep
        kernel in front of each pass keeps the GPU busy while the host enqueues
        the whole pass, so an interval is the kernel's own duration, not a host
        launch gap (the event between the append and the attention call still
        serialises the two)."""
        torch = self.torch
        for _ in range(W):
            self.one_pass(k)
        torch.cuda.synchronize()
        E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        passes, attn = [], np.zeros(self.n_chunks)
        for _ in range(K):
            ev = [(E(), E()) for _ in range(self.n_chunks)]
            p0, p1 = E(), E()
            torch.cuda._sleep(int(2e6))                   # ~1 ms of GPU time while the host enqueues
            p0.record()
            self.one_pass(k, ev)
            p1.record()
            torch.cuda.synchronize()
            passes.append(p0.elapsed_time(p1))
            attn += np.array([a.elapsed_time(b) for a, b in ev])
        return float(np.mean(passes)), attn / K                       # ms per prompt, ms per chunk call

    def timed_graph(self, K: int, W: int, k: int) -> float:
        """ms per prompt pass with the whole pass (reset, every chunk's append and
        attention call) captured once in a CUDA graph and replayed K times, the
        way a serving loop would issue it: no host launch gaps between calls."""
        torch = self.torch
        for _ in range(W):
            self.one_pass(k)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.one_pass(k)
        torch.cuda.synchronize()
        for _ in range(W):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(2e6))                  # the host submits the replays while the GPU sleeps
        e0.record()
        for _ in range(K):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / K

    def report(self, K: int, W: int, bf16_peak: float, peak_kind: str, dense_ref_ms: float | None = None,
               workload: str = "chunked-prefill-4096") -> dict:
        """The prompt at the workload's k against k = d_store (every stored
        dimension kept: the masked contraction is dense) on the same cache, and
        against dense_ref_ms (the full k = d pass on an untruncated cache) when
        given.  roofline.frac uses the algorithmic flops."""
        wl = self.wl
        k_dense = self.d_store
        eager_ms, attn_ms = self.timed(K, W, wl["k"])
        dense_eager_ms, _ = self.timed(K, W, k_dense)
        prompt_ms = self.timed_graph(K, W, wl["k"])
        dense_ms = self.timed_graph(K, W, k_dense)
        fl = [self.flops(c * wl["chunk"], wl["k"]) for c in range(self.n_chunks)]
        alg_f = sum(f[0] for f in fl)
        dense_f = sum(f[1] for f in fl)
        issued_f = sum(f[2] for f in fl)
        t_attn = float(attn_ms.sum()) / 1e3
        alg = alg_f / t_attn / 1e12
        line = {"workload": workload, **wl, "d": 128, "d_store": self.d_store,
                "prompt_ms": prompt_ms, "tokens_per_s": wl["B"] * wl["L_total"] / (prompt_ms / 1e3),
                "attn_call_us": [round(1e3 * x, 2) for x in attn_ms],
                "roofline": {"bound": "tensor", "achieved": alg, "peak": bf16_peak, "unit": "TFLOP/s",
                             "frac": alg / bf16_peak, "peak_source": peak_kind + " bf16 burst",
                             "achieved_note": "algorithmic flops (2 k on the selected dimensions + 2 d for p.v per "
                                              "visible pair and query head, %.1f GFLOP per prompt) / summed "
                                              "aqua_prefill_attn call time" % (alg_f / 1e9),
                             "dense_causal_tflops": dense_f / t_attn / 1e12,
                             "dense_causal_note": "4 d flops per visible pair and query head (%.1f GFLOP)"
                                                  % (dense_f / 1e9),
                             "issued_tflops": issued_f / t_attn / 1e12,
                             "issued_note": "tcgen05 flops issued (bf16 high+low splits, contraction d_store for "
                                            "the scores, whole 128-token tiles)"},
                "prompt_ms_note": "whole prompt pass captured in one CUDA graph; eager (issued call by call "
                                  "from Python, per-chunk events) in prompt_ms_eager",
                "prompt_ms_eager": eager_ms,
                "k_eq_dstore_prompt_ms": dense_ms,
                "k_eq_dstore_prompt_ms_eager": dense_eager_ms,
                "speedup_vs_k_eq_dstore": dense_ms / prompt_ms,
                "l2": "not flushed: a chunk's K~/V (<= 16 MB) were written by the append just before"}
        if dense_ref_ms is not None:
            line["dense_ref_prompt_ms"] = dense_ref_ms
            line["speedup_vs_dense"] = dense_ref_ms / prompt_ms
            line["speedup_note"] = "dense_ref: k = d = 128 on an untruncated cache (standard attention's work)"
        else:
            line["speedup_vs_dense"] = dense_ms / prompt_ms
        return line


class H2OBench:
    """Steady-state decode on a truncated cache with H2O eviction.  A step is
    aqua_decode_attn (fused append of the step's key/value, scores and lse out)
    followed by aqua_h2o_update (accumulate scores, evict one token): 3 launches."""

    GRAPH_STEPS = 256

    def __init__(self, wl: dict, P):
        import torch
        import sparse_dimension_attention_b200 as aq
        self.aq, self.torch, self.wl = aq, torch, wl
        self.P = P[:wl["Hkv"]].contiguous()
        B, Hq, Hkv, n0 = wl["B"], wl["Hq"], wl["Hkv"], wl["budget"]
        self.n_in = 64
        inp = synth.decode_inputs(B, Hq, Hkv, n0, bf16=True, steps=self.n_in)
        bf = torch.bfloat16
        self.cache = aq.AquaCache(B, Hkv, n0 + 16, d_store=wl["m"], h2o=True)
        for s0 in range(0, n0, 1024):                                       # warm-up fill: positions 0 .. budget-1
            e0 = min(n0, s0 + 1024)
            aq.aqua_project_keys(self.cache.desc, torch.from_numpy(np.ascontiguousarray(inp["k_hist"][:, s0:e0])).to(bf).cuda(),
                                 torch.from_numpy(np.ascontiguousarray(inp["v_hist"][:, s0:e0])).to(bf).cuda(), self.P, e0 - s0)
        self.q = torch.from_numpy(inp["q"]).to(bf).cuda()
        self.kn = torch.from_numpy(inp["k_new"]).to(bf).cuda()
        self.vn = torch.from_numpy(inp["v_new"]).to(bf).cuda()
        Tc = self.cache.Tcap
        self.sc = torch.zeros((B, Hq, Tc), dtype=torch.float32, device="cuda")
        self.lse = torch.zeros((B, Hq), dtype=torch.float32, device="cuda")
        self.out = torch.empty((B, Hq, 128), dtype=bf, device="cuda")
        self.ev = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
        self.ws = torch.zeros(aq.aqua_decode_workspace_size(self.cache.desc, Hq), dtype=torch.uint8, device="cuda")
        self.n_steps = 0
        torch.cuda.synchronize()

    def step(self, sel=None):
        aq, wl, i = self.aq, self.wl, self.n_steps % self.n_in
        aq.aqua_decode_attn(self.cache.desc, self.q[i], self.P, wl["Hq"], wl["k"], self.out, self.ws,
                            k_new=self.kn[i], v_new=self.vn[i], scores_out=self.sc, lse_out=self.lse, sel_out=sel)
        aq.aqua_h2o_update(self.cache.desc, self.sc, self.lse, wl["Hq"], wl["budget"], wl["recent"], self.ev)
        self.n_steps += 1

    def bytes_step(self, usz: float, score_roundtrip: bool = True) -> float:
        """Algorithmic HBM bytes of one step at n = budget+1 attended tokens per (b, g):
        K~ union rows and V rows, the cumulative score/position arrays, the
        append, q and the output; with score_roundtrip also the per-head scores
        the decode step writes and the H2O update reads back (a consequence of
        splitting the step into two kernels, not of the method)."""
        wl = self.wl
        B, Hq, Hkv, n = wl["B"], wl["Hq"], wl["Hkv"], wl["budget"] + 1
        units = B * Hkv
        attn = units * n * (2.0 * usz + 2 * 128)
        scores = 2.0 * B * Hq * n * 4 if score_roundtrip else 0.0
        h2o = units * n * (4 + 4 + 4)                       # score read + write, pos read
        move = units * (wl["m"] + 128) * 2 * 2              # victim slot <- last slot
        append = units * (128 * 2 * 2 + wl["m"] * 2 + 128 * 2)
        qo = B * Hq * 128 * 2 * 2
        return attn + scores + h2o + move + append + qo

    def report(self, W: int, hbm_peak: float, max_reps: int = 0) -> dict:
        """Steady state over the whole absolute-length range, from T_abs =
        budget + (warm-up steps) to T_end: 256-step graphs replayed back to back
        (max_reps > 0 limits the replays, for profiling runs; the line reports
        the range it ran)."""
        torch, wl = self.torch, self.wl
        G = wl["Hq"] // wl["Hkv"]
        for _ in range(W):
            self.step()
        usz = []
        for _ in range(4):
            sel = torch.empty((wl["B"], wl["Hq"], wl["k"]), dtype=torch.int32, device="cuda")
            self.step(sel)
            m = torch.zeros((wl["B"], wl["Hq"], 128), dtype=torch.bool, device="cuda")
            m.scatter_(2, sel.long(), True)
            usz.append(float(m.view(wl["B"], wl["Hkv"], G, 128).any(2).sum(-1).float().mean()))
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(self.GRAPH_STEPS):
                self.step()
        g.replay()                                                           # upload; state advances
        torch.cuda.synchronize()
        t_abs0 = wl["budget"] + self.n_steps                               # tokens seen so far
        reps = max(1, (wl["T_end"] - t_abs0) // self.GRAPH_STEPS)
        if max_reps > 0:
            reps = min(reps, max_reps)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(2e6))                  # the host submits the replays while the GPU sleeps
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        del g
        K = reps * self.GRAPH_STEPS
        n_len = int(self.cache.len[0].item())
        status = self.aq.aqua_status(self.cache.desc)
        by = self.bytes_step(float(np.mean(usz)))
        by_nrt = self.bytes_step(float(np.mean(usz)), score_roundtrip=False)
        gbs = by * K / (ms / 1e3) / 1e9
        gbs_nrt = by_nrt * K / (ms / 1e3) / 1e9
        return {"workload": "truncated-h2o-decode", **wl, "d": 128, "T_end": t_abs0 + K,
                "T_end_config": wl["T_end"],
                "steps": K, "T_abs_range": [t_abs0, t_abs0 + K], "cache_len_after": n_len, "status": status,
                "queries_per_s": wl["B"] * K / (ms / 1e3), "ms_per_step": ms / K,
                "mean_union": float(np.mean(usz)), "bytes_per_step": by, "hbm_gbs": gbs, "frac": gbs / hbm_peak,
                "bytes_per_step_no_score_roundtrip": by_nrt, "hbm_gbs_no_score_roundtrip": gbs_nrt,
                "frac_no_score_roundtrip": gbs_nrt / hbm_peak,
                "launch": "%d-step CUDA graph replayed %d times; 3 launches per step" % (self.GRAPH_STEPS, reps),
                "l2": "no flush: each step streams %.0f MB, above the 126 MB L2" % (by / 1e6)}


def t_sweep(P, K: int, W: int, world: int, Ts=None) -> dict:
    """Decode step time over context lengths T and selection sizes k at the
    Llama decode shape, against k = d at the same T (the same kernels: at k = d
    the selection keeps every dimension, so the comparison isolates what the
    smaller union saves against the fixed per-step costs).  Each point also
    carries the speedup its bytes allow, 2d / (|U| + d) (K~ union rows + V
    against K~ + V), and the pages' flop break-even T* = d^2 (1 + 1/G) / (d - k)
    of AQUA against dense attention per query head."""
    tw = dict(T_SWEEP)
    Ts, ks = Ts or tw.pop("Ts"), tw.pop("ks")
    tw.pop("Ts", None)
    wl = dict(tw, T=max(Ts), k=ks[0])
    tb = DecodeBench(wl, K, W, P=P)
    unions = {kk: tb.union_sizes(kk, min(K, 8)) for kk in ks}
    G, d = wl["Hq"] // wl["Hkv"], 128
    rows = []
    for T in Ts:
        tb.T0 = T - 1
        dense_us = None
        for kk in ks:
            t_ms, d_ms, _ = tb.timed(K, W, kk, world, clocks=False)
            t_ms = max_over_ranks(t_ms, world)
            u = unions[kk]
            by = [tb.bytes_decode(u[s % u.shape[0]], T + s) + tb.bytes_append() for s in range(K)]
            us = 1e3 * t_ms / K
            dense_us = us if kk == d else dense_us
            rows.append({"T": T, "k": kk, "decode_us": us, "mean_union": float(u.mean()),
                         "decode_gbs": sum(by) / (t_ms / 1e3) / 1e9,
                         "speedup_vs_k_d": (dense_us / us) if dense_us else None,
                         "byte_bound_speedup": 2.0 * d / (float(u.mean()) + d),
                         "l2_resident": by[0] < L2_BYTES})
    del tb
    return {"workload": "llama3.1-8b-decode T x k sweep", "B": wl["B"], "Hq": wl["Hq"], "Hkv": wl["Hkv"],
            "steps_per_point": K, "rows": rows, "launch": "K steps in one CUDA graph per (T, k)",
            "flop_breakeven_T": {str(kk): d * d * (1 + 1 / G) / (d - kk) for kk in ks if kk < d},
            "note": "l2_resident: a step's algorithmic bytes fit in the 126 MB L2 (no flush between steps)"}


def cpu_baseline(wl: dict, budget_s: float = 12.0) -> dict:
    """The oracle, as it stands, on the host cores: decode steps of one sequence
    (all its query heads) repeated until about budget_s seconds have run."""
    from oracle import aqua_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    B, Hq, Hkv, T, k = 1, wl["Hq"], wl["Hkv"], wl["T"], wl["k"]
    P, _ = O.calibrate(synth.calibration_matrix())
    P = np.broadcast_to(P, (Hkv, 128, 128))
    inp = synth.decode_inputs(B, Hq, Hkv, T - 1, bf16=(wl["kv"] == "bf16"), steps=1)
    k_all = np.concatenate([inp["k_hist"], inp["k_new"].transpose(1, 0, 2, 3)], axis=1)
    v_all = np.concatenate([inp["v_hist"], inp["v_new"].transpose(1, 0, 2, 3)], axis=1)
    Kt = O.build_key_cache(k_all, P, wl["kv"]).transpose(0, 2, 1, 3)
    V = v_all.transpose(0, 2, 1, 3).astype(np.float64)
    n, t0 = 0, time.perf_counter()
    while True:
        O.build_key_cache(inp["k_new"][0][:, None], P, wl["kv"])          # the step's key projection
        O.decode(inp["q"][0], P, Kt, V, [T], k, out_dtype=wl["kv"])
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 200:
            break
    return {"value": n / el, "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "sample": f"{n} decode steps of 1 sequence ({Hq} query heads, T={T}, k={k}) in {el:.1f} s; "
                      f"the job's unit is one sequence-step"}


def run_reference(args, world, rank):
    """--impl reference: the oracle timed on the host cores on this workload."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    from oracle import aqua_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    B, Hq, Hkv, T, k = 1, wl["Hq"], wl["Hkv"], wl["T"], wl["k"]
    P, _ = O.calibrate(synth.calibration_matrix())
    P = np.broadcast_to(P, (Hkv, 128, 128))
    inp = synth.decode_inputs(B, Hq, Hkv, T - 1, bf16=(wl["kv"] == "bf16"), steps=max(args.steps, args.warmup) + 1)
    k_all = np.concatenate([inp["k_hist"], inp["k_new"][0][:, None]], axis=1)
    v_all = np.concatenate([inp["v_hist"], inp["v_new"][0][:, None]], axis=1)
    Kt = O.build_key_cache(k_all, P, wl["kv"]).transpose(0, 2, 1, 3)
    V = v_all.transpose(0, 2, 1, 3).astype(np.float64)

    def one(s):
        O.build_key_cache(inp["k_new"][s][:, None], P, wl["kv"])          # the step's key projection
        O.decode(inp["q"][s], P, Kt, V, [T], k, out_dtype=wl["kv"])

    for s in range(args.warmup):
        one(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        one(s)
    el = time.perf_counter() - t0
    val = args.steps / el
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, **wl, "reference_sample": "1 of the B sequences per step"},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": int(threads), "kind": "oracle",
                             "sample": f"each step: one sequence (all {Hq} query heads) of {args.workload}"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="aqua", choices=["aqua", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--no-extras", action="store_true", help="only the main decode line")
    ap.add_argument("--extras", default="sweep,memory,tsweep,long,prefill,h2o",
                    help="comma list of extra lines: sweep (k sweep), memory (keys and values stored at 96 "
                         "projected dims), tsweep (break-even sweep over T in "
                         "{2048, 8192, 32768} and k), tsweep_full (T from 512 to 32768), long (long context), "
                         "prefill (chunked prefill, full and truncated cache), h2o (truncated cache + H2O steady "
                         "state)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--h2o-reps", type=int, default=0,
                    help="limit the H2O line's 256-step graph replays (profiling runs; default: the whole range)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    import torch
    torch.cuda.set_device(local)
    wl = dict(WORKLOADS[args.workload])
    if args.k is not None:
        wl["k"] = args.k
    K, W = args.steps, args.warmup
    hbm_peak, bf16_peak, peak_kind = peaks()

    bench = DecodeBench(wl, K, W)
    usz = bench.union_sizes(wl["k"], min(K, bench.n_in))                       # [K, B, Hkv]
    total_ms, step_ms, clk = bench.timed(K, W, wl["k"], world, clocks=(rank == 0))
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / K
    value = whole_job_rate(wl["B"], K, world, total_ms)
    T_steps = [wl["T"] + s for s in range(K)]
    dec_bytes = [bench.bytes_decode(usz[s % usz.shape[0]], T_steps[s]) for s in range(K)]
    step_gbs = (sum(dec_bytes) + K * bench.bytes_append()) / (total_ms / 1e3) / 1e9
    # the dominant kernel alone: the attention kernel's algorithmic bytes over its own duration
    Kk = min(K, 50)
    sel_ms, att_ms = bench.kernel_times(Kk, wl["k"])
    att_bytes = float(np.mean([bench.bytes_attend(usz[s % usz.shape[0]], T_steps[s]) for s in range(Kk)]))
    att_gbs = att_bytes / (att_ms / 1e3) / 1e9
    unfused_ms = bench.timed_unfused(min(K, 100), W, wl["k"])
    eager_ms, _, _ = bench.timed(min(K, 100), W, wl["k"], world, clocks=False, graph=False)
    e2e_ms, h2d, d2h = bench.e2e(K, wl["k"])
    e2e_ms = max_over_ranks(e2e_ms, world)
    kname = "decode_attn_bf16_kernel" if wl["kv"] == "bf16" else "decode_attn_f32_kernel"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl["kv"] == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": args.workload, "B": wl["B"], "Hq": wl["Hq"], "Hkv": wl["Hkv"], "d": 128,
                   "T": wl["T"], "T_range": [T_steps[0], T_steps[-1]], "k": wl["k"], "kv_cache": wl["kv"],
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": "cuda graph",
                   "l2": "no flush: each step streams %.0f MB of K~/V, above the 126 MB L2"
                         % (dec_bytes[0] / 1e6),
                   "inputs": "synthetic anisotropic Q/K (Llama-3.1-8B shape), P from GPU SVD calibration"},
        "hbm_gbs": step_gbs,
        "mean_union": float(usz.mean()),
        "roofline": {"bound": "hbm", "achieved": att_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": att_gbs / hbm_peak,
                     "traffic": profile_traffic(kname, "sparse_dimension_attention_b200/csrc/decode.cu"),
                     "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the "
                                     "kernel (profiles/ncu_traffic.json); null when its source changed since",
                     "kernel": kname, "kernel_us": 1e3 * att_ms, "bytes_per_launch": att_bytes,
                     "achieved_note": "algorithmic bytes of the attention kernel (K~ union rows + V rows per "
                                      "(b, KV head) and token, output write) / its mean duration alone (CUDA "
                                      "events around aqua_decode_attend, %d steps)" % Kk,
                     "peak_source": peak_kind,
                     "select_kernel_us": 1e3 * sel_ms,
                     "step_us": 1e3 * ms_step, "step_gbs": step_gbs, "step_frac": step_gbs / hbm_peak,
                     "step_note": "whole step (both kernels, programmatically overlapped, in one CUDA graph): "
                                  "all algorithmic bytes incl. the append / step time"},
        "launch": "K steps captured in one CUDA graph (kernels chained with programmatic dependent launch)",
        "eager_step_us": 1e3 * eager_ms / min(K, 100),
        "unfused_step_us": 1e3 * unfused_ms,
        "e2e": {"value": whole_job_rate(wl["B"], K, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "aqua_decode_attn from pinned host buffers; per step one packed input copy and one output "
                        "copy, both double-buffered on a second stream (input of step s+1 and output of step s "
                        "overlap the step's kernels)"},
        "gpu_launches": 2 * K,
        "clocks": clk,
    }
    extras = set() if args.no_extras else {x.strip() for x in args.extras.split(",") if x.strip()}
    if "sweep" in extras:
        sweep = []
        for kk in (128, 96, 64, 32):
            u = bench.union_sizes(kk, min(K, 8))
            t_ms, d_ms, _ = bench.timed(K, W, kk, world, clocks=False)
            t_ms = max_over_ranks(t_ms, world)
            by = [bench.bytes_decode(u[s % u.shape[0]], T_steps[s]) + bench.bytes_append() for s in range(K)]
            sweep.append({"k": kk, "queries_per_s": world * wl["B"] * K / (t_ms / 1e3), "ms_per_step": t_ms / K,
                          "decode_us": 1e3 * statistics.mean(d_ms), "mean_union": float(u.mean()),
                          "decode_gbs": sum(by) / (sum(d_ms) / 1e3) / 1e9,
                          "byte_bound_speedup": 256.0 / (float(u.mean()) + 128.0)})
        dense = sweep[0]["decode_us"]
        for r in sweep:
            r["speedup_vs_dense"] = dense / r["decode_us"]
        line["k_sweep"] = sweep
    P = bench.P
    del bench
    torch.cuda.empty_cache()
    if "memory" in extras:
        mwl = WORKLOADS["aqua-memory-decode"]
        mb = DecodeBench(mwl, K, W, P=P)
        mu = mb.union_sizes(mwl["k"], min(K, 8))
        t_ms, d_ms, _ = mb.timed(K, W, mwl["k"], world, clocks=False)
        t_ms = max_over_ranks(t_ms, world)
        by = [mb.bytes_decode(mu[s % mu.shape[0]], T_steps[s]) + mb.bytes_append() for s in range(K)]
        gbs = sum(by) / (t_ms / 1e3) / 1e9
        dense_us = line["k_sweep"][0]["decode_us"] if "k_sweep" in line else None
        us = 1e3 * t_ms / K
        line["aqua_memory"] = {"workload": "aqua-memory-decode", **mwl, "d": 128, "ms_per_step": t_ms / K,
                               "queries_per_s": world * mwl["B"] * K / (t_ms / 1e3), "decode_us": us,
                               "mean_union": float(mu.mean()), "bytes_per_step": float(np.mean(by)),
                               "decode_gbs": gbs, "frac": gbs / hbm_peak,
                               "speedup_vs_dense": dense_us / us if dense_us else None,
                               "byte_bound_speedup": 256.0 / (float(mu.mean()) + mwl["dv_store"]),
                               "note": "keys and values both stored at their first 96 projected dims; dense = the "
                                       "k = d = 128 step on the full cache (k_sweep[0]); 3 launches per step (the "
                                       "third brings the output back from the projected value dims)"}
        del mb
        torch.cuda.empty_cache()
    if "tsweep" in extras or "tsweep_full" in extras:
        line["t_sweep"] = t_sweep(P, min(K, 20), W, world, Ts=T_SWEEP_FULL_TS if "tsweep_full" in extras else None)
        torch.cuda.empty_cache()
    if "long" in extras:
        lwl = WORKLOADS["long-context-decode"]
        lb = DecodeBench(lwl, min(K, 50), W)
        lu = lb.union_sizes(lwl["k"], min(K, 50, lb.n_in))
        Kl = min(K, 50)
        t_ms, d_ms, _ = lb.timed(Kl, W, lwl["k"], world, clocks=False)
        t_ms = max_over_ranks(t_ms, world)
        by = [lb.bytes_decode(lu[s % lu.shape[0]], lwl["T"] + s) + lb.bytes_append() for s in range(Kl)]
        ach = sum(by) / (sum(d_ms) / 1e3) / 1e9
        line["long_context"] = {"workload": "long-context-decode", "B": 1, "T": lwl["T"], "k": lwl["k"],
                                "queries_per_s": world * Kl / (t_ms / 1e3), "ms_per_step": t_ms / Kl,
                                "decode_us": 1e3 * statistics.mean(d_ms), "decode_gbs": ach,
                                "frac": ach / hbm_peak}
        del lb
        torch.cuda.empty_cache()
    if "prefill" in extras:
        pb = PrefillBench(PREFILL, P)
        line["prefill"] = pb.report(min(K, 20), W, bf16_peak, peak_kind)
        del pb
        torch.cuda.empty_cache()
        pb = PrefillBench(PREFILL_TRUNC, P)
        line["prefill_truncated"] = pb.report(min(K, 20), W, bf16_peak, peak_kind,
                                              dense_ref_ms=line["prefill"]["k_eq_dstore_prompt_ms"],
                                              workload="chunked-prefill-4096-truncated-cache")
        del pb
        torch.cuda.empty_cache()
    if "h2o" in extras:
        hb = H2OBench(H2O_WL, P)
        line["truncated_h2o"] = hb.report(W, hbm_peak, args.h2o_reps)
        del hb
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
