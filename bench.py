"""Benchmark of the IndexMem hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2] [--budget 1024]
    python bench.py --impl reference ...     # the CPU oracle on a bounded sample

A step is one pass of the whole path over one batch of the workload:
indexer scoring with the streaming per-key max (chunked for long contexts),
top-B selection and compaction, the latent-memory update from the evicted
tokens, then the decode steps over the retained cache with the memory readout.
The metric counts tokens through the path: the b*L context keys scored and
evicted plus the b*n_decode decoded tokens, per second.

Under torchrun every rank runs its own replica on its own GPU (the batch
units are independent; no collective on the data path): weak scaling, the
time is the max over ranks and the value counts the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from learned_kv_cache_indexmem_b200 import binding, synth  # noqa: E402
from learned_kv_cache_indexmem_b200.layer import IndexMemLayer  # noqa: E402

METRIC = "evicted-cache decode tokens/s + indexer keys/s; % of HBM / tensor-core roofline"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples the GPU's SM clock and clock-event reasons through NVML every
    10 ms while the timed region runs (thread); nvidia-smi as a fallback."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: torch.device):
        self.device = device
        self.samples, self.maxes, self.reasons = [], [], set()
        self._stop = threading.Event()
        self._t = None
        self.h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(device)
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    self.h = None
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
        except Exception:
            self.h = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.maxes.append(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.01)

    def start(self):
        if self.h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        self._stop.set()
        self._t.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": max(self.maxes) if self.maxes else None,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def reduce_over_ranks(value: float, device, op: str = "max") -> float:
    """Max (or sum) of a float over the ranks of the default process group;
    the value itself without one."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX if op == "max"
                                 else torch.distributed.ReduceOp.SUM)
    return float(t.item())


def decode_traffic_from_profile(workload: str):
    """dram bytes per decode launch from the committed ncu summary, if it was
    taken on the current decode kernel source (else None)."""
    import hashlib
    src = os.path.join(ROOT, "learned_kv_cache_indexmem_b200", "csrc", "decode.cu")
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and parts[0] == "decode_kernel" and parts[1] == workload:
            kv = dict(p.split("=", 1) for p in parts[2:] if "=" in p)
            if kv.get("src_sha1") == sha:
                return float(kv["bytes_per_launch"])
    return None


# ------------------------------------------------------------------ workload

class Job:
    """One replica of the workload on one GPU, inputs resident in HBM."""

    def __init__(self, wl, B, device, seed):
        self.wl, self.B, self.dev = wl, B, device
        s = wl.shape
        self.batch, self.L, self.n_dec = wl.batch, wl.L, wl.n_decode
        self.cap = B + self.n_dec
        w = synth.make_weights(s, seed, device)
        self.inp = synth.make_layer_inputs(wl, w, seed, device)
        self.decin = synth.make_decode_inputs(wl, w, self.n_dec, seed, device)
        if wl.needles:
            synth.plant_needles(wl, self.inp["K"], self.decin["q"], wl.needles, seed)
        self.w = w
        self.layer = IndexMemLayer.from_shape(s, w)
        self.st = self.layer.new_state(self.batch, self.L, B, self.cap, device)
        self.layer.workspace(self.batch, self.L, B, device)
        self.zero_M = torch.zeros_like(self.st.M)
        self.zero_b = torch.zeros_like(self.st.bstab)
        self.len0 = torch.full_like(self.st.cache_len, B)
        self.out = torch.empty(self.n_dec, self.batch, s.n_q_heads, s.head_dim, dtype=s.torch_dtype,
                               device=device)
        ch = wl.prefill_chunk
        self.ranges = ([(i, min(self.L, i + ch)) for i in range(0, self.L, ch)] if ch else
                       [(0, self.L)])
        self.stream = torch.cuda.Stream(device)   # capture needs a non-default stream
        self.graph = None

    # kernels per call (see the library's launchers)
    def launches_per_step(self):
        n_e = self.L - self.B
        return 2 * len(self.ranges) + 2 + (2 if n_e > 0 else 0) + self.n_dec

    def reset(self):
        # kernels, not device-to-device memcpys: those share the copy engines
        # with the next step's inputs in flight (the end-to-end loop)
        self.st.cache_len.fill_(self.B)
        self.st.M.zero_()
        self.st.bstab.zero_()

    def prefill(self):
        d = self.inp
        self.layer.score_and_evict(d["X"], d["Q"], d["K"], d["V"], self.st, self.B,
                                   q_ranges=self.ranges, stream=self.stream)

    def memory(self):
        self.layer.update_memory(self.inp["K"], self.inp["V"], self.st, self.B,
                                 chunk=self.wl.mem_chunk, stream=self.stream)

    def decode_loop(self):
        for s in range(self.n_dec):
            self.layer.decode(self.decin["q"][s], self.decin["k_new"][s], self.decin["v_new"][s],
                              self.st, out=self.out[s], stream=self.stream)

    def capture_decode(self):
        """The decode steps as one CUDA graph (removes per-launch host overhead)."""
        with torch.cuda.stream(self.stream):
            self.reset()
            self.prefill()
            self.memory()
            self.decode_loop()          # warm (and exercise) outside capture
        torch.cuda.synchronize()
        self.layer.sync(self.stream)
        with torch.cuda.stream(self.stream):
            self.reset()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self.decode_loop()
        torch.cuda.synchronize()
        self.graph = g

    def step(self, ev=None):
        with torch.cuda.stream(self.stream):
            self._step(ev)

    def _step(self, ev):
        self.reset()
        if ev: ev[0].record(self.stream)
        self.prefill()
        if ev: ev[1].record(self.stream)
        self.memory()
        if ev: ev[2].record(self.stream)
        if self.graph is not None:
            self.graph.replay()
        else:
            self.decode_loop()
        if ev: ev[3].record(self.stream)

    # algorithmic work -------------------------------------------------------
    def decode_bytes_per_launch(self):
        """K/V rows read (cache incl. the new row), memory state, q in, out,
        new row written; averaged over the decode steps of a step."""
        s = self.wl.shape
        es = 2 if s.dtype == "bf16" else 4
        row = s.n_kv_heads * s.head_dim * es * 2
        avg_rows = self.B + (self.n_dec + 1) / 2.0
        mstate = s.n_kv_heads * (s.mem_r * s.head_dim + s.mem_r) * 4
        qo = 2 * s.n_q_heads * s.head_dim * es
        return self.batch * (avg_rows * row + mstate + qo + row / 2)

    def prefill_bytes(self):
        s = self.wl.shape
        es = 2 if s.dtype == "bf16" else 4
        xq = self.batch * self.L * (s.hidden + s.n_q_heads * s.head_dim) * es
        kv_ret = 2 * self.batch * self.B * s.n_kv_heads * s.head_dim * es * 2
        return xq + kv_ret

    def memory_bytes(self):
        s = self.wl.shape
        es = 2 if s.dtype == "bf16" else 4
        return self.batch * (self.L - self.B) * s.n_kv_heads * s.head_dim * es * 2

    def scoring_flops(self):
        pairs = 0
        for (q0, q1) in self.ranges:
            # pairs (s, t) with t <= s, s in [q0, q1)
            pairs += (q1 * (q1 + 1) - q0 * (q0 + 1)) // 2
        return 2 * self.wl.shape.idx_dim * pairs * self.batch

    def tokens_per_step(self):
        return self.batch * (self.L + self.n_dec)


# ------------------------------------------------------------------ full-cache decode

def full_cache_decode(job, steps=64, reps=3):
    """The same decode kernel over the full context (budget B = L: nothing
    evicted, memory state empty) next to the evicted cache, per decode step:
    the pages' claim that decoding with eviction and memory stays competitive
    with the full cache ("IndexMem" technical summary §4, Efficiency)."""
    s = job.wl.shape
    b, L = job.batch, job.L
    cap = L + steps
    full = job.layer.new_state(b, L, L, cap, job.dev)
    full.K_ret[:, :L] = job.inp["K"]
    full.V_ret[:, :L] = job.inp["V"]
    full.cache_len.fill_(L)
    len0 = full.cache_len.clone()
    evicted = job.layer.new_state(b, L, job.B, job.B + steps, job.dev)
    evicted.K_ret[:, :job.B] = job.st.K_ret[:, :job.B]
    evicted.V_ret[:, :job.B] = job.st.V_ret[:, :job.B]
    evicted.M.copy_(job.st.M)
    evicted.bstab.copy_(job.st.bstab)
    evicted.cache_len.fill_(job.B)
    elen0 = evicted.cache_len.clone()
    out = torch.empty_like(job.decin["q"][0])
    res = {}
    for name, st, l0 in (("full", full, len0), ("evicted", evicted, elen0)):
        with torch.cuda.stream(job.stream):
            st.cache_len.copy_(l0)
            job.layer.invalidate_decode(b, stream=job.stream)   # the state was written directly
            job.layer.decode(job.decin["q"][0], job.decin["k_new"][0], job.decin["v_new"][0], st,
                             out=out, stream=job.stream)
            torch.cuda.synchronize()
            st.cache_len.copy_(l0)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=job.stream):
                for i in range(steps):
                    job.layer.decode(job.decin["q"][i], job.decin["k_new"][i], job.decin["v_new"][i],
                                     st, out=out, stream=job.stream)
            best = None
            for _ in range(reps):
                st.cache_len.copy_(l0)
                job.layer.invalidate_decode(b, stream=job.stream)
                torch.cuda.synchronize()
                a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(job.stream)
                g.replay()
                e.record(job.stream)
                torch.cuda.synchronize()
                t = a.elapsed_time(e) / steps * 1e3
                best = t if best is None else min(best, t)
            del g
        res[name] = best
    job.layer.sync(job.stream)
    row = s.n_kv_heads * s.head_dim * (2 if s.dtype == "bf16" else 4) * 2
    return {"steps": steps, "us_per_step_full_cache": res["full"],
            "us_per_step_evicted": res["evicted"], "speedup": res["full"] / res["evicted"],
            "full_cache_GBps": b * (L + steps / 2) * row / (res["full"] * 1e-6) / 1e9}


# ------------------------------------------------------------------ moment readout

def moment_readout(job, steps=64, reps=3):
    """The MomentKV readout ("MomentKV" technical summary, Method §1, §2, §4) on
    the same workload, next to IndexMem's gated memory readout: the statistics
    update from the evicted tokens and the decode step, each timed with CUDA
    events (the decode steps as one CUDA graph)."""
    s = job.wl.shape
    b, L, Bud = job.batch, job.L, job.B
    lay = IndexMemLayer.from_shape(s, job.w, readout="moment")
    st = lay.new_state(b, L, Bud, Bud + steps, job.dev)
    lay.workspace(b, L, Bud, job.dev)
    res = {}

    def timed(fn, n=reps):
        best = None
        for _ in range(n):
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(job.stream)
            fn()
            e.record(job.stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(e)
            best = t if best is None else min(best, t)
        return best

    with torch.cuda.stream(job.stream):
        d = job.inp
        lay.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st, Bud, q_ranges=job.ranges,
                            stream=job.stream)

        def upd_m():
            st.M.zero_(); st.bstab.zero_(); st.s_v.zero_(); st.n_e.zero_()
            lay.update_memory(d["K"], d["V"], st, Bud, chunk=job.wl.mem_chunk, stream=job.stream)

        def upd_g():
            job.st.M.zero_(); job.st.bstab.zero_()
            job.memory()

        res["update_ms_moment"] = timed(upd_m)
        res["update_ms_gated"] = timed(upd_g)
        len0 = torch.full_like(st.cache_len, Bud)
        out = torch.empty_like(job.decin["q"][0])
        graphs = {}
        for name, layer, state in (("moment", lay, st), ("gated", job.layer, job.st)):
            state.cache_len.copy_(len0)
            layer.invalidate_decode(state.cache_len.shape[0], stream=job.stream)
            layer.decode(job.decin["q"][0], job.decin["k_new"][0], job.decin["v_new"][0], state,
                         out=out, stream=job.stream)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            state.cache_len.copy_(len0)
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=job.stream):
                for i in range(steps):
                    layer.decode(job.decin["q"][i], job.decin["k_new"][i], job.decin["v_new"][i],
                                 state, out=out, stream=job.stream)

            def rep(g=g, state=state, layer=layer):
                state.cache_len.copy_(len0)
                layer.invalidate_decode(state.cache_len.shape[0], stream=job.stream)
                g.replay()
            res["decode_us_per_step_" + name] = timed(rep) / steps * 1e3
            graphs[name] = g
        del graphs
    lay.sync(job.stream)
    job.layer.sync(job.stream)
    lay.close()
    res["steps"] = steps
    return res


# ------------------------------------------------------------------ stage split, budgets

def prefill_split(job, peaks, reps=5, inner=10):
    """The prefill by kernel, each through its own C-ABI call and timed alone
    with CUDA events on the launching stream: `inner` back-to-back calls
    between two events (each call is idempotent: the prologue rewrites the
    same features, the scoring's running maxima are already the maxima, the
    selection rewrites the same outputs), the average per call, best of
    `reps`; this takes the host's launch latency out of the figure: the indexer
    prologue (imem_indexer_features: read X and Q, write q~ and k^), the
    scoring with the streaming per-key max (imem_indexer_score: 128 flop per
    causal pair) and the selection + compaction (imem_select_compact). Each
    gets its roofline: the prologue against HBM, the scoring against the
    burst bf16 tensor peak (a kernel timed alone), the selection + compaction
    against HBM."""
    d = job.inp
    st = job.st
    ws = job.layer._ws
    ctx = job.layer.ctx
    b, L, B = job.batch, job.L, job.B

    def timed(fn, n=inner):
        fn()
        torch.cuda.synchronize()
        best = None
        for _ in range(reps):
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(job.stream)
            for _ in range(n):
                fn()
            e.record(job.stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(e) / n
            best = t if best is None else min(best, t)
        return best

    def features():
        for q0, q1 in job.ranges:
            binding.indexer_features(ctx, b, L, d["X"], d["Q"], st.running_max, q0, q1, ws,
                                     job.stream)

    def score():
        # the prologue's features are in the workspace; the scoring re-runs
        # over them (running_max only rises, so repeats give the same result)
        for q0, q1 in job.ranges:
            binding.indexer_score(ctx, b, L, st.running_max, q0, q1, ws, job.stream)

    def select():
        binding.select_compact(ctx, b, L, B, st.running_max, d["K"], d["V"], st.idx_retained,
                               st.idx_evicted, st.K_ret, st.V_ret, st.K_ret.shape[1], ws,
                               job.stream)

    def whole():
        for i, (q0, q1) in enumerate(job.ranges):
            last = i == len(job.ranges) - 1
            binding.score_and_evict(ctx, b, L, B, d["X"], d["Q"], d["K"], d["V"],
                                    st.running_max, q0, q1, 1 if last else 0, st.idx_retained,
                                    st.idx_evicted, st.K_ret, st.V_ret, st.K_ret.shape[1], ws,
                                    job.stream)

    features()                       # features in place for the score-only timing
    t_pro = timed(features)
    t_sco = timed(score)
    t_sel = timed(select)
    t_all = timed(whole)
    s = job.wl.shape
    es = 2 if s.dtype == "bf16" else 4
    row = s.n_kv_heads * s.head_dim * es * 2
    pro_bytes = job.prefill_bytes() - 2 * b * B * row + b * L * 2 * 64 * 2   # X, Q in; q~, k^ out
    sel_bytes = b * (4 * L + 4 * L + 2 * B * row)      # scores in, indices out, K/V rows in+out
    flops = job.scoring_flops()
    pro_gbs = pro_bytes / (t_pro * 1e-3) / 1e9
    sco_tf = flops / (t_sco * 1e-3) / 1e12
    sel_gbs = sel_bytes / (t_sel * 1e-3) / 1e9
    return {
        "prologue": {"ms": t_pro, "keys_per_s": b * L / (t_pro * 1e-3), "bytes": pro_bytes,
                     "GBps": pro_gbs, "roofline": {"bound": "hbm", "peak": peaks["hbm_gbs"],
                                                   "unit": "GB/s",
                                                   "frac": pro_gbs / peaks["hbm_gbs"]}},
        "scoring": {"ms": t_sco, "keys_per_s": b * L / (t_sco * 1e-3), "flop": flops,
                    "TFLOPs": sco_tf, "roofline": {"bound": "tensor", "peak": peaks["bf16_tflops"],
                                                   "unit": "TFLOP/s",
                                                   "frac": sco_tf / peaks["bf16_tflops"],
                                                   "peak_kind": "burst (kernel timed alone)"}},
        "select_compact": {"ms": t_sel, "bytes": sel_bytes, "GBps": sel_gbs,
                           "roofline": {"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                        "frac": sel_gbs / peaks["hbm_gbs"]}},
        "indexer_ms": t_pro + t_sco,
        "indexer_keys_per_s": b * L / ((t_pro + t_sco) * 1e-3),
        "score_and_evict_ms": t_all,
        "note": "each kernel alone: CUDA events on its stream around %d back-to-back calls, "
                "average per call, best of %d; score_and_evict_ms is the one-call prefill "
                "timed the same way" % (inner, reps)}


def other_workload_step(name, dev, seed, steps=5, warmup=3):
    """The whole step (prefill, memory update, decode steps in a CUDA graph) on
    another single-layer workload, timed like the main line: ms per step,
    tokens/s, decode tokens/s and decode per launch."""
    wl = synth.WORKLOADS[name]
    j = Job(wl, wl.budget, dev, seed)
    j.capture_decode()
    for _ in range(warmup):
        j.step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(j.stream)
    for i in range(steps):
        j.step(ev[i])
    e.record(j.stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(e) / steps
    dec = statistics.mean(x[2].elapsed_time(x[3]) for x in ev)
    pre = statistics.mean(x[0].elapsed_time(x[1]) for x in ev)
    mem = statistics.mean(x[1].elapsed_time(x[2]) for x in ev)
    dec_launch_ms = dec / j.n_dec
    dec_bytes = j.decode_bytes_per_launch()
    j.layer.sync(j.stream)
    out = {"workload": "%s: batch %d, L=%d, B=%d, %d decode steps" % (
               name, wl.batch, wl.L, wl.budget, wl.n_decode),
           "ms_per_step": ms, "tokens_per_s": j.tokens_per_step() / (ms * 1e-3),
           "prefill_ms": pre, "indexer_keys_per_s": j.batch * j.L / (pre * 1e-3),
           "memory_ms": mem, "decode_ms": dec,
           "decode_tokens_per_s": j.batch * j.n_dec / (dec * 1e-3),
           "decode_us_per_launch": dec_launch_ms * 1e3,
           "decode_bytes_per_launch": dec_bytes,
           "decode_GBps": dec_bytes / (dec_launch_ms * 1e-3) / 1e9}
    del j
    torch.cuda.empty_cache()
    return out


def budget_sweep(wl, dev, seed, budgets=(128, 256, 512), steps=5, warmup=3):
    """The whole step at the other budgets of the workload (the benchmark's own
    budget is the main line): time per step, tokens/s and decode per launch."""
    out = {}
    for B in budgets:
        j = Job(wl, B, dev, seed)
        j.capture_decode()
        for _ in range(warmup):
            j.step()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(j.stream)
        for i in range(steps):
            j.step(ev[i])
        e.record(j.stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(e) / steps
        dec = statistics.mean(x[2].elapsed_time(x[3]) for x in ev)
        out[str(B)] = {"ms_per_step": ms, "tokens_per_s": j.tokens_per_step() / (ms * 1e-3),
                       "decode_us_per_launch": dec / j.n_dec * 1e3}
        j.layer.sync(j.stream)
        del j
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ online eviction

def online_decode(job, steps=64, reps=3):
    """Decode steps that keep the cache at the budget (each step's least
    important token leaves into the memory: "IndexMem" technical summary
    §2.B, memory updated online) next to the plain decode over the same
    evicted cache; per step, CUDA graphs of `steps` steps."""
    b, B, L = job.batch, job.B, job.L
    lay = job.layer
    st = lay.new_state(b, L, B, job.cap, job.dev)
    for k in ("running_max", "idx_retained", "K_ret", "V_ret", "M", "bstab"):
        getattr(st, k).copy_(getattr(job.st, k))
    st.cache_len.fill_(B)
    out = torch.empty_like(job.decin["q"][0])
    res = {}
    with torch.cuda.stream(job.stream):
        on = lay.online_init(st, B, L, stream=job.stream)
        lay.invalidate_decode(b, stream=job.stream)   # the state was copied in directly
        dec = job.decin

        def step(i):
            lay.decode_online(dec["x"][i], dec["q"][i], dec["k_new"][i], dec["v_new"][i], st, on,
                              B, out=out, stream=job.stream)
        step(0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=job.stream):
            for i in range(steps):
                step(i)
        best = None
        for _ in range(reps):
            torch.cuda.synchronize()
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(job.stream)
            g.replay()
            e.record(job.stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(e) / steps * 1e3
            best = t if best is None else min(best, t)
        del g
    lay.sync(job.stream)
    res["us_per_step_online"] = best
    res["launches_per_step_online"] = 3   # features (second stream); attention, score and evict
    res["steps"] = steps
    res["cache_rows"] = B
    return res


# ------------------------------------------------------------------ pre-eviction

def pre_eviction(dev, reps=3):
    """Chunked prefill that evicts after every query range (the cache never
    holds more than B tokens; "IndexMem" technical summary §2.A, eviction
    before the full prefill) next to the chunked prefill that selects once at
    the end, on the long-context workload (c3: one sequence, L = 131072,
    ranges of 8192, B = 13107, memory update included in both). CUDA events
    around each whole prefill."""
    wl = synth.WORKLOADS["c3"]
    s = wl.shape
    b, L, B, ch = wl.batch, wl.L, wl.budget, wl.prefill_chunk
    w = synth.make_weights(s, wl.seed, dev)
    inp = synth.make_layer_inputs(wl, w, wl.seed, dev)
    ranges = [(q, min(L, q + ch)) for q in range(0, L, ch)]
    stream = torch.cuda.Stream(dev)
    lay_e, lay_o = IndexMemLayer.from_shape(s, w), IndexMemLayer.from_shape(s, w)
    st_e = lay_e.new_state(b, L, B, B, dev)
    st_o = lay_o.new_state(b, L, B, B, dev)
    d = inp

    def evict():
        st_e.M.zero_(); st_e.bstab.zero_()
        lay_e.prefill_evict(d["X"], d["Q"], d["K"], d["V"], st_e, B, ch, mem_chunk=wl.mem_chunk,
                            stream=stream)

    def at_end():
        st_o.M.zero_(); st_o.bstab.zero_()
        lay_o.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st_o, B, q_ranges=ranges,
                              stream=stream)
        lay_o.update_memory(d["K"], d["V"], st_o, B, chunk=wl.mem_chunk, stream=stream)

    res = {}
    with torch.cuda.stream(stream):
        for name, fn in (("pre_evict", evict), ("select_at_end", at_end)):
            fn()
            torch.cuda.synchronize()
            best = None
            for _ in range(reps):
                a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                e.record(stream)
                torch.cuda.synchronize()
                t = a.elapsed_time(e)
                best = t if best is None else min(best, t)
            res["ms_" + name] = best
            res["keys_per_s_" + name] = b * L / (best * 1e-3)
    lay_e.sync(stream)
    lay_o.sync(stream)
    res.update({"workload": "c3: batch %d, L=%d, ranges of %d, B=%d" % (b, L, ch, B),
                "candidate_rows_pre_evict": B + ch, "indexer_rows_select_at_end": L,
                "retained_same_set_fraction": float(np.intersect1d(
                    st_e.idx_retained.cpu().numpy(), st_o.idx_retained.cpu().numpy()).size) / B})
    lay_e.close()
    lay_o.close()
    del inp
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ whole-model decode

def model_decode(dev, peak_gbs, steps=8, reps=3):
    """Decode through the retained caches of a whole model: the 36-layer
    workload (batch 64, 2048 retained rows per sequence and layer, memory state
    resident), independent random-init layers, caches filled with N(0,1)
    values (values do not change the work; parity at this shape is a test).
    The caches (about 20 GB) are far beyond L2, so every step streams them
    from HBM. One CUDA graph holds `steps` decode steps through all layers."""
    wl = synth.WORKLOADS["c4"]
    s = wl.shape
    b, B = wl.batch, wl.budget
    cap = B + steps
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    dec = synth.make_decode_inputs(wl, synth.make_weights(s, wl.seed, dev), steps, wl.seed, dev)
    layers = []
    for li in range(wl.n_layers):
        w = synth.make_weights(s, wl.seed + li, dev)
        lay = IndexMemLayer.from_shape(s, w)
        st = lay.new_state(b, B + 1, B, cap, dev)
        st.K_ret.normal_(generator=gen)
        st.V_ret.normal_(generator=gen)
        M0, b0 = synth.make_memory_state(s, b, wl.seed + li, dev)
        st.M.copy_(M0)
        st.bstab.copy_(b0)
        lay.workspace(b, B + 1, B, dev)
        layers.append((lay, st))
        del w
    out = torch.empty_like(dec["q"][0])
    stream = torch.cuda.Stream(dev)

    def run():
        for i in range(steps):
            for lay, st in layers:
                lay.decode(dec["q"][i], dec["k_new"][i], dec["v_new"][i], st, out=out,
                           stream=stream)

    def reset():
        for lay, st in layers:
            st.cache_len.fill_(B)
            lay.invalidate_decode(b, stream=stream)

    with torch.cuda.stream(stream):
        reset()
        run()
        torch.cuda.synchronize()
        reset()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run()
        best = None
        for _ in range(reps):
            reset()
            torch.cuda.synchronize()
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            e.record(stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(e) * 1e-3
            best = t if best is None else min(best, t)
        del g
    for lay, _ in layers:
        lay.sync(stream)
    es = 2 if s.dtype == "bf16" else 4
    row = s.n_kv_heads * s.head_dim * es * 2
    per_launch = b * ((B + (steps + 1) / 2.0) * row +
                      s.n_kv_heads * (s.mem_r * s.head_dim + s.mem_r) * 4 +
                      2 * s.n_q_heads * s.head_dim * es + row / 2)
    launches = steps * wl.n_layers
    gbs = per_launch * launches / best / 1e9
    del layers
    torch.cuda.empty_cache()
    return {"workload": "c4: %d independent layers, batch %d, %d retained rows per sequence and "
                        "layer, memory r=%d, %d decode steps" % (wl.n_layers, b, B, s.mem_r, steps),
            "us_per_layer_step": best / launches * 1e6,
            "tokens_per_s": b * steps / best,
            "bytes_per_launch": per_launch, "GBps": gbs, "hbm_frac": gbs / peak_gbs,
            "note": "caches ~%.1f GB, beyond L2: HBM-bound" % (
                wl.n_layers * 2 * b * cap * s.n_kv_heads * s.head_dim * es / 1e9)}


# ------------------------------------------------------------------ e2e

def run_e2e(job, steps, warmup):
    """Same step through the public API with the step's inputs in pinned host
    memory: H2D copies of X, Q, K, V and the decode inputs, D2H of the decode
    outputs and the retained indices, all inside the timed region. Pipelined as
    a serving loop would: the next step's X, Q, K, V are copied on a second
    stream into a second set of device buffers while the current step
    computes (events keep a set from being overwritten before the step that
    reads it is done); the decode inputs, which the decode graph reads in
    place, are copied on the compute stream just before it."""
    big, dec = ("X", "Q", "K", "V"), ("q", "k_new", "v_new")
    base = job.inp
    sets = [dict(base), {k: torch.empty_like(base[k]) for k in big}]
    # decode inputs travel with the step's other inputs on the copy stream
    # (copies are ordered on the copy engines across streams) and move into
    # the buffers the decode graph reads with an elementwise kernel
    stage = [{k: torch.empty_like(job.decin[k]) for k in dec} for _ in range(2)]
    host_big = {k: base[k].cpu().pin_memory() for k in big}
    host_dec = {k: job.decin[k].cpu().pin_memory() for k in dec}
    host_out = torch.empty(job.out.shape, dtype=job.out.dtype).pin_memory()
    host_idx = torch.empty(job.st.idx_retained.shape, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in list(host_big.values()) + list(host_dec.values()))
    d2h = host_out.numel() * host_out.element_size() + host_idx.numel() * 4
    cs = torch.cuda.Stream(job.dev)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def issue_copy(i):
        s = i % 2
        with torch.cuda.stream(cs):
            if i >= 2:
                cs.wait_event(consumed[s])   # the step two back has read this set
            for k in dec:
                stage[s][k].copy_(host_dec[k], non_blocking=True)
            for k in big:
                sets[s][k].copy_(host_big[k], non_blocking=True)
            copied[s].record(cs)

    def compute(i):
        s = i % 2
        with torch.cuda.stream(job.stream):
            job.stream.wait_event(copied[s])
            for k in dec:
                torch.mul(stage[s][k], 1, out=job.decin[k])   # exact; an SM kernel
            job.inp = sets[s]
            job.step()
            consumed[s].record(job.stream)
            host_out.copy_(job.out, non_blocking=True)
            host_idx.copy_(job.st.idx_retained, non_blocking=True)

    def run(n, start=None):
        if start is not None:
            cs.wait_event(start)
        issue_copy(0)
        if n > 1:
            issue_copy(1)
        for i in range(n):
            compute(i)
            if i + 2 < n:
                issue_copy(i + 2)

    run(max(1, warmup))
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(job.stream)
    run(steps, start=a)
    b.record(job.stream)
    torch.cuda.synchronize()
    job.inp = base
    return a.elapsed_time(b) / steps, h2d, d2h


# ------------------------------------------------------------------ cpu oracle

def cpu_oracle_sample(wl, B, scale=1):
    """Times the CPU oracle on a bounded sample of the workload and scales each
    stage to the full step by its unit count. Returns (seconds per full step,
    description of the sample). `scale` multiplies the sample's tokens, keys,
    evicted tokens and decode steps (1: ~2 s of CPU work, 4: ~10 s)."""
    from oracle import indexmem_oracle as om
    s = wl.shape
    torch.manual_seed(0)
    Ls = min(wl.L, 2048 * scale)               # one sequence, first Ls tokens
    w = synth.make_weights(s, wl.seed, "cpu")
    inp = synth.make_layer_inputs(wl, w, wl.seed, "cpu", L=Ls, batch=1)
    t0 = time.perf_counter()
    qhat, khat, gate = om.indexer_features(inp["X"], inp["Q"], w["W_iq"], w["W_ik"], w["w_ig"])
    t_feat = (time.perf_counter() - t0) / Ls                      # per token
    keys = np.arange(0, Ls, max(1, Ls // (64 * scale)))
    t0 = time.perf_counter()
    om.pooled_importance(qhat, khat, gate, keys=keys)
    pairs_s = sum(Ls - k for k in keys)
    t_pair = (time.perf_counter() - t0) / pairs_s                  # per causal pair
    I = np.random.default_rng(0).standard_normal((1, wl.L))
    t0 = time.perf_counter()
    R, E = om.select_budget(I, B)
    t_sel = time.perf_counter() - t0                               # per sequence
    n_mem = min(512 * scale, Ls - 1)
    Em = np.arange(n_mem)[None]
    t0 = time.perf_counter()
    M, bs = om.memory_update(inp["K"], inp["V"], Em, w["W_phi"], s.lam)
    t_mem = (time.perf_counter() - t0) / n_mem                     # per evicted token
    n_steps = 4 * scale
    dec = synth.make_decode_inputs(wl, w, n_steps, wl.seed, "cpu", batch=1)
    Bs = min(B, Ls)
    KR, VR = om.compact(inp["K"].float().numpy(), inp["V"].float().numpy(), np.arange(Bs)[None],
                        Bs + n_steps)
    f = lambda t: t.float().numpy().astype(np.float64)
    clen = np.array([Bs])
    t0 = time.perf_counter()
    for st in range(n_steps):
        _, clen, _, _, _ = om.decode_step(f(dec["q"][st]), f(dec["k_new"][st]), f(dec["v_new"][st]),
                                          KR, VR, clen, M, bs, f(w["W_phi"]), f(w["w_gate"]))
    t_dec = (time.perf_counter() - t0) / n_steps * (B + wl.n_decode / 2) / (Bs + n_steps / 2)
    pairs_full = wl.batch * wl.L * (wl.L + 1) / 2
    full = (t_feat * wl.batch * wl.L + t_pair * pairs_full + t_sel * wl.batch +
            t_mem * wl.batch * (wl.L - B) + t_dec * wl.batch * wl.n_decode)
    sample = ("1 sequence: indexer features of %d tokens, pooled importance of %d keys over "
              "their causal queries, selection of %d scores, memory update of %d tokens, %d "
              "decode steps at budget %d; each stage scaled to the full step by its unit count "
              "(tokens, causal pairs, sequences, evicted tokens, decode tokens x cache length)"
              % (Ls, len(keys), wl.L, n_mem, n_steps, Bs))
    return full, sample


def oracle_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [os.cpu_count()])
    except Exception:
        return os.cpu_count()


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c2", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-full-cache", action="store_true",
                    help="skip the full-cache decode comparison")
    ap.add_argument("--no-model-decode", action="store_true",
                    help="skip the 36-layer decode measurement")
    ap.add_argument("--no-moment", action="store_true",
                    help="skip the MomentKV readout measurement")
    ap.add_argument("--no-budget-sweep", action="store_true",
                    help="skip the other budgets of the workload")
    ap.add_argument("--no-online", action="store_true",
                    help="skip the decode-time online eviction measurement")
    ap.add_argument("--no-pre-eviction", action="store_true",
                    help="skip the pre-eviction (long-context chunked prefill) measurement")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the whole-step lines of the 4K (c1) and 128K (c3) workloads")
    a = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.WORKLOADS[a.workload]
    B = a.budget or wl.budget
    if wl.n_layers != 1:
        raise SystemExit("the bench step covers single-layer workloads (c0-c3)")
    config = {"workload": "%s: batch %d, L=%d, budget B=%d (%.1f%% eviction), %d decode steps, "
                          "%s, Llama-3.1-8B-shaped layer" % (
                              wl.name, wl.batch, wl.L, B, 100.0 * (wl.L - B) / wl.L, wl.n_decode,
                              wl.shape.dtype),
              "batch": wl.batch, "L": wl.L, "budget": B, "n_decode": wl.n_decode,
              "prefill_chunk": wl.prefill_chunk,
              "l2": "inputs larger than L2: X, Q, K, V (%.2f GiB) are read every step" % (
                  wl.batch * wl.L * (wl.shape.hidden + wl.shape.n_q_heads * wl.shape.head_dim +
                                     2 * wl.shape.n_kv_heads * wl.shape.head_dim) *
                  (2 if wl.shape.dtype == "bf16" else 4) / 2 ** 30),
              "parallelism": "replica per GPU" if world > 1 else "1 GPU"}

    if a.impl == "reference":
        if rank != 0:
            return
        per_step = []
        desc = None
        for i in range(a.warmup + a.steps):
            t, desc = cpu_oracle_sample(wl, B, scale=2)   # ~3 s a step
            if i >= a.warmup:
                per_step.append(t)
        t = statistics.mean(per_step)
        tok = wl.batch * (wl.L + wl.n_decode)
        v = tok / t
        cores = oracle_threads()
        print(json.dumps({
            "metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference",
            "n_gpus": 1, "steps": a.steps, "warmup": a.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    binding.load()
    job = Job(wl, B, dev, wl.seed + 1000 * rank)
    job.capture_decode()
    for _ in range(a.warmup):
        job.step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(a.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    start.record(job.stream)
    for i in range(a.steps):
        job.step(ev[i])
    end.record(job.stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end) / a.steps
    stage_ms = {
        "prefill": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
        "memory": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
        "decode": statistics.mean(e[2].elapsed_time(e[3]) for e in ev),
    }
    ms = reduce_over_ranks(ms, dev, "max")
    layer_sync_ok = True
    try:
        job.layer.sync(job.stream)
    except binding.IndexMemError:
        layer_sync_ok = False

    peaks = load_peaks()
    tokens = job.tokens_per_step() * world
    value = tokens / (ms / 1e3)
    dec_launch_ms = stage_ms["decode"] / job.n_dec
    dec_bytes = job.decode_bytes_per_launch()
    achieved = dec_bytes / (dec_launch_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    stages = {
        "prefill_score_select_compact": {
            "ms": stage_ms["prefill"],
            "indexer_keys_per_s": job.batch * job.L / (stage_ms["prefill"] / 1e3),
            "scoring_tflops_if_all_time": job.scoring_flops() / (stage_ms["prefill"] / 1e3) / 1e12},
        "memory_update": {
            "ms": stage_ms["memory"],
            "evicted_tokens_per_s": job.batch * (job.L - B) / max(stage_ms["memory"], 1e-9) * 1e3,
            "GBps": job.memory_bytes() / max(stage_ms["memory"], 1e-9) / 1e6},
        "decode": {"ms": stage_ms["decode"], "ms_per_launch": dec_launch_ms,
                   "tokens_per_s": job.batch * job.n_dec / (stage_ms["decode"] / 1e3),
                   "GBps": achieved},
    }
    e2e = None
    if not a.no_e2e:
        e2e_ms, h2d, d2h = run_e2e(job, max(2, a.steps // 2), 1)
        e2e_ms = reduce_over_ranks(e2e_ms, dev, "max")
        e2e = {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
    full_cmp = None
    if not a.no_full_cache:
        full_cmp = full_cache_decode(job)
    moment = None
    if not a.no_moment:
        moment = moment_readout(job)
    split = prefill_split(job, peaks)
    stages["prefill_split"] = split
    others = {}
    if not a.no_other_workloads and wl.name == "c2":
        for name in ("c1", "c3"):
            others[name] = other_workload_step(name, dev, synth.WORKLOADS[name].seed + 1000 * rank)
            others[name]["decode_hbm_frac"] = others[name]["decode_GBps"] / peak
    sweep = None
    if not a.no_budget_sweep and wl.name == "c2" and a.budget is None:
        sweep = budget_sweep(wl, dev, wl.seed + 1000 * rank)
    online = None
    if not a.no_online:
        online = online_decode(job)
        if full_cmp is not None:
            online["us_per_step_plain"] = full_cmp["us_per_step_evicted"]
    pre_ev = None
    if not a.no_pre_eviction:
        pre_ev = pre_eviction(dev)
    model_dec = None
    if not a.no_model_decode:
        model_dec = model_decode(dev, peak)
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        t_full, desc = cpu_oracle_sample(wl, B, scale=8)   # ~10-15 s of CPU work
        cpu = {"value": job.tokens_per_step() / t_full, "unit": "tokens/s",
               "cores": oracle_threads(), "kind": "oracle", "sample": desc}
    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "decode_tokens_per_s": stages["decode"]["tokens_per_s"] * world,
            "indexer_keys_per_s": split["indexer_keys_per_s"] * world,
            "value_counts": "b*L context keys + b*n_decode decoded tokens per whole step; "
                            "decode_tokens_per_s and indexer_keys_per_s are the metric's two "
                            "quantities on their own",
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.shape.dtype == "bf16" else "f32", "data": "synthetic",
            "config": config,
            "roofline": {"kernel": "decode", "bound": "hbm", "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak,
                         "traffic": decode_traffic_from_profile(wl.name),
                         "algorithmic_bytes_per_launch": dec_bytes,
                         "peak_source": peaks["source"]},
            "stages": stages,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "full_cache_decode": full_cmp,
            "moment_readout": moment,
            "budget_sweep": sweep,
            "online_eviction": online,
            "pre_eviction": pre_ev,
            "model_decode": model_dec,
            "other_workloads": others or None,
            "roofline_scoring": dict(split["scoring"]["roofline"],
                                     achieved=split["scoring"]["TFLOPs"], kernel="scoring"),
            "roofline_prologue": dict(split["prologue"]["roofline"],
                                      achieved=split["prologue"]["GBps"], kernel="prologue"),
            "gpu_launches": job.launches_per_step() * a.steps,
            "device_errors": not layer_sync_ok,
        }))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
