#!/usr/bin/env python
"""S4R compressed-KV decode benchmark on B200.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl s4r|reference]
                    [--workload 1] [--extra 0,2,3,4,1b,3b | none]
                    [--no-encode] [--no-basis] [--no-cpu-baseline]

Headline (the line's top-level keys): Llama-3-8B-shaped attention, 32 layers
with their own bases, batch 1, prompt L = 32768 (4 sinks + 32764 coefficient
rows), rank 192, top-k 1024, local window 128, query window 16.  One step =
one decode step of all 32 layers, issued as 32 sequential per-layer
s4r_decode_step calls (the layers of a real model run one after another);
each step's calls are captured once in a CUDA graph and replayed.  Step t
uses query rows t .. t+15.

`workloads` (one GPU only) times the other configurations in the same run,
each with its own roofline, end-to-end figure and oracle sample:
  0   tiny fp32 single layer (L = 2048, r = 32);
  2   batched decode, 16 sequences x 32 layers, L = 8192, r = 128;
  3   long context, 32 layers, L = 131072, r = 256;
  4   ragged encode + decode: 8 sequences, L ~ U[4096, 65536], r = 256; each
      step appends one encoded token per sequence, then decodes;
  1b  the headline's 32 layers in ONE call (batch of 32 problems);
  3b  the long-context 32 layers in ONE call.
The layers-in-one-call variants are labelled as such: a real model cannot
batch its layers, whose queries depend on the previous layer's output.

Everything is synthetic (seeded generator, see synth/); the coefficient
caches are made on the GPU by the library's own encode kernel before timing.
Every workload's per-step reads exceed L2 (126 MB) except the tiny one,
which is latency-bound (stated in its entry); no L2 flush is used.

With --gpus N > 1 (torchrun), every rank runs an independent replica of the
headline: the problems shard with no exchange, so there is no collective on
the data path; the timed region is bracketed by barriers and the time is the
max over ranks.  `--impl reference` times the fp64 CPU oracle on the host
cores instead (rank 0 only), on the same workload and config.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "compressed-KV decode steps/s and achieved HBM GB/s (% of roofline) at L=32K"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
EXTRA_DEFAULT = "0,2,3,4,1b,3b,1h"
MAX_WINDOWS = 32          # distinct query windows per workload (steps cycle through them)


# ----------------------------------------------------------------- helpers

def peaks():
    """(HBM GB/s, dense bf16 TFLOP/s burst, source)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a thread."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s=0.01):
        self.samples, self.period, self.ok = [], period_s, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return None
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:   # region shorter than the sampling period: nearest samples
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:2]
        reasons = sorted({name for _, _, rs in inside for bit, name in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(m for _, m, _ in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


def max_over_ranks(x: float, dist, device) -> float:
    """Largest value of x over all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(world: int, steps: int, elapsed_s: float) -> float:
    """Whole-job steps/s: every rank runs its own replica of the workload."""
    return world * steps / elapsed_s


def source_sha(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:16]


def profiled(kernel: str, workload: str):
    """ncu figures of one kernel on one workload from the committed summary
    (profiles/traffic.json): DRAM bytes per launch and the serialised launch
    duration, each only while the sources the entry lists (the kernel's and
    the launch plan's) are unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    d = json.load(open(p)).get(f"{kernel}/{workload}")
    if not d or d.get("source_sha") != source_sha(d["sources"]):
        return None, None
    return d.get("dram_bytes_per_launch"), d.get("ncu_duration_us")


def workload_config(w: synth.Workload, calls: str) -> dict:
    """The `config` object of a workload."""
    L = synth.lengths(w)
    return {"workload": w.name, "layers": w.layers, "batch": w.batch,
            "prompt_len": L[0] if not w.ragged else f"U[{w.ragged[0]}, {w.ragged[1]}] (drawn: {L})",
            "rank": w.rank, "top_k": w.top_k, "local_window": w.local_window,
            "query_window": w.query_window, "n_heads_q": w.n_heads_q, "n_heads_kv": w.n_heads_kv,
            "head_dim": w.head_dim, "n_sink": w.n_sink, "storage": w.dtype,
            "append_per_step": w.append, "calls": calls}


def headline_config(w: synth.Workload, world: int) -> dict:
    """The headline line's `config`, identical in the GPU arm and the
    reference arm."""
    Lc = [L - w.n_sink for L in synth.lengths(w)]
    step_bytes = algorithmic_bytes(w, Lc)[0] * w.layers
    cfg = workload_config(w, HEADLINE_CALLS)
    cfg["l2"] = f"inputs larger than L2: {step_bytes / 1e6:.1f} MB read per step"
    cfg["parallelism"] = f"replicas x{world}"
    return cfg


HEADLINE_CALLS = "32 sequential per-layer calls per step, CUDA graph per step"


# ----------------------------------------------------------------- workload on the GPU

class GpuWorkload:
    """Every (layer, sequence) problem of one replica, resident in HBM.
    Problem p = layer * batch + sequence; the problems of one layer are a
    contiguous slice, so the per-layer calls and the all-layers call read the
    same memory."""

    def __init__(self, w: synth.Workload, replica: int, device, n_windows: int, append_rows: int = 0):
        import rank_decode_attention_b200 as s4r
        self.w, self.dev = w, device
        B, s, Ly, W = w.batch, w.n_sink, w.layers, w.query_window
        self.P = P = B * Ly
        self.L_seq = synth.lengths(w)
        self.Lc = [L - s for L in self.L_seq] * Ly
        self.cap = max(self.Lc) + append_rows
        self.n_windows = n_windows
        sdt = synth.storage_dtype(w.dtype)
        D, r = w.d_model, w.rank
        self.ck = torch.zeros(P, self.cap, r, dtype=sdt, device=device)
        self.cv = torch.zeros_like(self.ck)
        self.bk = torch.empty(P, D, r, dtype=sdt, device=device)
        self.bv = torch.empty_like(self.bk)
        self.sk = torch.empty(P, s, D, dtype=sdt, device=device)
        self.sv = torch.empty_like(self.sk)
        self.q = torch.empty(n_windows, P, W, w.n_heads_q, w.head_dim, dtype=sdt, device=device)
        for layer in range(Ly):
            for b in range(B):
                p = layer * B + b
                pin = synth.problem_inputs(w, layer, b, device=device, L=self.L_seq[b],
                                           n_query_rows=n_windows + W - 1, tag=f"replica{replica}")
                self.bk[p], self.bv[p] = pin.basis_k, pin.basis_v
                self.sk[p], self.sv[p] = pin.states_k[:s], pin.states_v[:s]
                # prefill encode through the library (C = S . B)
                s4r.s4r_encode(pin.states_k[s:], pin.basis_k, self.ck[p, :self.Lc[p]])
                s4r.s4r_encode(pin.states_v[s:], pin.basis_v, self.cv[p, :self.Lc[p]])
                for t in range(n_windows):
                    self.q[t, p] = pin.window(t, W)
                del pin
        # lengths: one tensor per layer (each 16-byte aligned) and one for all problems
        self.lengths0 = torch.tensor(self.Lc, dtype=torch.int32, device=device)
        self.len_layer = [self.lengths0[l * B:(l + 1) * B].clone() for l in range(Ly)]
        self.len_all = self.lengths0.clone()
        self.out = torch.empty(P, w.n_heads_q, w.head_dim, device=device)
        self.idx = torch.empty(P, w.top_k, dtype=torch.int32, device=device)
        if w.append:
            g = torch.Generator(device=device).manual_seed(synth.seed_of(w.name, "append", replica))
            self.new_k = synth.store(torch.randn(n_windows, P, D, generator=g, device=device,
                                                 dtype=torch.float64), w.dtype)
            self.new_v = synth.store(torch.randn(n_windows, P, D, generator=g, device=device,
                                                 dtype=torch.float64), w.dtype)
        torch.cuda.synchronize()
        big = self.args(None, 0)
        self.ws_bytes = max(s4r.s4r_decode_workspace_bytes(big),
                            max(s4r.s4r_decode_workspace_bytes(self.args(l, 0)) for l in range(Ly)))
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        s4r.s4r_workspace_init(self.ws)
        self.launches_layer = s4r.s4r_decode_kernel_launches(self.args(0, 0))
        self.launches_all = s4r.s4r_decode_kernel_launches(big)

    def reset_lengths(self):
        """Undo the appends of a timed pass (append workloads)."""
        self.len_all.copy_(self.lengths0)
        for l, t in enumerate(self.len_layer):
            t.copy_(self.lengths0[l * self.w.batch:(l + 1) * self.w.batch])

    def _slice(self, layer):
        B = self.w.batch
        return slice(0, self.P) if layer is None else slice(layer * B, (layer + 1) * B)

    def args(self, layer, window, events=None):
        """Decode arguments of one layer's problems, or of every problem
        (layer None, the all-layers call)."""
        import rank_decode_attention_b200 as s4r
        sl = self._slice(layer)
        lengths = self.len_all if layer is None else self.len_layer[layer]
        return s4r.decode_args(q=self.q[window, sl], coeff_k=self.ck[sl], coeff_v=self.cv[sl],
                               basis_k=self.bk[sl], basis_v=self.bv[sl], sink_k=self.sk[sl],
                               sink_v=self.sv[sl], lengths=lengths, n_heads_kv=self.w.n_heads_kv,
                               local_window=self.w.local_window, top_k=self.w.top_k,
                               out=self.out[sl], idx=self.idx[sl], workspace=getattr(self, "ws", None),
                               workspace_bytes=getattr(self, "ws_bytes", None),
                               pool_kernel=self.w.pool_kernel, row_mode=self.w.row_mode, profile_events=events)

    def append(self, layer, window):
        import rank_decode_attention_b200 as s4r
        sl = self._slice(layer)
        lengths = self.len_all if layer is None else self.len_layer[layer]
        s4r.s4r_append(state_k=self.new_k[window, sl], state_v=self.new_v[window, sl],
                       basis_k=self.bk[sl], basis_v=self.bv[sl], coeff_k=self.ck[sl], coeff_v=self.cv[sl],
                       lengths=lengths, status_workspace=self.ws)

    def step_calls(self, window, batched=False, events=None):
        """One decode step: the per-layer calls in layer order, or one call."""
        import rank_decode_attention_b200 as s4r
        layers = [None] if batched else list(range(self.w.layers))
        for i, layer in enumerate(layers):
            if self.w.append:
                self.append(layer, window)
            ev = events[i] if events is not None else None
            s4r.s4r_decode_step(self.args(layer, window, ev))

    def calls_per_step(self, batched):
        return 1 if batched else self.w.layers

    def launches_per_step(self, batched):
        per = self.launches_all if batched else self.launches_layer * self.w.layers
        return per + (self.calls_per_step(batched) * 2 if self.w.append else 0)   # append: 2 kernels


def algorithmic_bytes(w: synth.Workload, Lc: list):
    """Per decode call over the given problems: (whole path, scoring kernel).
    Whole path per problem: L_c*r*e (C_K once) + 2(k+w)*r*e (selected C_K and
    C_V rows) + 2*D'*r*e (bases) + 2*s*D'*e (sinks) + W*H_q*d_h*e (queries).
    Scoring kernel per problem: L_c*r*e + R*r*4 (C_Q) + L_c*4 (scores out)."""
    e = 2 if w.dtype == "bf16" else 4
    R = w.query_window * (w.n_heads_q if w.row_mode else w.n_heads_q // w.n_heads_kv)
    step = score = 0
    for L in Lc:
        nsel = min(w.top_k, max(0, L - w.local_window)) + min(w.local_window, L)
        step += (L * w.rank * e + 2 * nsel * w.rank * e + 2 * w.d_model * w.rank * e
                 + 2 * w.n_sink * w.d_model * e + w.query_window * w.n_heads_q * w.head_dim * e)
        score += L * w.rank * e + R * w.rank * 4 + L * 4
    return step, score


def time_decode(wl: GpuWorkload, steps: int, warmup: int, batched: bool, dist, device, world: int,
                clocks: ClockSampler | None = None):
    """Time `steps` decode steps of the workload (CUDA graphs of each step's
    calls), then the same steps again with event pairs around every scoring
    kernel, then end to end through the ABI from pinned host memory."""
    import rank_decode_attention_b200 as s4r
    w = wl.w
    n_win = min(steps, wl.n_windows)
    n_calls = wl.calls_per_step(batched)
    events = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_calls)] for _ in range(n_win)]
    for evs in events:
        for a, b in evs:
            a.record(); b.record()          # materialise the event handles
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device)
    graphs, graphs_ev = [], []
    with torch.cuda.stream(stream):
        wl.step_calls(0, batched)           # warm the launch path before capture
        torch.cuda.synchronize()
        for t in range(n_win):
            for evs, dst in ((None, graphs), (events[t], graphs_ev)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    wl.step_calls(t, batched, evs)
                dst.append(g)
    torch.cuda.synchronize()

    def replay_pass(gs):
        wl.reset_lengths()
        for i in range(warmup):
            gs[i % n_win].replay()
        if w.append:
            torch.cuda.synchronize()
            wl.reset_lengths()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(steps):
                gs[i % n_win].replay()
            e1.record(stream)
        torch.cuda.synchronize()
        h1 = time.perf_counter()
        if dist:
            dist.barrier()
        return max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, device), h0, h1

    torch.cuda.cudart().cudaProfilerStart()   # a profiler started with capture off sees this pass only
    elapsed, h0, h1 = replay_pass(graphs)
    torch.cuda.cudart().cudaProfilerStop()
    clk = clocks.summary(h0, h1) if clocks is not None else None
    elapsed_ev, _, _ = replay_pass(graphs_ev)
    score_ms = []
    for i in range(min(steps, n_win)):
        score_ms += [a.elapsed_time(b) for a, b in events[i]]
    del graphs, graphs_ev

    # End to end through the public API from pinned host memory: every step
    # copies the new query row of every problem (and, when appending, the new
    # token states) host -> device, makes the decode calls directly (no
    # graph) and reads out + idx back to pinned host memory.
    W = w.query_window
    host_q = wl.q.cpu().pin_memory()
    host_out = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
    host_idx = torch.empty(wl.idx.shape, dtype=wl.idx.dtype).pin_memory()
    h2d = host_q[0, :, W - 1].numel() * host_q.element_size()
    if w.append:
        host_nk, host_nv = wl.new_k.cpu().pin_memory(), wl.new_v.cpu().pin_memory()
        h2d += 2 * host_nk[0].numel() * host_nk.element_size()
    d2h = host_out.numel() * 4 + host_idx.numel() * 4
    layers = [None] if batched else list(range(w.layers))
    call_args = [[wl.args(l, t) for l in layers] for t in range(n_win)]
    wl.reset_lengths()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(steps):
            t = i % n_win
            wl.q[t, :, W - 1].copy_(host_q[t, :, W - 1], non_blocking=True)
            if w.append:
                wl.new_k[t].copy_(host_nk[t], non_blocking=True)
                wl.new_v[t].copy_(host_nv[t], non_blocking=True)
            for j, l in enumerate(layers):
                if w.append:
                    wl.append(l, t)
                s4r.s4r_decode_step(call_args[t][j])
            host_out.copy_(wl.out, non_blocking=True)
            host_idx.copy_(wl.idx, non_blocking=True)
        f1.record(stream)
    torch.cuda.synchronize()
    e2e_elapsed = max_over_ranks(f0.elapsed_time(f1) / 1e3, dist, device)
    status = s4r.s4r_read_device_status(wl.ws)
    if status != 0:
        raise RuntimeError(f"{w.name}: device status {status} after the timed passes")
    wl.reset_lengths()
    return {"elapsed": elapsed, "elapsed_ev": elapsed_ev, "score_ms": score_ms, "clocks": clk,
            "e2e": {"value": replica_value(world, steps, e2e_elapsed), "unit": "steps/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}}


def roofline_entry(w, wl, batched, res, steps, hbm, src, label):
    """Roofline of the latent-scoring kernel (the dominant byte mover) and the
    whole path's achieved bandwidth for one timed workload."""
    B = w.batch
    per_call_Lc = wl.Lc if batched else wl.Lc[:B]
    step_bytes_call, score_bytes = algorithmic_bytes(w, per_call_Lc)
    n_calls = wl.calls_per_step(batched)
    step_bytes = step_bytes_call * n_calls
    avg_score_s = statistics.mean(res["score_ms"]) / 1e3
    achieved = score_bytes / avg_score_s / 1e9
    traffic, ncu_us = profiled("latent_scoring", label)
    ms_per_step = res["elapsed"] / steps * 1e3
    return step_bytes, {
        "bound": "hbm", "kernel": "latent_scoring", "achieved": achieved, "peak": hbm, "unit": "GB/s",
        "frac": achieved / hbm, "peak_source": src, "traffic": traffic,
        "algorithmic_bytes_per_launch": score_bytes, "avg_launch_us": avg_score_s * 1e6,
        "launches_timed": len(res["score_ms"]), "ncu_launch_us": ncu_us,
        "timing": "CUDA events on the launching stream around every scoring kernel, in a second timed "
                  "pass of the same steps (the event nodes keep the kernel from overlapping its "
                  "neighbours' launch); ncu_launch_us is ncu's serialised duration of the same launch",
        "ms_per_step_with_events": res["elapsed_ev"] / steps * 1e3,
        "whole_path_gbs": step_bytes / (ms_per_step / 1e3) / 1e9,
        "whole_path_frac": step_bytes / (ms_per_step / 1e3) / 1e9 / hbm}


# ----------------------------------------------------------------- oracle (CPU) leg

def oracle_problem(w: synth.Workload, seq: int = 0, tag="cpu-sample"):
    """One (sequence, layer) problem of the workload at full length, on the CPU."""
    import oracle
    L = synth.lengths(w)[seq]
    pin = synth.problem_inputs(w, 0, seq, L=L, n_query_rows=w.query_window, tag=tag)
    s = w.n_sink
    enc = lambda S, Bm: synth.store(S.double() @ Bm.double(), w.dtype).double().numpy()
    return oracle.Problem(q=pin.window(0, w.query_window).double().numpy(),
                          coeff_k=enc(pin.states_k[s:], pin.basis_k),
                          coeff_v=enc(pin.states_v[s:], pin.basis_v),
                          basis_k=pin.basis_k.double().numpy(), basis_v=pin.basis_v.double().numpy(),
                          sink_k=pin.states_k[:s].double().numpy(), sink_v=pin.states_v[:s].double().numpy(),
                          n_heads_kv=w.n_heads_kv, local_window=w.local_window, top_k=w.top_k,
                          pool_kernel=w.pool_kernel, row_mode=w.row_mode)


def time_oracle(w, budget_s=15.0, max_calls=50, min_calls=1, threads=None):
    """The oracle timed on one full-length problem; steps/s extrapolated to
    every (layer, sequence) problem of a step."""
    import oracle
    p = oracle_problem(w)
    n_cores = oracle.threads() if threads is None else threads
    if threads is not None:
        oracle.set_threads(threads)
    try:
        oracle.decode_step(p)            # warm-up
        times, t_begin = [], time.perf_counter()
        while len(times) < max_calls and (len(times) < min_calls or time.perf_counter() - t_begin < budget_s):
            t0 = time.perf_counter()
            oracle.decode_step(p)
            times.append(time.perf_counter() - t0)
    finally:
        if threads is not None:
            oracle.set_threads(n_cores_all())
    t = statistics.mean(times)
    per_step = w.layers * w.batch
    L = synth.lengths(w)[0]
    return {"value": 1.0 / (t * per_step), "unit": "steps/s", "cores": n_cores, "kind": "oracle",
            "sample": f"{len(times)} oracle decode calls of one (sequence, layer) problem at full length "
                      f"(L={L}, r={w.rank}), mean {t * 1e3:.1f} ms; a step is {per_step} such problems"}


def n_cores_all() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


# ----------------------------------------------------------------- main legs

def run_reference(args, w, rank):
    """The reference arm: the fp64 oracle on the host cores.  One step is the
    full step of the workload: one oracle decode call per (layer, sequence)
    problem, on one full-length problem standing in for each of them."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    p = oracle_problem(w)
    per_step = w.layers * w.batch

    def one_step():
        for _ in range(per_step):
            oracle.decode_step(p)

    for _ in range(args.warmup):
        one_step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        one_step()
        times.append(time.perf_counter() - t0)
    t = statistics.mean(times)
    value = 1.0 / t
    cores = oracle.threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": headline_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step = {per_step} oracle decode calls (one per layer) on one "
                                       f"full-length (sequence, layer) problem (L={synth.lengths(w)[0]}, "
                                       f"r={w.rank})"},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_encode_bench(device, reps=5):
    import rank_decode_attention_b200 as s4r
    n, D, r = synth.BULK_ENCODE_TOKENS, 1024, 256
    g = torch.Generator(device=device).manual_seed(1234)
    S = [synth.store(torch.randn(n, D, generator=g, device=device, dtype=torch.float32), "bf16")
         for _ in range(2)]
    Bs = [synth.store(torch.randn(D, r, generator=g, device=device, dtype=torch.float32) / 32, "bf16")
          for _ in range(2)]
    C = [torch.empty(n, r, dtype=torch.bfloat16, device=device) for _ in range(2)]
    for _ in range(2):
        s4r.s4r_encode2(S, Bs, C)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        s4r.s4r_encode2(S, Bs, C)
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps          # seconds for K + V
    flops = 2 * 2 * n * D * r
    nbytes = 2 * (n * D * 2 + D * r * 2 + n * r * 2)
    hbm, bf16_tf, src = peaks()
    return {"tokens": n, "rank": r, "tokens_per_s": n / t, "ms_k_plus_v": t * 1e3,
            "tflops": flops / t / 1e12, "hbm_gbs": nbytes / t / 1e9,
            "frac_hbm": nbytes / t / 1e9 / hbm, "frac_tensor": flops / t / 1e12 / bf16_tf,
            "peaks": src, "timing": f"CUDA events around {reps} x s4r_encode2 (K and V in one launch), inputs 268 MB"}


def run_basis_bench(w, device, reps=3):
    """Prefill bases for every (layer, K or V) problem of one sequence of the
    workload: 7:3 sample of n_sample non-sink rows, unit-norm rows, top-r
    right singular vectors in fp64 (s4r_build_basis, Eqs. 1-2)."""
    import rank_decode_attention_b200 as s4r
    P, L, D, r = 2 * w.layers, w.prompt_len, w.d_model, w.rank
    states = torch.empty(P, L, D, dtype=synth.storage_dtype(w.dtype), device=device)
    for p in range(P):
        states[p] = synth.states(L, D, w.true_rank, w.n_sink, w.n_needles, w.needle_middle,
                                 synth.seed_of(w.name, "basis", p), device).to(torch.float32).to(states.dtype)
    lengths = torch.full((P,), L, dtype=torch.int32, device=device)
    out = torch.empty(P, D, r, dtype=states.dtype, device=device)
    a = s4r.basis_args(states=states, lengths=lengths, rank=r, n_sink=w.n_sink, n_sample=w.n_sample)
    ws = torch.empty(s4r.s4r_basis_workspace_bytes(a), dtype=torch.uint8, device=device)
    s4r.s4r_workspace_init(ws)
    a = s4r.basis_args(states=states, lengths=lengths, rank=r, n_sink=w.n_sink, n_sample=w.n_sample,
                       basis_out=out, workspace=ws)
    s4r.s4r_build_basis(a)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        s4r.s4r_build_basis(a)
    e1.record()
    torch.cuda.synchronize()
    status = s4r.s4r_read_device_status(ws)
    t = e0.elapsed_time(e1) / reps / 1e3
    m = min(w.n_sample, D)
    del states
    return {"problems": P, "n_sample": w.n_sample, "rank": r, "gram_dim": m, "ms_all_problems": t * 1e3,
            "us_per_basis": t / P * 1e6, "status": s4r.s4r_status_string(status),
            "timing": "CUDA events around the whole call (6 kernels: sample norms, Gram, "
                      "cooperative Jacobi sweeps, order, columns, sign and output), mean of "
                      f"{reps} calls after one untimed call"}


def run_extra(key, args, device):
    """One entry of `workloads`: a configuration other than the headline."""
    batched = key.endswith("b")
    per_head = key.endswith("h")
    w = synth.WORKLOADS[int(key.rstrip("bh"))]
    if per_head:
        # the per-head reading of the scoring rows (W * H_q of them)
        w = dataclasses.replace(w, row_mode=1)
    steps = min(args.steps, w.steps) if w.append else args.steps
    n_win = max(1, min(steps, w.steps, MAX_WINDOWS))
    append_rows = (args.warmup + 3 * steps + 8) if w.append else 0
    wl = GpuWorkload(w, 0, device, n_win, append_rows=append_rows)
    res = time_decode(wl, steps, args.warmup, batched, None, device, 1)
    hbm, _, src = peaks()
    label = w.name + ("/layers-in-one-call" if batched else "") + ("/per-head-rows" if per_head else "")
    step_bytes, roof = roofline_entry(w, wl, batched, res, steps, hbm, src, label)
    calls = (f"all {w.layers * w.batch} (layer, sequence) problems in ONE call per step (layers batched, "
             "not a model's sequential order), CUDA graph per step") if batched else \
        (f"{w.layers} sequential per-layer calls per step" if w.layers > 1 else "1 call per step") + \
        (", each preceded by s4r_append of one token per sequence" if w.append else "") + ", CUDA graph per step"
    cfg = workload_config(w, calls)
    l2 = ("per-step reads exceed L2" if step_bytes > 126e6 else
          "per-step reads fit in L2 (latency-bound; no flush)")
    cfg["l2"] = f"{l2}: {step_bytes / 1e6:.1f} MB read per step"
    entry = {"value": replica_value(1, steps, res["elapsed"]), "unit": "steps/s", "steps": steps,
             "warmup": args.warmup, "ms_per_step": res["elapsed"] / steps * 1e3, "config": cfg,
             "roofline": roof, "e2e": res["e2e"], "gpu_launches": steps * wl.launches_per_step(batched),
             "clocks": None}
    if not args.no_cpu_baseline:
        entry["cpu_baseline"] = time_oracle(w, budget_s=3.0, max_calls=3)
    del wl
    torch.cuda.empty_cache()
    return label, entry


def run_s4r(args, w, rank, world, local_rank):
    import rank_decode_attention_b200 as s4r
    s4r.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = torch.distributed if world > 1 else None
    n_windows = max(1, min(args.steps, w.steps, 64))
    wl = GpuWorkload(w, rank, device, n_windows)
    clocks = ClockSampler(device.index)
    clocks.start()
    time.sleep(0.05)
    res = time_decode(wl, args.steps, args.warmup, False, dist, device, world, clocks)
    clocks.stop()
    value = replica_value(world, args.steps, res["elapsed"])
    launches = wl.launches_per_step(False)
    if rank != 0:
        return
    hbm, bf16_tf, src = peaks()
    step_bytes, roof = roofline_entry(w, wl, False, res, args.steps, hbm, src, w.name)
    del wl
    torch.cuda.empty_cache()
    cfg = headline_config(w, world)
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["elapsed"] / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "storage": w.dtype, "data": "synthetic",
        "config": cfg,
        "achieved_step_gbs": roof["whole_path_gbs"],
        "roofline": roof,
        "e2e": res["e2e"],
        "gpu_launches": args.steps * launches,
        "clocks": res["clocks"],
    }
    if world == 1 and args.extra != "none":
        line["workloads"] = {}
        for key in args.extra.split(","):
            label, entry = run_extra(key.strip(), args, device)
            line["workloads"][label] = entry
    if not args.no_encode:
        line["encode"] = run_encode_bench(device)
    if not args.no_basis and world == 1:
        line["basis"] = run_basis_bench(w, device)
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        cpu = time_oracle(w)
        cpu["single_thread"] = time_oracle(w, budget_s=4.0, max_calls=3, min_calls=2, threads=1)
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def run_profile_case(args, w: synth.Workload):
    """A short untimed run for ncu captures (committed so that every profile
    summary names a command of this repository): `decode` makes four
    s4r_decode_step calls on one layer of the workload (every problem of that
    layer), `encode` three s4r_encode2 calls of the bulk K + V encode."""
    import rank_decode_attention_b200 as s4r
    dev = torch.device("cuda", 0)
    if args.profile_case == "encode":
        n, D, r = synth.BULK_ENCODE_TOKENS, 1024, 256
        g = torch.Generator(device=dev).manual_seed(1234)
        S = [synth.store(torch.randn(n, D, generator=g, device=dev, dtype=torch.float32), "bf16") for _ in range(2)]
        Bs = [synth.store(torch.randn(D, r, generator=g, device=dev, dtype=torch.float32) / 32, "bf16")
              for _ in range(2)]
        C = [torch.empty(n, r, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        for _ in range(3):
            s4r.s4r_encode2(S, Bs, C)
        calls = 3
    else:
        wl = GpuWorkload(dataclasses.replace(w, layers=1), 0, dev, 1)
        for _ in range(4):
            wl.step_calls(0)
        calls = 4
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": args.profile_case, "workload": w.name, "calls": calls}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="s4r", choices=["s4r", "reference"])
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--extra", default=EXTRA_DEFAULT,
                    help="comma list of other workloads to time on one GPU (0,2,3,4,1b,3b,1h) or 'none'")
    ap.add_argument("--no-encode", action="store_true")
    ap.add_argument("--no-basis", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=["decode", "encode"],
                    help="untimed small case for ncu: one layer of --workload, or the bulk encode")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.profile_case:
        run_profile_case(args, w)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_s4r(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
