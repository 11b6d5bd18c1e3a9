#!/usr/bin/env python
"""S4R compressed-KV decode benchmark on B200.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl s4r|reference]
                    [--workload 1] [--no-encode] [--no-basis]

Workload (default 1): Llama-3-8B-shaped attention, 32 layers with their own
bases, batch 1, prompt L = 32768 (4 sinks + 32764 coefficient rows), rank 192,
top-k 1024, local window 128, query window 16.  One step = one decode step of
all 32 layers, issued as 32 sequential per-layer s4r_decode_step calls (the
layers of a real model run one after another); each step's calls are captured
once in a CUDA graph and replayed.  Step t uses query rows t .. t+15.

Everything is synthetic (seeded generator, see synth/); the coefficient
caches are made on the GPU by the library's own encode kernel before timing.
The caches (805 MB) exceed L2 (126 MB) and each step streams 460.8 MB, so no
L2 flush is needed between steps.

With --gpus N > 1 (torchrun), every rank runs an independent replica of the
workload: the problems shard with no exchange, so there is no collective on
the data path; the timed region is bracketed by barriers and the time is the
max over ranks.  `--impl reference` times the fp64 CPU oracle on the host
cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
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


# ----------------------------------------------------------------- helpers

def peaks():
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


def profiled_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, only while the
    kernel source is unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d or d.get("source_sha") != source_sha(d["sources"]):
        return None
    return d["dram_bytes_per_launch"]


# ----------------------------------------------------------------- workload on the GPU

class GpuWorkload:
    """All layers of one replica, resident in HBM."""

    def __init__(self, w: synth.Workload, replica: int, device, n_windows: int):
        import rank_decode_attention_b200 as s4r
        self.w, self.dev = w, device
        B, s = w.batch, w.n_sink
        self.Lc = [L - s for L in synth.lengths(w)]
        self.cap = max(self.Lc)
        self.n_windows = n_windows
        sdt = synth.storage_dtype(w.dtype)
        self.layers = []
        for layer in range(w.layers):
            ck = torch.zeros(B, self.cap, w.rank, dtype=sdt, device=device)
            cv = torch.zeros_like(ck)
            bk = torch.empty(B, w.d_model, w.rank, dtype=sdt, device=device)
            bv = torch.empty_like(bk)
            sk = torch.empty(B, s, w.d_model, dtype=sdt, device=device)
            sv = torch.empty_like(sk)
            qs = torch.empty(n_windows, B, w.query_window, w.n_heads_q, w.head_dim, dtype=sdt,
                             device=device)
            for b in range(B):
                pin = synth.problem_inputs(w, layer, b, device=device, L=self.Lc[b] + s,
                                           n_query_rows=n_windows + w.query_window - 1,
                                           tag=f"replica{replica}")
                bk[b], bv[b] = pin.basis_k, pin.basis_v
                sk[b], sv[b] = pin.states_k[:s], pin.states_v[:s]
                # prefill encode through the library (C = S . B)
                s4r.s4r_encode(pin.states_k[s:], pin.basis_k, ck[b, :self.Lc[b]])
                s4r.s4r_encode(pin.states_v[s:], pin.basis_v, cv[b, :self.Lc[b]])
                for t in range(n_windows):
                    qs[t, b] = pin.window(t, w.query_window)
                del pin
            lengths = torch.tensor(self.Lc, dtype=torch.int32, device=device)
            self.layers.append(dict(ck=ck, cv=cv, bk=bk, bv=bv, sk=sk, sv=sv, q=qs, lengths=lengths))
        torch.cuda.synchronize()
        L0 = self.layers[0]
        self.out = torch.empty(w.layers, B, w.n_heads_q, w.head_dim, device=device)
        self.idx = torch.empty(w.layers, B, w.top_k, dtype=torch.int32, device=device)
        a = self.args(0, 0)
        self.ws_bytes = s4r.s4r_decode_workspace_bytes(a)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        s4r.s4r_workspace_init(self.ws)
        self.launches_per_call = s4r.s4r_decode_kernel_launches(a)

    def args(self, layer, window, events=None):
        import rank_decode_attention_b200 as s4r
        L = self.layers[layer]
        return s4r.decode_args(q=L["q"][window], coeff_k=L["ck"], coeff_v=L["cv"], basis_k=L["bk"],
                               basis_v=L["bv"], sink_k=L["sk"], sink_v=L["sv"],
                               lengths=L["lengths"], n_heads_kv=self.w.n_heads_kv,
                               local_window=self.w.local_window, top_k=self.w.top_k,
                               out=self.out[layer], idx=self.idx[layer],
                               workspace=getattr(self, "ws", None),
                               workspace_bytes=getattr(self, "ws_bytes", None),
                               pool_kernel=self.w.pool_kernel, profile_events=events)

    def step_calls(self, window, events=None):
        import rank_decode_attention_b200 as s4r
        for layer in range(self.w.layers):
            ev = events[layer] if events is not None else None
            s4r.s4r_decode_step(self.args(layer, window, ev))


def algorithmic_bytes(w: synth.Workload, Lc: list):
    """Per decode call (one layer, all problems): (whole step, scoring kernel).
    Whole step per problem: L_c*r*e (C_K once) + 2(k+w)*r*e (selected C_K and
    C_V rows) + 2*D'*r*e (bases) + 2*s*D'*e (sinks) + W*H_q*d_h*e (queries).
    Scoring kernel per problem: L_c*r*e + R*r*4 (C_Q) + L_c*4 (scores out)."""
    e = 2 if w.dtype == "bf16" else 4
    R = w.query_window * (w.n_heads_q // w.n_heads_kv)
    step = score = 0
    for L in Lc:
        nsel = min(w.top_k, max(0, L - w.local_window)) + min(w.local_window, L)
        step += (L * w.rank * e + 2 * nsel * w.rank * e + 2 * w.d_model * w.rank * e
                 + 2 * w.n_sink * w.d_model * e + w.query_window * w.n_heads_q * w.head_dim * e)
        score += L * w.rank * e + R * w.rank * 4 + L * 4
    return step, score


# ----------------------------------------------------------------- oracle (CPU) leg

def oracle_layer_sample(w: synth.Workload):
    """One (sequence, layer) problem of the workload at full length, on the CPU."""
    import oracle
    L = synth.lengths(w)[0]
    pin = synth.problem_inputs(w, 0, 0, L=L, n_query_rows=w.query_window, tag="cpu-sample")
    s = w.n_sink
    enc = lambda S, Bm: synth.store(S.double() @ Bm.double(), w.dtype).double().numpy()
    p = oracle.Problem(q=pin.window(0, w.query_window).double().numpy(),
                       coeff_k=enc(pin.states_k[s:], pin.basis_k),
                       coeff_v=enc(pin.states_v[s:], pin.basis_v),
                       basis_k=pin.basis_k.double().numpy(), basis_v=pin.basis_v.double().numpy(),
                       sink_k=pin.states_k[:s].double().numpy(), sink_v=pin.states_v[:s].double().numpy(),
                       n_heads_kv=w.n_heads_kv, local_window=w.local_window, top_k=w.top_k,
                       pool_kernel=w.pool_kernel)
    return p


def time_oracle(w, n_calls=None, budget_s=15.0, warmup=1):
    import oracle
    p = oracle_layer_sample(w)
    for _ in range(warmup):
        oracle.decode_step(p)
    times, t_begin = [], time.perf_counter()
    while True:
        t0 = time.perf_counter()
        oracle.decode_step(p)
        times.append(time.perf_counter() - t0)
        if n_calls is not None and len(times) >= n_calls:
            break
        if n_calls is None and (time.perf_counter() - t_begin > budget_s or len(times) >= 50):
            break
    t = statistics.mean(times)
    problems_per_step = w.layers * w.batch
    return {"value": 1.0 / (t * problems_per_step), "unit": "steps/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"{len(times)} oracle decode calls of one (sequence, layer) problem at full "
                      f"length (L={synth.lengths(w)[0]}, r={w.rank}); a step is {problems_per_step} "
                      f"such problems, mean {t * 1e3:.1f} ms per problem"}, times


# ----------------------------------------------------------------- main legs

def run_reference(args, w, rank):
    if rank != 0:
        return
    import oracle
    oracle.build()
    p = oracle_layer_sample(w)
    for _ in range(args.warmup):
        oracle.decode_step(p)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode_step(p)
        times.append(time.perf_counter() - t0)
    t = statistics.mean(times) * w.layers * w.batch
    value = 1.0 / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "layers": w.layers, "batch": w.batch,
                       "prompt_len": synth.lengths(w)[0], "rank": w.rank, "top_k": w.top_k,
                       "local_window": w.local_window, "query_window": w.query_window},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": oracle.threads(),
                             "kind": "oracle",
                             "sample": f"each step = one oracle decode call of one (sequence, layer) "
                                       f"problem at full length, scaled by {w.layers * w.batch} "
                                       f"problems per step"},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_encode_bench(w, device, reps=5):
    import rank_decode_attention_b200 as s4r
    n, D, r = synth.BULK_ENCODE_TOKENS, w.d_model, 256
    g = torch.Generator(device=device).manual_seed(1234)
    S = [synth.store(torch.randn(n, D, generator=g, device=device, dtype=torch.float32), "bf16")
         for _ in range(2)]
    Bs = [synth.store(torch.randn(D, r, generator=g, device=device, dtype=torch.float32) / 32, "bf16")
          for _ in range(2)]
    C = [torch.empty(n, r, dtype=torch.bfloat16, device=device) for _ in range(2)]
    for _ in range(2):
        for i in range(2):
            s4r.s4r_encode(S[i], Bs[i], C[i])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        for i in range(2):
            s4r.s4r_encode(S[i], Bs[i], C[i])
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps          # seconds for K + V
    flops = 2 * 2 * n * D * r
    nbytes = 2 * (n * D * 2 + D * r * 2 + n * r * 2)
    hbm, bf16_tf, src = peaks()
    return {"tokens": n, "rank": r, "tokens_per_s": n / t, "ms_k_plus_v": t * 1e3,
            "tflops": flops / t / 1e12, "hbm_gbs": nbytes / t / 1e9,
            "frac_hbm": nbytes / t / 1e9 / hbm, "frac_tensor": flops / t / 1e12 / bf16_tf,
            "peaks": src}


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
                      "cooperative Jacobi sweeps, order, columns, sign and output)"}


def run_s4r(args, w, rank, world, local_rank):
    import rank_decode_attention_b200 as s4r
    s4r.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = torch.distributed if world > 1 else None
    n_windows = max(1, min(args.steps, w.steps))
    wl = GpuWorkload(w, rank, device, n_windows)
    # One graph per distinct query window holding the 32 per-layer calls.  A
    # second set carries an event pair around every layer's scoring kernel;
    # it is timed in its own pass, because event nodes between kernels stop
    # the kernels on either side from overlapping their launch.
    events = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(w.layers)] for _ in range(n_windows)]
    for evs in events:
        for a, b in evs:
            a.record(); b.record()          # materialise the event handles
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device)
    graphs, graphs_ev = [], []
    with torch.cuda.stream(stream):
        wl.step_calls(0)                    # warm the launch path before capture
        torch.cuda.synchronize()
        for t in range(n_windows):
            for evs, dst in ((None, graphs), (events[t], graphs_ev)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    wl.step_calls(t, evs)
                dst.append(g)
    torch.cuda.synchronize()
    for i in range(args.warmup):
        graphs[i % n_windows].replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(device.index)
    clocks.start()
    time.sleep(0.05)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    torch.cuda.cudart().cudaProfilerStart()   # a profiler started with capture off sees this region only
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(args.steps):
            graphs[i % n_windows].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStop()
    h1 = time.perf_counter()
    if dist:
        dist.barrier()
    clocks.stop()
    elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, device)
    value = replica_value(world, args.steps, elapsed)

    # The same K steps again with the event pairs around the scoring kernels.
    graphs_ev[0].replay()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(args.steps):
            graphs_ev[i % n_windows].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    elapsed_ev = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, device)
    score_ms = []
    for i in range(min(args.steps, n_windows)):
        score_ms += [a.elapsed_time(b) for a, b in events[i]]

    # End to end through the public API from pinned host memory: every step
    # copies its new query row of every layer host->device, makes the 32
    # per-layer s4r_decode_step calls (no graph) and reads the outputs
    # (out + idx) back to pinned host memory.
    B, W = w.batch, w.query_window
    call_args = [[wl.args(l, t) for l in range(w.layers)] for t in range(n_windows)]
    host_q = [wl.layers[l]["q"].cpu().pin_memory() for l in range(w.layers)]
    host_out = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
    host_idx = torch.empty(wl.idx.shape, dtype=wl.idx.dtype).pin_memory()
    h2d = sum(hq[0, :, W - 1].numel() * hq.element_size() for hq in host_q)
    d2h = host_out.numel() * 4 + host_idx.numel() * 4
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(args.steps):
            t = i % n_windows
            for l in range(w.layers):
                wl.layers[l]["q"][t, :, W - 1].copy_(host_q[l][t, :, W - 1], non_blocking=True)
            for l in range(w.layers):
                s4r.s4r_decode_step(call_args[t][l])
            host_out.copy_(wl.out, non_blocking=True)
            host_idx.copy_(wl.idx, non_blocking=True)
        f1.record(stream)
    torch.cuda.synchronize()
    e2e_elapsed = max_over_ranks(f0.elapsed_time(f1) / 1e3, dist, device)
    e2e_value = replica_value(world, args.steps, e2e_elapsed)

    status = s4r.s4r_read_device_status(wl.ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    if rank != 0:
        return
    hbm, bf16_tf, src = peaks()
    step_bytes, score_bytes = algorithmic_bytes(w, wl.Lc)
    avg_score_s = statistics.mean(score_ms) / 1e3
    achieved = score_bytes / avg_score_s / 1e9
    traffic = profiled_traffic("latent_scoring")
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "storage": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "batch": w.batch,
                   "prompt_len": synth.lengths(w)[0], "rank": w.rank, "top_k": w.top_k,
                   "local_window": w.local_window, "query_window": w.query_window,
                   "n_heads_q": w.n_heads_q, "n_heads_kv": w.n_heads_kv, "head_dim": w.head_dim,
                   "calls": "32 sequential per-layer calls per step, CUDA graph per step",
                   "l2": f"inputs larger than L2: {step_bytes * w.layers / 1e6:.1f} MB read per step",
                   "parallelism": f"replicas x{world}"},
        "achieved_step_gbs": step_bytes * w.layers / (elapsed / args.steps) / 1e9,
        "roofline": {"bound": "hbm", "kernel": "latent_scoring", "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "peak_source": src,
                     "traffic": traffic, "algorithmic_bytes_per_launch": score_bytes,
                     "avg_launch_us": avg_score_s * 1e6, "launches_timed": len(score_ms),
                     "timing": "CUDA events on the launching stream around every layer's scoring kernel, "
                               "in a second timed pass of the same steps",
                     "ms_per_step_with_events": elapsed_ev / args.steps * 1e3},
        "e2e": {"value": e2e_value, "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * w.layers * wl.launches_per_call,
        "clocks": clocks.summary(h0, h1),
    }
    if not args.no_encode:
        line["encode"] = run_encode_bench(w, device)
    if not args.no_basis and world == 1:
        line["basis"] = run_basis_bench(w, device)
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        cpu, _ = time_oracle(w)
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="s4r", choices=["s4r", "reference"])
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--no-encode", action="store_true")
    ap.add_argument("--no-basis", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
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
