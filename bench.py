"""Benchmark of the ARL2 hybrid attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 480p_bf16]
                    [--impl reference]

One step = one whole stream of the workload through the C ABI: state reset,
then every frame's denoising passes (read-only passes, then the clean pass
that updates the state).  For the default 480p workload that is 21 latent
frames x 4 passes of 12 heads x 128 dims x 1560 tokens.  Inputs for every
pass are generated once, resident in HBM (1.2 GB, larger than the 126 MB L2)
before timing starts.

Printed (rank 0, one JSON line): frames/s over all ranks, the fused
attention kernel's roofline (algorithmic FLOPs per launch over its
CUDA-event duration, against the measured bf16 tensor peak), SM clocks
sampled during the timed region, an end-to-end number through the
host-buffer entry point, and the CPU oracle's frames/s on a bounded sample.

N > 1 (torchrun): every rank runs its own independent stream (replicas, no
collective on the data path); the time is the max over ranks.
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
import torch

import workloads

ROOT = os.path.dirname(os.path.abspath(__file__))


# ----------------------------------------------------------------- flops --
def attn_flops(w: workloads.Workload) -> float:
    """Algorithmic FLOPs of one fused-kernel launch: intra-frame softmax
    attention 4 L^2 d H plus the state read 2 L d^2 H, per stream."""
    L, d, H, B = w.tokens, w.head_dim, w.heads, w.batch
    return (4.0 * L * L * d * H + 2.0 * L * d * d * H) * B


def frame_flops(w: workloads.Workload) -> float:
    """Algorithmic FLOPs of one frame: every pass 4L^2dH + 2Ld^2H + 2Ld^2H
    (intra, read, phi_q); the clean pass adds 4Ld^2H (phi_k, phi_v) and
    4Ld^2H (update)."""
    L, d, H, B = w.tokens, w.head_dim, w.heads, w.batch
    per_pass = 4.0 * L * L * d * H + 4.0 * L * d * d * H
    return B * (w.passes * per_pass + 8.0 * L * d * d * H)


def measured_traffic(workload: str) -> int | None:
    """DRAM bytes per launch of the fused kernel from the last ncu capture
    (profiles/attn_tc_traffic.json), or None once the kernel source has
    changed since that capture, or for a workload other than the captured
    one."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "attn_tc_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d["workload"].split()[0] != workload:
            return None
        h = hashlib.sha256()
        for rel in d["source_files"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        return int(d["dram_bytes_per_launch"]) if h.hexdigest() == d["source_sha256"] else None
    except (OSError, KeyError, ValueError):
        return None


def fp32_simt_tflops() -> float:
    """Peak fp32 FMA throughput from the unit counts and the clock: 148 SMs x
    128 FP32 lanes x 2 flop per FMA x 1965 MHz (B200)."""
    return 148 * 128 * 2 * 1.965e9 / 1e12


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------- clocks --
class ClockSampler:
    """SM clock, power and clock-event reasons sampled every ~2 ms during the
    timed region by a host thread reading NVML (nvidia-ml-py), so that even a
    region of a few tens of milliseconds carries its own samples.  start()
    before the region, stop() right after it: the samples taken in between
    are summarised.  Without NVML, nvidia-smi's loop mode (50 ms) is used and
    only the samples nearest the region remain."""

    INTERVAL_S = 0.002
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device: int):
        import threading
        self.samples = []
        self.max_mhz = None
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._smi = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByUUID(ident.encode())
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            self._bits = [(n, getattr(pynvml, c)) for n, c in self.REASONS if hasattr(pynvml, c)]
            self.source = "nvml"
        except Exception:
            self._nv = None
            self._smi = _SmiSampler(device)
            self.source = "nvidia-smi" if self._smi.proc is not None else None

    def _poll(self):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                watts = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((mhz, watts, {n for n, b in self._bits if bits & b}))
            except Exception:
                pass
            time.sleep(self.INTERVAL_S)

    def start(self) -> None:
        import threading
        if self._nv is not None:
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
            t_end = time.time() + 2.0  # the region starts once samples flow
            while not self.samples and time.time() < t_end:
                time.sleep(0.001)
            self.samples.clear()
        self._t0 = time.time()

    def stop(self) -> dict | None:
        t1 = time.time()
        if self._nv is None:
            return self._smi.summary(self._t0, t1) if self._smi is not None else None
        self._stop.set()
        self._thread.join(timeout=5)
        inside = list(self.samples)
        if not inside:
            return None
        sm = [x[0] for x in inside]
        loaded = [v for v in sm if v > 0.5 * self.max_mhz] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(set().union(*(x[2] for x in inside))), "samples": len(inside),
                "power_w_max": max(x[1] for x in inside), "source": "nvml, every ~2 ms"}


class _SmiSampler:
    """Fallback: nvidia-smi's loop mode every 50 ms."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        import tempfile
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.path = os.path.join(tempfile.gettempdir(), f"clocks_{os.getpid()}.csv")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", ident, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t_end = time.time() + 10.0
            while time.time() < t_end and self.proc.poll() is None and os.path.getsize(self.path) == 0:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def summary(self, t0: float, t1: float) -> dict | None:
        import datetime
        time.sleep(0.1)  # one sample after the region
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
            rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        except Exception:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        parsed = []
        for r in rows:
            r = [x.strip() for x in r]
            try:
                when = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                parsed.append((when, float(r[2]), float(r[3]),
                               {n for n, v in zip(names, r[6:10]) if v.lower() in ("active", "0x1", "1")}))
            except (ValueError, IndexError):
                continue
        if not parsed:
            return None
        inside = [p for p in parsed if t0 <= p[0] <= t1]
        if not inside:
            inside = [p for p in parsed if p[0] < t0][-1:] + [p for p in parsed if p[0] > t1][:1]
        sm = [p[1] for p in inside]
        mx = max(p[2] for p in parsed)
        loaded = [v for v in sm if v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(set().union(*(p[3] for p in inside))), "samples": len(inside),
                "source": "nvidia-smi, every 50 ms"}


# ------------------------------------------------------------ distributed --
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """The slowest rank's time (NCCL on the GPU; gloo keeps the tensor on the host)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(frames_per_rank: int, ws: int, t_max_ms: float) -> float:
    """Frames per second of the whole job: every rank's frames over the slowest rank's time."""
    return frames_per_rank * ws / (t_max_ms / 1e3)


# -------------------------------------------------------------- CPU side --
def oracle_frame(w: workloads.Workload, ins, wq, wk, wv, alpha, beta, S):
    """One whole frame through the CPU oracle as it stands: every pass's
    full output (all L rows of every head) and the clean pass's state
    update.  Returns the state after the frame."""
    import oracle
    for p in range(w.passes):
        q, k, v = ins[p]
        _, S = oracle.frame_pass(q, k, v, wq, wk, wv, alpha, beta, S, workloads.is_clean(w, p))
    return S


def oracle_frame_seconds(w: workloads.Workload, budget_s: float = 10.0):
    """Time the CPU oracle on whole frames of the workload (frame 0's inputs,
    carried state) until `budget_s` of work is done (one frame at least).
    Returns (seconds per frame, threads, description)."""
    import oracle
    oracle.build()
    wq, wk, wv = workloads.phi_weights(w, 0)
    alpha, beta = workloads.frame_gates(w, 0, 0)
    ins = [workloads.pass_inputs(w, 0, 0, p) for p in range(w.passes)]
    S = oracle.zero_state(w.batch, w.heads, w.head_dim)
    n, t0 = 0, time.perf_counter()
    while True:
        S = oracle_frame(w, ins, wq, wk, wv, alpha, beta, S)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    per_frame = (time.perf_counter() - t0) / n
    desc = (f"oracle fp64 (C, OpenMP): {n} whole {w.name} frame(s), every pass's full output and the "
            f"clean pass's state update, {per_frame:.2f} s per frame")
    return per_frame, oracle_threads(), desc


def oracle_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS, else the cores
    this process may run on)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


METRIC = "hybrid-attn frames/s (12h x 128d, 1560 tok/frame) & % of B200 BF16 tensor peak"


def arm_config(args, w: workloads.Workload, ws: int) -> dict:
    """The `config` object of the bench line, the same for both arms."""
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "head_dim": w.head_dim,
            "tokens_per_frame": w.tokens, "frames_per_step": w.frames, "passes": w.passes,
            "parallelism": f"replicas{ws}", "l2": "inputs larger than L2 (1.2 GB ring)",
            "gating": args.gating, "access": args.access, "gates": args.gates}


def run_reference(args, w: workloads.Workload):
    """--impl reference: the CPU oracle as it stands.  One step is one whole
    frame of the workload (every pass's full output and the clean pass's
    state update), timed on the host; the state carries across steps."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    wq, wk, wv = workloads.phi_weights(w, 0)
    alpha, beta = workloads.frame_gates(w, 0, 0)
    ins = [workloads.pass_inputs(w, 0, 0, p) for p in range(w.passes)]
    S = oracle.zero_state(w.batch, w.heads, w.head_dim)
    for _ in range(args.warmup):
        S = oracle_frame(w, ins, wq, wk, wv, alpha, beta, S)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        S = oracle_frame(w, ins, wq, wk, wv, alpha, beta, S)
    secs = time.perf_counter() - t0
    spf = secs / max(1, args.steps)
    value = w.batch / spf
    sample = (f"per step: one whole {w.name} frame (all {w.passes} passes' full outputs and the clean "
              f"pass's state update) through the fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "frames/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": spf * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": arm_config(args, w, ws),
        "cpu_baseline": {"value": value, "unit": "frames/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------- GPU side --
def profile_teacher_case(args, w: workloads.Workload) -> int:
    """Profiling case of the teacher layer: a cache of --profile-teacher
    frames loaded directly (cache_set, no attention launches), then
    --profile-passes passes over a ring of inputs, the last one clean."""
    from hybrid_softmax_gated_b200 import TeacherLayer
    n = args.profile_teacher
    B, L, H, d = w.batch, w.tokens, w.heads, w.head_dim
    tea = TeacherLayer(B, H, d, L, n + 1, dtype=w.torch_dtype)
    g = torch.Generator(device="cuda").manual_seed(workloads.subseed(workloads.SEED_BASE, 7, n))
    kc = torch.randn(B, n * L, H, d, generator=g, device="cuda").to(w.torch_dtype)
    vc = torch.randn(B, n * L, H, d, generator=g, device="cuda").to(w.torch_dtype)
    tea.cache_set(kc, vc)
    ring = 4
    ins = [workloads.pass_inputs(w, 0, 0, i, device="cuda") for i in range(ring)]
    out = torch.empty_like(ins[0][0])
    passes = max(1, args.profile_passes)
    for i in range(passes):  # the last pass is clean: it appends to the cache
        tea.forward(*ins[i % ring], clean_pass=i == passes - 1, out=out)
    torch.cuda.synchronize()
    st = tea.device_status()
    tea.close()
    print(f"teacher profile case {w.name}: {n} cached frames ({n * L} keys), "
          f"{passes} passes (the last one clean), status {st}")
    return 0 if st == 0 else 1


def profile_gates_case(args, w: workloads.Workload) -> int:
    """Profiling case of the gate projection: --profile-gates launches of
    arl2_gates_apply over a ring of frames' hidden states."""
    from hybrid_softmax_gated_b200 import Arl2Layer
    wq, wk, wv = workloads.phi_weights(w, 0)
    wg, bg = workloads.gate_projection_weights(w, 0)
    lay = Arl2Layer(w.batch, w.heads, w.head_dim, w.tokens, wq.cuda(), wk.cuda(), wv.cuda(),
                    dtype=w.torch_dtype, gate_weights=(wg.cuda(), bg.cuda()), impl=args.layer_impl)
    ring = 8
    xs = [workloads.hidden_states(w, 0, f, device="cuda") for f in range(ring)]
    for i in range(args.profile_gates):
        lay.gates_apply(xs[i % ring])
    torch.cuda.synchronize()
    st = lay.device_status()
    lay.close()
    print(f"gate profile case {w.name}: {args.profile_gates} launches, status {st}")
    return 0 if st == 0 else 1


def profile_case(args, w: workloads.Workload) -> int:
    """A small case for ncu: one clean pass (non-zero state), then
    --profile-passes read-only passes cycling through a ring of input sets
    whose total size exceeds the 126 MB L2."""
    from hybrid_softmax_gated_b200 import Arl2Layer
    wq, wk, wv = workloads.phi_weights(w, 0)
    lay = Arl2Layer(w.batch, w.heads, w.head_dim, w.tokens, wq.cuda(), wk.cuda(), wv.cuda(),
                    dtype=w.torch_dtype, access=args.access)
    per_set = 3 * w.batch * w.tokens * w.heads * w.head_dim * (2 if w.dtype == "bf16" else 4)
    ring = max(2, (160 << 20) // per_set + 1)
    ins = [workloads.pass_inputs(w, 0, 0, i, device="cuda") for i in range(ring)]
    a, b = (t.cuda() for t in workloads.frame_gates(w, 0, 0))
    out = torch.empty_like(ins[0][0])
    lay.forward(*ins[0], a, b, clean_pass=True, out=out)
    for i in range(args.profile_passes):
        # (token-level access reads through the gates on every pass)
        gates = (a, b) if args.access == "token" else ()
        lay.forward(*ins[(i + 1) % ring], *gates, out=out)
    torch.cuda.synchronize()
    st = lay.device_status()
    lay.close()
    print(f"profile case {w.name}: {args.profile_passes} read-only passes, ring of {ring} input sets, "
          f"status {st}")
    return 0 if st == 0 else 1


def teacher_flops(w: workloads.Workload, cached_frames: int) -> float:
    """Algorithmic FLOPs of one teacher-layer pass with `cached_frames`
    frames in the KV cache: 4 L (N L + L) d H per stream."""
    L, d, H, B = w.tokens, w.head_dim, w.heads, w.batch
    return 4.0 * L * (cached_frames + 1) * L * d * H * B


def stack_curve(args, w: workloads.Workload) -> int:
    """Softmax teacher layer (KV cache) against the hybrid layer over one long
    stream: per-frame attention time and memory as the video grows, and the
    30-layer stacks with 0, 50, 75 and 100 % of the layers replaced
    (technical summary section 4 "Efficiency": the speedup and the memory
    saving grow with video length as the KV cache comes to dominate).

    Each layer kind runs the whole stream of `--curve-frames` frames once
    untimed, then once timed with an event pair around every frame (all of
    its passes, the clean pass's cache append or state update included); each
    frame is one CUDA graph.  Inputs cycle through a ring of pass inputs
    larger than L2.  A stack's attention time is the sum over its layers
    (the layers are independent work of identical cost per kind); its memory
    is the sum of the teacher layers' KV caches and the hybrid layers' state
    copies and workspaces.  Real mixed stacks of 30 layers (50 % and 75 %
    hybrid, spread evenly) then run the first --stack-frames frames, every
    layer with its own handle, to check that sum.  Attention only: the pages'
    figures are whole-model.
    """
    from hybrid_softmax_gated_b200 import Arl2Layer, TeacherLayer
    F = args.curve_frames
    B, L, H, d = w.batch, w.tokens, w.heads, w.head_dim
    esz = 2 if w.dtype == "bf16" else 4
    per_set = 3 * B * L * H * d * esz
    ring = max(2, (160 << 20) // per_set + 1)
    ins = [workloads.pass_inputs(w, 0, 0, i, device="cuda") for i in range(ring)]
    a, b = (t.cuda() for t in workloads.frame_gates(w, 0, 0))
    out = torch.empty_like(ins[0][0])
    st = torch.cuda.current_stream()
    cap_stream = torch.cuda.Stream()
    wq, wk, wv = workloads.phi_weights(w, 0)
    hyb = Arl2Layer(B, H, d, L, wq.cuda(), wk.cuda(), wv.cuda(), dtype=w.torch_dtype)
    tea = TeacherLayer(B, H, d, L, F, dtype=w.torch_dtype)

    def frame_call(kind, f):
        for p in range(w.passes):
            q, k, v = ins[(f * w.passes + p) % ring]
            clean = workloads.is_clean(w, p)
            if kind == "teacher":
                tea.forward(q, k, v, clean_pass=clean, out=out)
            else:
                hyb.forward(q, k, v, a, b, clean_pass=clean, out=out)

    def run(kind):
        graphs = []
        for f in range(F):  # the teacher's graphs keep the cache length each frame saw
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                frame_call(kind, f)
            graphs.append(g)
        for g in graphs:  # upload and warm up: the whole stream once, untimed
            g.replay()
        torch.cuda.synchronize()
        if kind == "hybrid":
            hyb.state_reset()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(F + 1)]
        evs[0].record(st)
        for f, g in enumerate(graphs):
            g.replay()
            evs[f + 1].record(st)
        torch.cuda.synchronize()
        ms = [evs[f].elapsed_time(evs[f + 1]) for f in range(F)]
        del graphs
        return ms

    t_tea = run("teacher")
    t_hyb = run("hybrid")
    bad = (tea.device_status(), hyb.device_status())
    if bad != (0, 0):
        raise SystemExit(f"device status {bad}")
    frame_b = B * L * H * d * esz
    hyb_bytes = hyb.device_bytes()
    marks = sorted({m for m in (1, 21, 81, 231, F) if m <= F})
    peaks = load_peaks()
    n_layers = 30
    curve = []
    for m in marks:
        T_t, T_h = sum(t_tea[:m]), sum(t_hyb[:m])
        cache = 2 * m * frame_b
        row = {"frames": m, "video_frames": 4 * (m - 1) + 1,
               "teacher_ms_frame": t_tea[m - 1], "hybrid_ms_frame": t_hyb[m - 1],
               "teacher_ms_video": T_t, "hybrid_ms_video": T_h,
               "teacher_cache_bytes": cache, "hybrid_state_bytes": hyb_bytes,
               "teacher_tflops_last_frame": w.passes * teacher_flops(w, m - 1) / (t_tea[m - 1] * 1e-3) / 1e12}
        stacks = {}
        for r in (0.0, 0.5, 0.75, 1.0):
            n_h = int(round(n_layers * r))
            n_t = n_layers - n_h
            t = n_t * T_t + n_h * T_h
            mem = n_t * cache + n_h * hyb_bytes
            stacks[f"{int(r * 100)}%"] = {"attn_ms_video": t, "attn_bytes": mem}
        base = stacks["0%"]
        for v in stacks.values():
            v["speedup_vs_all_softmax"] = base["attn_ms_video"] / v["attn_ms_video"]
            v["memory_vs_all_softmax"] = v["attn_bytes"] / base["attn_bytes"]
        row["stack30"] = stacks
        curve.append(row)
    # A real mixed stack: 30 layers (each its own handle and weights) run
    # frame by frame, pass by pass, layer by layer over the first
    # --stack-frames frames, against the sum of the single-layer times.
    measured = []
    Fs = min(args.stack_frames, F)
    for r in (0.5, 0.75):
        n_h = int(round(n_layers * r))
        kinds = ["hybrid" if (i * n_h) // n_layers != ((i + 1) * n_h) // n_layers else "teacher"
                 for i in range(n_layers)]
        layers = []
        for i, kind in enumerate(kinds):
            if kind == "teacher":
                layers.append(TeacherLayer(B, H, d, L, Fs, dtype=w.torch_dtype))
            else:
                wq_i, wk_i, wv_i = workloads.phi_weights(w, i)
                layers.append(Arl2Layer(B, H, d, L, wq_i.cuda(), wk_i.cuda(), wv_i.cuda(), dtype=w.torch_dtype))
        outs = [torch.empty_like(out) for _ in range(2)]

        def stack_frame(f):
            for p in range(w.passes):
                clean = workloads.is_clean(w, p)
                for i, lay in enumerate(layers):
                    q, k, v = ins[(f * w.passes * n_layers + p * n_layers + i) % ring]
                    if kinds[i] == "teacher":
                        lay.forward(q, k, v, clean_pass=clean, out=outs[i & 1])
                    else:
                        lay.forward(q, k, v, a, b, clean_pass=clean, out=outs[i & 1])

        graphs = []
        for f in range(Fs):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                stack_frame(f)
            graphs.append(g)
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
        for kind, lay in zip(kinds, layers):
            if kind == "hybrid":
                lay.state_reset()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for g in graphs:
            g.replay()
        e1.record(st)
        torch.cuda.synchronize()
        t_meas = e0.elapsed_time(e1)
        n_t = n_layers - n_h
        t_model = n_t * sum(t_tea[:Fs]) + n_h * sum(t_hyb[:Fs])
        mem = sum(lay.cache_bytes() if kind == "teacher" else lay.device_bytes()
                  for kind, lay in zip(kinds, layers))
        bad = [lay.device_status() for lay in layers]
        del graphs
        for lay in layers:
            lay.close()
        if any(bad):
            raise SystemExit(f"device status {bad}")
        measured.append({"hybrid_share": f"{int(r * 100)}%", "frames": Fs, "layers": n_layers,
                         "hybrid_layers": n_h, "attn_ms_video_measured": t_meas,
                         "attn_ms_video_sum_of_layers": t_model, "attn_bytes": mem})
    last = curve[-1]
    line = {
        "metric": "attention per video: softmax KV-cache teacher vs ARL2 hybrid layer (480p, 30-layer stacks)",
        "unit": "ms", "data": "synthetic", "dtype": w.dtype, "n_gpus": 1,
        "config": {"workload": w.name, "batch": B, "heads": H, "head_dim": d, "tokens_per_frame": L,
                   "passes": w.passes, "frames": F, "layers": n_layers,
                   "l2": f"inputs larger than L2 ({ring} input sets)"},
        "curve": curve,
        "stack_measured": measured,
        "roofline": {"kernel": "attn_tc_kernel (teacher, longest cache)", "bound": "tensor",
                     "achieved": last["teacher_tflops_last_frame"], "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": last["teacher_tflops_last_frame"] / peaks["bf16_tflops_sustained"],
                     "note": "whole frame (4 passes and the append) timed; peak: bf16 sustained "
                             f"({peaks['source']})"},
    }
    tea.close()
    hyb.close()
    print(json.dumps(line))
    return 0


def stack30(args, w: workloads.Workload) -> int:
    """The batched 30-layer stack: w.layers hybrid layers, each with its own
    handle (own phi maps, gates and fp32 states for w.batch streams), run
    frame by frame, pass by pass, layer by layer over w.frames frames; the
    clean pass of every layer updates its states.  One CUDA graph per frame
    (all layers, all passes).  Inputs cycle through a ring of per-(layer,
    pass) input sets larger than L2, and each layer's gates through four
    frames of its own draws.  Prints one JSON line: stream-frames/s through
    the whole stack, the fused kernel's time per launch at this batch (event
    pair around a layer's back-to-back read-only passes), peak device
    memory, and the SM clocks sampled during the timed region."""
    from hybrid_softmax_gated_b200 import Arl2Layer
    B, L, H, d = w.batch, w.tokens, w.heads, w.head_dim
    per_set = 3 * B * L * H * d * 2
    ring = max(4, (400 << 20) // per_set + 1)
    ins = [workloads.pass_inputs(w, i % w.layers, 0, i // w.layers, device="cuda") for i in range(ring)]
    layers, gates = [], []
    for l in range(w.layers):
        wq, wk, wv = workloads.phi_weights(w, l)
        layers.append(Arl2Layer(B, H, d, L, wq.cuda(), wk.cuda(), wv.cuda(), dtype=w.torch_dtype))
        gates.append([tuple(t.cuda() for t in workloads.frame_gates(w, l, f)) for f in range(4)])
    outs = [torch.empty_like(ins[0][0]) for _ in range(2)]
    st = torch.cuda.current_stream()
    cap = torch.cuda.Stream()

    def frame(f):
        for p in range(w.passes):
            clean = workloads.is_clean(w, p)
            for l, lay in enumerate(layers):
                q, k, v = ins[(f * w.passes * w.layers + p * w.layers + l) % ring]
                a, b = gates[l][f % 4]
                lay.forward(q, k, v, a, b, clean_pass=clean, out=outs[l & 1])

    launches0 = sum(lay.kernel_launches() for lay in layers)
    graphs = []
    for f in range(w.frames):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            frame(f)
        graphs.append(g)
    launches_per_run = sum(lay.kernel_launches() for lay in layers) - launches0
    for _ in range(max(1, args.warmup // 3)):  # the whole stream once per warm-up round
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    for lay in layers:
        lay.state_reset()
    clocks = ClockSampler(torch.cuda.current_device())
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    clocks.start()
    e0.record(st)
    for g in graphs:
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    bad = [lay.device_status() for lay in layers]
    if any(bad):
        raise SystemExit(f"device status {bad}")
    del graphs
    # the fused kernel at this batch: layer 0's read-only passes back to back
    n_k = max(1, w.passes - 1) * 8
    kg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(kg, stream=cap):
        for i in range(n_k):
            layers[0].forward(*ins[i % ring], out=outs[0])
    kg.replay()
    torch.cuda.synchronize()
    k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    k0.record(st)
    kg.replay()
    k1.record(st)
    torch.cuda.synchronize()
    k_ms = k0.elapsed_time(k1) / n_k
    del kg
    peaks = load_peaks()
    achieved = attn_flops(w) / (k_ms / 1e3) / 1e12
    value = B * w.frames / (ms / 1e3)
    line = {
        "metric": "hybrid-attn stream-frames/s through a 30-layer stack (12h x 128d, 1560 tok/frame, 4 streams)",
        "value": value, "unit": "frames/s", "n_gpus": 1, "steps": 1, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "batch": B, "heads": H, "head_dim": d,
                   "tokens_per_frame": L, "frames": w.frames, "passes": w.passes,
                   "l2": f"inputs larger than L2 ({ring} input sets of {per_set >> 20} MiB)",
                   "step": "the whole stream: frames x passes x layers, one CUDA graph per frame"},
        "layer_frames_per_s": value * w.layers,
        "tflops_algorithmic": w.layers * B * w.frames * frame_flops(dataclasses_replace(w, batch=1)) / (ms / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "kernel": "attn_tc_kernel", "kernel_ms": k_ms,
                     "flops_per_launch": attn_flops(w), "peak_kind": f"bf16 burst ({peaks['source']})"},
        "clocks": clk,
        "gpu_launches": launches_per_run,
        "peak_device_bytes": torch.cuda.max_memory_allocated() + sum(lay.device_bytes() for lay in layers),
    }
    for lay in layers:
        lay.close()
    print(json.dumps(line), flush=True)
    return 0


def dataclasses_replace(w, **kw):
    import dataclasses
    return dataclasses.replace(w, **kw)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="480p_bf16")
    ap.add_argument("--impl", default="arl2", choices=["arl2", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--gating", default="headwise", choices=["headwise", "elementwise"],
                    help="forget gate per head (the pages' form) or per key feature")
    ap.add_argument("--access", default="frame", choices=["frame", "token"],
                    help="frame-level state access (the method) or token-level (the ablation)")
    ap.add_argument("--gates", default="given", choices=["given", "projected"],
                    help="alpha and beta as inputs, or projected in-kernel from the hidden states")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stack-curve", action="store_true",
                    help="softmax KV-cache teacher vs hybrid layer over one long stream, and the "
                         "30-layer stacks built from them (one JSON line, not the headline)")
    ap.add_argument("--profile-gates", type=int, default=0,
                    help="profiling case of the gate projection: this many launches (no timing)")
    ap.add_argument("--layer-impl", default="auto", choices=["auto", "simt"],
                    help="kernels of the gate profiling case: tensor cores (bf16) or SIMT")
    ap.add_argument("--profile-teacher", type=int, default=0,
                    help="profiling case of the teacher layer with this many cached frames "
                         "(read-only passes as --profile-passes; no timing, no JSON line)")
    ap.add_argument("--stack-frames", type=int, default=21,
                    help="frames of the real mixed 30-layer stacks run by --stack-curve")
    ap.add_argument("--curve-frames", type=int, default=231,
                    help="latent frames of the stack-curve stream (231: 921 video frames)")
    ap.add_argument("--profile-passes", type=int, default=0,
                    help="profiling case: run this many read-only passes over a ring of inputs "
                         "larger than L2 and exit (no timing, no JSON line)")
    args = ap.parse_args()
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if args.profile_teacher > 0:
        return profile_teacher_case(args, w)
    if args.profile_gates > 0:
        return profile_gates_case(args, w)
    if args.profile_passes > 0:
        return profile_case(args, w)
    if args.stack_curve:
        return stack_curve(args, w)
    if w.layers > 1:
        return stack30(args, w)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from hybrid_softmax_gated_b200 import Arl2Layer

    stream_idx = rank  # each rank: its own independent stream (replica)
    wq, wk, wv = workloads.phi_weights(w, 0)
    projected = args.gates == "projected"
    if projected and args.gating != "headwise":
        raise SystemExit("--gates projected makes headwise gates")
    gate_w = None
    if projected:
        wg, bg = workloads.gate_projection_weights(w, 0)
        gate_w = (wg.cuda(), bg.cuda())
    # host_staging=2: the end-to-end calls' copies overlap the neighbouring
    # passes (two staging sets, the handle's own copy streams)
    lay = Arl2Layer(w.batch, w.heads, w.head_dim, w.tokens, wq.cuda(), wk.cuda(), wv.cuda(),
                    dtype=w.torch_dtype, host_staging=2, gating=args.gating, access=args.access,
                    gate_weights=gate_w)
    gate_draw = workloads.frame_gates_elementwise if args.gating == "elementwise" else workloads.frame_gates
    # all inputs of the stream, resident in HBM before timing; with projected
    # gates, the frame's hidden states instead of its alpha and beta
    ins, gates, hidden = [], [], []
    for f in range(w.frames):
        if projected:
            hidden.append(workloads.hidden_states(w, stream_idx, f, device="cuda"))
            gates.append((None, None))
        else:
            a, b = gate_draw(w, stream_idx, f)
            gates.append((a.cuda(), b.cuda()))
        for p in range(w.passes):
            ins.append(workloads.pass_inputs(w, stream_idx, f, p, device="cuda"))
    out = torch.empty_like(ins[0][0])
    st = torch.cuda.current_stream()

    def step(evs=None):
        """One stream: reset, then every pass of every frame.  With evs, an
        event pair brackets each frame's run of read-only passes (each of
        which launches the fused attention kernel alone)."""
        lay.state_reset()
        i = 0
        for f in range(w.frames):
            a, b = gates[f]
            for p in range(w.passes):
                q, k, v = ins[i]
                i += 1
                clean = workloads.is_clean(w, p)
                if evs is not None and p == 0:
                    evs[f][0].record()
                if projected:
                    needs_x = clean or lay.token_level
                    lay.forward_hidden(q, k, v, hidden[f] if needs_x else None, clean_pass=clean, out=out)
                else:
                    lay.forward(q, k, v, a, b, clean_pass=clean, out=out)
                if evs is not None and p == w.passes - 2:
                    evs[f][1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if lay.device_status() != 0:
        raise SystemExit("device status not ok after warm-up")

    # One CUDA graph per timed step, so that the timed region is free of
    # launch overhead and consecutive kernels overlap their set-up
    # (programmatic dependent launch).  The headline graphs hold no events.
    launches0 = lay.kernel_launches()
    cap = torch.cuda.Stream()

    def capture(with_events):
        gs, es = [], []
        for _ in range(args.steps):
            evs = None
            if with_events:
                evs = [(torch.cuda.Event(enable_timing=True, external=True),
                        torch.cuda.Event(enable_timing=True, external=True)) for _ in range(w.frames)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step(evs)
            gs.append(g)
            es.append(evs)
        for g in gs:  # upload each graph once, untimed
            g.replay()
        torch.cuda.synchronize()
        return gs, es

    graphs, _ = capture(False)
    launches_per_step = (lay.kernel_launches() - launches0) // args.steps

    clocks = ClockSampler(local)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    clocks.start()
    start.record(st)
    for g in graphs:
        g.replay()
    stop.record(st)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(ws)
    elapsed_ms = start.elapsed_time(stop)
    status = lay.device_status()
    if status != 0:
        raise SystemExit(f"device status {status}")
    t_max = max_over_ranks(elapsed_ms, ws)
    value = whole_job_rate(args.steps * w.frames * w.batch, ws, t_max)
    del graphs

    # Fused-kernel duration: the same steps again, with an event pair around
    # each frame's back-to-back read-only passes (passes - 1 launches).
    if w.passes < 2:
        raise SystemExit("the kernel timing needs read-only passes")
    kgraphs, kevents = capture(True)
    torch.cuda.synchronize()
    for g in kgraphs:
        g.replay()
    torch.cuda.synchronize()
    kernel_ms = [e0.elapsed_time(e1) / (w.passes - 1) for evs in kevents for e0, e1 in evs]
    del kgraphs
    if lay.device_status() != 0:
        raise SystemExit("device status not ok after the kernel timing")

    gate_kernel = None
    if projected:
        # the gate projection alone: back-to-back launches over the frames'
        # hidden states, one CUDA graph, an event pair around it
        n_g = 4 * w.frames
        lay.gates_apply(hidden[0])
        gg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gg, stream=cap):
            for i in range(n_g):
                lay.gates_apply(hidden[i % w.frames])
        gg.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(st)
        gg.replay()
        g1.record(st)
        torch.cuda.synchronize()
        g_ms = g0.elapsed_time(g1) / n_g
        del gg
        D = workloads.hidden_dim(w)
        g_bytes = w.batch * w.tokens * D * 2 + D * 2 * w.heads * 2 + w.batch * w.heads * (w.tokens + 1) * 4
        g_flops = 2.0 * w.batch * w.tokens * D * 2 * w.heads
        gate_kernel = {"kernel": "gate_proj_kernel", "kernel_ms": g_ms, "bytes_per_launch": g_bytes,
                       "achieved_gbs": g_bytes / (g_ms / 1e3) / 1e9, "hbm_peak_gbs": load_peaks()["hbm_gbs"],
                       "achieved_tflops": g_flops / (g_ms / 1e3) / 1e12,
                       "fp32_fma_peak_tflops": fp32_simt_tflops()}

    # end to end: host (pinned) buffers through arl2_frame_forward_host
    ring = 8
    host_in = [tuple(t.cpu().pin_memory() for t in ins[i]) for i in range(ring)]
    if projected:
        host_gates = [(hidden[f].cpu().pin_memory(),) for f in range(min(ring, w.frames))]
    else:
        host_gates = [tuple(t.cpu().pin_memory() for t in gates[f]) for f in range(min(ring, w.frames))]
    host_out = torch.empty(ins[0][0].shape, dtype=ins[0][0].dtype).pin_memory()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h2d = d2h = 0
    tok_bytes = ins[0][0].numel() * ins[0][0].element_size()
    gate_bytes = (hidden[0].numel() * hidden[0].element_size() if projected
                  else (gates[0][0].numel() + gates[0][1].numel()) * 4)

    def e2e_step():
        lay.state_reset()
        i = 0
        for f in range(w.frames):
            g = host_gates[f % len(host_gates)]
            for p in range(w.passes):
                q, k, v = host_in[i % ring]
                i += 1
                clean = workloads.is_clean(w, p)
                if projected:
                    needs_x = clean or lay.token_level
                    lay.forward_hidden_host(q, k, v, g[0] if needs_x else None, clean, host_out)
                else:
                    lay.forward_host(q, k, v, g[0], g[1], clean, host_out)

    e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    e_start.record(st)
    for _ in range(args.e2e_steps):
        e2e_step()
    e_stop.record(st)
    e_stop.synchronize()
    barrier(ws)
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_stop), ws)
    gate_passes = w.passes if args.access == "token" else 1  # the passes that carry gate inputs
    h2d = w.frames * (w.passes * 3 * tok_bytes + gate_passes * gate_bytes)
    d2h = w.frames * w.passes * tok_bytes
    e2e_value = args.e2e_steps * w.frames * w.batch * ws / (e2e_ms / 1e3)
    # the bound the copies set: a pinned host-to-device copy of the size of a
    # pass's inputs, best of a few, against the step's input bytes
    probe = torch.empty(3 * tok_bytes, dtype=torch.uint8).pin_memory()
    probe_d = torch.empty(probe.shape, dtype=torch.uint8, device="cuda")
    h2d_gbs = 0.0
    for _ in range(5):
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(st)
        for _ in range(8):
            probe_d.copy_(probe, non_blocking=True)
        c1.record(st)
        c1.synchronize()
        h2d_gbs = max(h2d_gbs, 8 * probe.numel() / (c0.elapsed_time(c1) / 1e3) / 1e9)
    del probe, probe_d
    copy_bound = {"h2d_gbs": h2d_gbs,
                  "frames_per_s": w.frames * w.batch * ws / (h2d / (h2d_gbs * 1e9)),
                  "how": "pinned host-to-device copies of one pass's q, k, v bytes, back to back, best of 5"}

    peaks = load_peaks()
    k_ms = float(np.mean(kernel_ms))
    if args.access == "token":
        # the ablation's read-only pass: the fused kernel for the intra-frame
        # term, then the tensor-core chunk preparation and the sequential
        # chunk scan; its algorithmic work is the intra term plus, per token,
        # the three phi maps and the sequential read, residual and update
        # (6 d^2 per head)
        L, d, H, B = w.tokens, w.head_dim, w.heads, w.batch
        flops = (4.0 * L * L * d * H + 6.0 * L * d * d * H + 6.0 * L * d * d * H) * B
        achieved = flops / (k_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "kernel": "token-level pass (attn_tc_kernel, tl_tc_prep_kernel, tl_tc_scan_kernel)",
                    "kernel_ms": k_ms, "flops_per_launch": flops,
                    "peak_kind": f"bf16 burst ({peaks['source']})"}
    else:
        # The kernel is timed in a replay of tens of milliseconds, the regime
        # of the burst GEMM figure; the sustained (seconds-long, power-capped)
        # figure is reported beside it for reference only.
        achieved = attn_flops(w) / (k_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": measured_traffic(w.name), "kernel": "attn_tc_kernel",
                    "kernel_ms": k_ms, "flops_per_launch": attn_flops(w),
                    "peak_kind": f"bf16 burst ({peaks['source']})",
                    "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        spf, threads, desc = oracle_frame_seconds(w)
        cpu = {"value": w.batch / spf, "unit": "frames/s", "cores": threads, "kind": "oracle",
               "sample": desc}

    line = {
        "metric": METRIC,
        "value": value, "unit": "frames/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": arm_config(args, w, ws),
        "tokens_per_s": value * w.tokens,
        "tflops_per_frame_algorithmic": frame_flops(w) / 1e12,
        "roofline": roofline, "clocks": clk,
        "e2e": {"value": e2e_value, "unit": "frames/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "copies": "pinned host buffers, two staging sets: a call's "
                "input copies overlap the previous call's pass and output copy", "copy_bound": copy_bound},
        "gpu_launches": args.steps * launches_per_step * ws,
        "cpu_baseline": cpu,
        "peak_device_bytes": torch.cuda.max_memory_allocated() + lay.device_bytes(),
    }
    if gate_kernel is not None:
        line["gate_kernel"] = gate_kernel
    if rank == 0:
        print(json.dumps(line), flush=True)
    lay.close()
    if ws > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
