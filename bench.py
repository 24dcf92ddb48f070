"""Benchmark: BitNet W1A8 decode GEMV (M=1) on the Llama-7B projection shapes.

One step = one decode token through a 32-layer Llama-7B linear stack at
W1A8: per decoder layer q, k, v, o [4096x4096], gate, up [11008x4096] and
down [4096x11008], each layer call = bq_linear, i.e. the activation quantization
fused into the GEMV kernel (224 calls,
about 820 MB of packed weights, so every step streams inputs larger than L2).
Weights ~ N(0, 0.02^2) and activations ~ N(0, 1) are synthetic (seeded torch
generator on the device; no model or dataset).

Prints one JSON line (rank 0). `value` = algorithmic HBM bytes of all ranks'
steps / max-over-ranks device time, in GB/s; `us_per_layer` is the same run
expressed per layer call. `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/layer & achieved HBM GB/s (% of B200 peak), quantized GEMV/GEMM, M=1..64"
LLAMA7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
           ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
# projections of a decoder layer that read the same input: one grouped launch each
LLAMA7B_CALLS = [("q", "k", "v"), ("o",), ("gate", "up"), ("down",)]
NOMINAL_HBM_GBS = 8000.0


def layer_bytes(fmt: str, N: int, K: int, M: int = 1, w_bits: int = 1, a_bits: int = 8) -> dict:
    """Algorithmic bytes of one layer call: packed weights + per-row/tensor scales,
    x bf16 read by the act kernel, act codes written and read once, y fp32."""
    if fmt in ("rabit", "rabit3"):
        # P sign planes + g_p + h_p; act: x bf16 in, h_p x f32 out and back in; y f32
        P = 2 if fmt == "rabit" else 3
        w = P * N * K // 8 + 4 * P * N + 4 * P * K
        return dict(gemv=w + 4 * P * M * K + 4 * M * N, act=2 * M * K + 4 * P * M * K + 4 * P * K,
                    total=w + 2 * M * K + 8 * P * M * K + 4 * P * K + 4 * M * N, fused=w + 2 * M * K + 4 * M * N)
    bits = {"bitnet": 1, "ternary": 2, "abq": w_bits, "bvsr": 4}[fmt]
    w = N * K * bits // 8
    extra = {"bitnet": 4, "ternary": 4, "abq": 12 * N, "bvsr": N * K // 32 + 256 * 32}[fmt]
    x = 2 * M * K
    act = M * K
    y = 4 * M * N
    lora_g = lora_a = 0
    if fmt == "ternary":   # rank-32 bf16 A read by the act kernel, B^T by the GEMV, u f32 between them
        lora_a, lora_g = 32 * K * 2 + 32 * 4 * M, 32 * N * 2 + 32 * 4 * M
    gemv = w + extra + act + y + 16 * M + lora_g
    actb = x + act + 16 * M + lora_a
    # bq_linear: the codes never leave shared memory; x is read by the layer kernel (and by
    # the LoRA partial kernel for ternary)
    fused = w + extra + x + y + lora_g + (lora_a + x if fmt == "ternary" else 0)
    return dict(gemv=gemv, act=actb, total=gemv + actb, fused=fused)


def call_bytes(Ns, K: int) -> int:
    """Algorithmic bytes of one fused BitNet call (bq_linear, or bq_linear_group over several
    layers) at M = 1: each layer's weights, scale and y, and the shared input x read once."""
    return sum(layer_bytes("bitnet", N, K)["fused"] for N in Ns) - (len(Ns) - 1) * 2 * K


def reduce_max_over_ranks(values, dist=None, device=None) -> list:
    """Each value's maximum over the ranks (a job's device time is its slowest rank's). With no
    initialized process group, or one rank, the values come back unchanged."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_value(bytes_per_step: float, steps: int, ms_max: float, world: int) -> float:
    """Whole-job GB/s of `world` replicas, each streaming bytes_per_step for `steps` steps,
    timed by the slowest rank (ms_max)."""
    return world * bytes_per_step * steps / (ms_max * 1e-3) / 1e9


def clock_record(clk: dict) -> dict:
    """The bench line's clocks: the SM clock median and reasons of the timed window when it
    holds samples, else of the soak and timed windows together (the whole sampled run)."""
    t = clk.get("timed") or {}
    s = clk.get("soak") or {}
    src = t if t.get("samples") else clk
    out = {"sm_mhz": src.get("sm_mhz"), "sm_max_mhz": clk.get("sm_max_mhz"),
           "reasons": sorted(set(clk.get("reasons", [])) | set(t.get("reasons", [])) | set(s.get("reasons", []))),
           "samples": clk.get("samples", 0), "timed_samples": t.get("samples", 0), "soak_samples": s.get("samples", 0),
           "soak_sm_mhz": s.get("sm_mhz"), "timed_sm_mhz": t.get("sm_mhz"), "power_w_max": clk.get("power_w_max"),
           "window": "timed regions" if t.get("samples") else "soak + timed"}
    return out


def measured_peaks() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash() -> str:
    """Hash of what sets the layer kernel's DRAM traffic: its code (bq_gemv.cuh,
    bq_internal.cuh) and its launch plan (plan_layer in bq_abi.cuh)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "bit_weight_quantization_b200", "csrc")
    for fn in ("bq_gemv.cuh", "bq_internal.cuh"):
        with open(os.path.join(d, fn), "rb") as f:
            h.update(f.read())
    with open(os.path.join(d, "bq_abi.cuh")) as f:
        src = f.read()
    i0 = src.index("inline bool plan_layer(")
    h.update(src[i0:src.index("\n}\n", i0)].encode())
    return h.hexdigest()[:16]


def profile_traffic(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampled every `period_ms` in a background reader; each line is stamped with
    the host time it arrived, so samples can be assigned to the soak and timed windows."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 100):
        import threading
        self.proc, self.lines, self.windows = None, [], {}
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", str(period_ms), "-i", str(index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line))

    def wait_first(self, timeout: float = 5.0) -> bool:
        """Block until the first sample has arrived (or `timeout` s)."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.01)
        return bool(self.lines)

    def window(self, name: str, t0: float, t1: float):
        self.windows[name] = (t0, t1)

    def stats(self, t0: float, t1: float) -> dict:
        """The samples that arrived in [t0, t1 + 0.15 s] so far, parsed."""
        return self.parse("".join(l for t, l in list(self.lines) if t0 <= t <= t1 + 0.15))

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)   # one more period after the last window
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        out = self.parse("".join(l for _, l in self.lines))
        for name, (t0, t1) in self.windows.items():
            sel = "".join(l for t, l in self.lines if t0 <= t <= t1 + 0.15)
            out[name] = self.parse(sel)
        return out

    @staticmethod
    def parse(out: str) -> dict:
        """Median SM clock, max clock and the throttle reasons seen, from `nvidia-smi
        --query-gpu=FIELDS --format=csv,noheader,nounits` lines."""
        sm, mx, reasons, pw = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx.append(float(f[2])); pw.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() in ("active", "1"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(pw)}


# ---------------------------------------------------------------------------
# CPU oracle arm / baseline
# ---------------------------------------------------------------------------
def cpu_model() -> str:
    """The host CPU's model name (first processor in /proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def oracle_sample(seconds: float, seed: int = 0, min_calls: int = 2, threads: int = 0) -> dict:
    """Time the C++ oracle (act quantization + reference layer, oracle/bq_ref.cpp) on
    q-projection sized BitNet W1A8 layer calls (4096x4096, M=1) for about `seconds`, on
    `threads` OpenMP threads (0: all host cores). Returns the sample's GB/s over all calls and the
    best single call (time.perf_counter around each call)."""
    import bq_inputs as I
    from oracle import cref as O
    O.set_threads(threads if threads > 0 else (os.cpu_count() or 1))
    W = I.weights(4096, 4096, seed)
    x = I.activations(1, 4096, seed)
    p = O.bitnet_pack(W)
    calls, times, t0 = 0, [], time.perf_counter()
    while True:
        c0 = time.perf_counter()
        O.bitnet_layer(p, x)
        times.append(time.perf_counter() - c0)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds and calls >= min_calls:
            break
    b = layer_bytes("bitnet", 4096, 4096)["fused"]
    return dict(seconds=el, calls=calls, gbs=calls * b / el / 1e9, us_per_layer=el / calls * 1e6,
                best_us=min(times) * 1e6, best3_us=sorted(times)[min(2, len(times) - 1)] * 1e6,
                cores=O.threads(), cpu=cpu_model(), nproc=os.cpu_count())


def cpu_baseline_record(all_cores: dict, one_core: dict) -> dict:
    """The bench line's cpu_baseline: the oracle on all host cores (the value) and on one core."""
    return {"value": all_cores["gbs"], "unit": "GB/s", "cores": all_cores["cores"], "kind": "oracle (C++)",
            "cpu": all_cores["cpu"], "nproc": all_cores["nproc"],
            "sample": f"{all_cores['calls']} BitNet W1A8 4096x4096 layer calls (act quant + layer) of the C++ "
                      f"oracle in {all_cores['seconds']:.1f} s; best call {all_cores['best_us']:.0f} us",
            "one_core": {"value": one_core["gbs"], "unit": "GB/s", "cores": one_core["cores"],
                         "calls": one_core["calls"], "seconds": one_core["seconds"],
                         "best_us": one_core["best_us"]}}


def workload_name(layers: int, no_group: bool) -> str:
    """The bench workload's name, shared by the CUDA arm and the reference arm."""
    return (f"BitNet W1A8 decode GEMV, M=1: {layers}-layer Llama-7B linear stack "
            "(q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008), "
            + ("q,k,v and gate,up each one bq_linear_group call on their shared input, "
               "o and down one bq_linear call each" if not no_group else "one bq_linear call per projection")
            + " (act quantization fused into the layer kernel), PDL between launches, CUDA graph per step")


def run_reference(args) -> None:
    """The reference arm: the C++ oracle on the host cores, one BitNet W1A8 4096x4096 layer call
    (act quantization + layer) per step, on all cores; a one-core sample beside it."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(0.0, min_calls=1)
    res = [oracle_sample(0.0, min_calls=1) for _ in range(args.steps)]
    el = sum(r["seconds"] for r in res)
    calls = sum(r["calls"] for r in res)
    b = layer_bytes("bitnet", 4096, 4096)["fused"]
    val = calls * b / el / 1e9
    one = oracle_sample(min(args.cpu_seconds, 3.0), min_calls=2, threads=1)
    cores = res[0]["cores"]
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64+f64",
        "data": "synthetic",
        "config": {"workload": workload_name(args.layers, args.no_group), "seq_len": 1, "global_batch": 1,
                   "parallelism": "single",
                   "sample": "each step one bounded sample of the workload: a BitNet W1A8 4096x4096 layer "
                             "call (act quantization + layer) of the C++ oracle; GB/s over its algorithmic bytes"},
        "us_per_layer": el / calls * 1e6,
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": cores, "kind": "oracle (C++)", "cpu": res[0]["cpu"],
                         "nproc": res[0]["nproc"],
                         "sample": f"{calls} BitNet W1A8 4096x4096 layer calls (act quant + layer) of the C++ oracle",
                         "one_core": {"value": one["gbs"], "unit": "GB/s", "cores": one["cores"],
                                      "calls": one["calls"], "best_us": one["best_us"]}},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# CUDA arm
# ---------------------------------------------------------------------------
def build_stack(layers: int, seed: int, device, group: bool = True):
    """The decode step's layer calls: per decoder layer q,k,v in one grouped call on a shared
    input, o, gate+up grouped on a shared input, down (or, ungrouped, one call per
    projection, each with its own input)."""
    import torch
    from bit_weight_quantization_b200 import bq
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    shapes = {n: (N, K) for n, N, K in LLAMA7B}
    calls = []
    for l in range(layers):
        members = {}
        for name, N, K in LLAMA7B:
            W = torch.randn(N, K, device=device, generator=gen, dtype=torch.float32) * 0.02
            ql = bq.QuantLinear("bitnet", W)
            del W
            members[name] = dict(name=name, N=N, K=K, ql=ql, y=torch.empty(1, N, device=device, dtype=torch.float32))
        groups = LLAMA7B_CALLS if group else [(n,) for n, _, _ in LLAMA7B]
        for names in groups:
            K = shapes[names[0]][1]
            x = torch.randn(1, K, device=device, generator=gen).to(torch.bfloat16)
            ms = [members[n] for n in names]
            calls.append(dict(members=ms, x=x, K=K, bytes=call_bytes([m["N"] for m in ms], K)))
    torch.cuda.synchronize()
    return calls


def one_call(c, x=None, ys=None):
    from bit_weight_quantization_b200 import bq
    x = c["x"] if x is None else x
    ys = [m["y"] for m in c["members"]] if ys is None else ys
    if len(c["members"]) == 1:
        bq.bq_linear(c["members"][0]["ql"].layer, x, 1, ys[0])
    else:
        bq.bq_linear_group([m["ql"].layer for m in c["members"]], x, 1, ys)


def step_calls(calls, timing=None):
    """One decode step: every layer call (activation quantization fused into the layer)."""
    for i, c in enumerate(calls):
        if timing is not None:
            timing[i][0].record()
        one_call(c)
        if timing is not None:
            timing[i][1].record()


def run_cuda(args) -> None:
    import torch
    import torch.distributed as dist
    from bit_weight_quantization_b200 import bq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    stack = build_stack(args.layers, args.seed + rank, dev, group=not args.no_group)
    per_step = sum(c["bytes"] for c in stack)
    n_calls = len(stack)                               # launches per step
    n_layers = sum(len(c["members"]) for c in stack)   # projections per step
    stream = torch.cuda.Stream(device=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    with torch.cuda.stream(stream):
        step_calls(stack)                      # eager warm-up, also loads the module
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step_calls(stack)
        torch.cuda.synchronize()
        bq.bq_device_check()

        # clocks: the sampler runs from before the soak to after the last timed region
        clocks = ClockSampler(local)
        clocks.wait_first()
        # soak: the same step replayed for about --soak-seconds (untimed) so that the clocks
        # sampled are those of this workload under load
        ts0 = time.time()
        n_soak = 0
        while time.time() - ts0 < args.soak_seconds or n_soak == 0:
            for _ in range(8):
                g.replay()
            torch.cuda.synchronize()
            n_soak += 8
        ts1 = time.time()
        host_ms_step = (ts1 - ts0) * 1e3 / n_soak
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        # timed: R back-to-back regions of exactly K steps each, every region bracketed by a
        # barrier and a synchronize, so that together they last about --timed-seconds
        R = int(reduce_max_over_ranks([max(1, min(200, -(-args.timed_seconds * 1e3 // (host_ms_step * args.steps))))],
                                      dist if world > 1 else None, dev)[0])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        region_ms = []
        tt0 = time.time()
        for _ in range(R):
            barrier()
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            region_ms.append(e0.elapsed_time(e1))
        tt1 = time.time()
        clocks.window("soak", ts0, ts1)
        clocks.window("timed", tt0, tt1)
        clk = clocks.stop()
        region_ms = reduce_max_over_ranks(region_ms, dist if world > 1 else None, dev)
        ms = statistics.median(region_ms)

        # serialized per-launch time (context only): a second capture of the same step with
        # events around every bq_linear; the events between launches remove the PDL overlap
        timing = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True)) for _ in stack]
        gi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gi, stream=stream):
            step_calls(stack, timing)
        torch.cuda.synchronize()
        gemv_ms = []
        for _ in range(max(3, min(args.steps, 50))):
            gi.replay()
            torch.cuda.synchronize()
            gemv_ms.append(sum(a.elapsed_time(b) for a, b in timing))
        gemv_ms_step = statistics.median(gemv_ms)

        # end to end through the public API: pinned host x -> device, every call, y -> host
        xs_h = torch.cat([c["x"].view(-1) for c in stack]).cpu().pin_memory()
        xs_d = torch.empty_like(xs_h, device=dev)
        ys_h = torch.empty(sum(m["N"] for c in stack for m in c["members"]), dtype=torch.float32).pin_memory()
        ys_d = torch.empty(ys_h.numel(), dtype=torch.float32, device=dev)
        views, xo, yo = [], 0, 0
        for c in stack:
            yv, y0 = [], yo
            for m in c["members"]:
                yv.append(ys_d[yo:yo + m["N"]].view(1, -1))
                yo += m["N"]
            # the call's outputs are contiguous: one readback each, device slice -> pinned host slice
            views.append((xs_d[xo:xo + c["K"]].view(1, -1), yv, ys_d[y0:yo], ys_h[y0:yo]))
            xo += c["K"]

        # the step's calls captured once through the public helper (bq.StepGraph). Each call's
        # outputs go back to pinned host memory on a copy stream as soon as that call is done,
        # overlapping the later calls; the copy stream joins before the step ends. Every step then
        # copies the inputs in and replays.
        copy_stream = torch.cuda.Stream(device=dev)

        def issue_step():
            for c, (x, yv, yd, yh) in zip(stack, views):
                one_call(c, x, yv)
                done = torch.cuda.Event()
                done.record()
                copy_stream.wait_event(done)
                with torch.cuda.stream(copy_stream):
                    yh.copy_(yd, non_blocking=True)
            torch.cuda.current_stream().wait_stream(copy_stream)

        step_graph = bq.StepGraph(issue_step, stream=stream)

        def e2e_step():
            xs_d.copy_(xs_h, non_blocking=True)
            step_graph.replay()

        for _ in range(max(1, min(args.warmup, 3))):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        n_e2e = max(1, min(args.steps, 50))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        t1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = t0.elapsed_time(t1) / n_e2e
        bq.bq_device_check()

    e2e_ms = reduce_max_over_ranks([e2e_ms], dist if world > 1 else None, dev)[0]
    ms_step = ms / args.steps
    value = job_value(per_step, args.steps, ms, world)
    peak, peak_kind = measured_peaks()
    # every launch in the timed region is the dominant kernel (k_layer<BitNet, fused>): its
    # average launch duration is the timed region over the launches in it
    us_launch = ms_step * 1e3 / n_calls
    achieved = per_step / (ms_step * 1e-3) / 1e9
    traffic = profile_traffic("bitnet_fused_llama7b_mix" if args.no_group else "bitnet_fused_llama7b_grouped")
    out = None
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": workload_name(args.layers, args.no_group),
                       "layers_per_step": n_layers, "launches_per_step": n_calls, "seq_len": 1,
                       "timing": "median of %d back-to-back timed regions of %d steps each (CUDA events; "
                                 "region ms min %.3f, median %.3f, max %.3f); %.1f s untimed soak before the "
                                 "warm-up" % (len(region_ms), args.steps, min(region_ms), ms, max(region_ms),
                                              args.soak_seconds),
                       "global_batch": world,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (each step streams %.0f MB of distinct packed weights)"
                             % (per_step / 1e6)},
            "us_per_layer": ms_step * 1e3 / n_layers,
            "frac_of_peak": value / world / peak, "frac_of_nominal_8tbs": value / world / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                         "kernel": "k_layer<BitNet W1A8, fused>: all %d launches of a step" % n_calls,
                         "bytes_per_launch": per_step / n_calls, "us_per_launch": us_launch,
                         "serialized_us_per_launch": gemv_ms_step * 1e3 / n_calls},
            "e2e": {"value": job_value(per_step, 1, e2e_ms, world), "unit": "GB/s",
                    "h2d_bytes_per_step": int(xs_h.numel() * 2), "d2h_bytes_per_step": int(ys_h.numel() * 4),
                    "ms_per_step": e2e_ms,
                    "path": "public API: the step's C-ABI calls captured once with bq.StepGraph and replayed; "
                            "every step one copy of all inputs from pinned host memory before the replay, and "
                            "each call's results read back to pinned host memory on a copy stream as soon as "
                            "that call is done (inside the graph, overlapping the later calls); timed with "
                            "CUDA events around copy + replay, the readbacks joined before the end"},
            "gpu_launches": n_calls * args.steps,
            "clocks": clock_record(clk),
        }
    if world > 1:
        del g, gi, step_graph
        dist.destroy_process_group()
    if rank == 0:
        if world == 1:
            out["cpu_baseline"] = cpu_baseline_record(oracle_sample(args.cpu_seconds),
                                                      oracle_sample(args.cpu_seconds / 2, threads=1))
        print(json.dumps(out), flush=True)


# ---------------------------------------------------------------------------
# per-config measurement (every format / shape / M) and a single-layer mode
# ---------------------------------------------------------------------------
def make_layer(fmt, N, K, M, w_bits, a_bits, gen, device):
    import torch
    from bit_weight_quantization_b200 import bq
    W = torch.randn(N, K, device=device, generator=gen) * 0.02
    kw = {}
    if fmt in ("rabit", "rabit3"):
        kw["h2"] = torch.rand(K, device=device, generator=gen) + 0.5
    if fmt == "rabit3":
        kw["h3"] = torch.rand(K, device=device, generator=gen) + 0.5
    if fmt == "ternary":
        kw.update(lora_rank=32, lora_alpha=0.1,
                  lora_A=torch.randn(K, 32, device=device, generator=gen) * 0.02,
                  lora_B=torch.randn(32, N, device=device, generator=gen) * 0.01)
    if fmt == "abq":
        kw.update(w_bits=w_bits, a_bits=a_bits)
        flat = W.view(-1)
        idx = torch.randperm(flat.numel(), device=device, generator=gen)[: flat.numel() // 1000]
        flat[idx] *= 20.0
    ql = bq.QuantLinear(fmt, W, **kw)
    x = torch.randn(M, K, device=device, generator=gen)
    if fmt == "abq":
        ch = torch.randperm(K, device=device, generator=gen)[: K // 100]
        x[:, ch] *= 10.0
    x = x.to(torch.bfloat16)
    y = torch.empty(M, N, device=device)
    return dict(ql=ql, x=x, y=y, act=ql.act_buffer(M), ws=ql.workspace(M), M=M, keep=kw)


def layer_call(L, timing=None, fused=True):
    from bit_weight_quantization_b200 import bq
    ql, M = L["ql"], L["M"]
    if timing is not None:
        timing[0].record()
    if fused:
        bq.bq_linear(ql.layer, L["x"], M, L["y"], None, L["ws"], L["ws"].numel())
    else:
        bq.bq_quantize_act(ql.layer, L["x"], M, L["act"], L["act"].numel())
        if M == 1:
            bq.bq_gemv(ql.layer, L["act"], L["y"])
        else:
            bq.bq_gemm(ql.layer, L["act"], M, L["y"])
    if timing is not None:
        timing[1].record()


def config_list():
    out = [("rabit", 256, 512, 1, 0, 0), ("rabit3", 256, 512, 1, 0, 0)]
    out += [("bitnet", N, K, 1, 1, 8) for N, K in [(4096, 4096), (11008, 4096), (4096, 11008)]]
    out += [("ternary", 2048, 2048, M, 2, 8) for M in (1, 4, 16)]
    out += [("abq", N, 4096, M, w, a) for (w, a) in [(2, 8), (4, 4), (6, 6), (8, 8)]
            for N in (4096, 11008) for M in (1, 8, 64)]
    out += [("bvsr", N, K, 1, 4, 8) for N, K in [(5120, 5120), (13824, 5120), (5120, 13824)]]
    out += [("bvsr", 5120, 5120, M, 4, 8) for M in (4, 16, 64)]  # the multi-token path
    return out


def run_configs(args) -> None:
    """For each configuration: a CUDA graph over R distinct packed copies of the
    layer (R copies total >= 3x L2, capped at 512) of act + gemv; reports the
    per-layer-call time, the GEMV launch time, the algorithmic GB/s, and one cold single call
    (no graph, L2 flushed just before; the median of three)."""
    import torch
    from bit_weight_quantization_b200 import bq
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed)
    peak, peak_kind = measured_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)   # twice the L2 size
    # clocks: one sampler for the whole run; every config's timed replays last >= 0.3 s so that
    # its window holds samples (100 ms period)
    clocks = ClockSampler(0)
    clocks.wait_first()
    sel = config_list()
    if args.only:
        sel = [c for c in sel if c[0] == args.only]
    for fmt, N, K, M, w, a in sel:
        lb = layer_bytes(fmt, N, K, M, w, a)
        R = int(min(512, max(2, -(-3 * l2 // lb["total"]))))
        with torch.cuda.stream(stream):
            Ls = [make_layer(fmt, N, K, M, w, a, gen, dev) for _ in range(R)]
            fused = not args.unfused
            for L in Ls:
                layer_call(L, fused=fused)
            torch.cuda.synchronize()
            bq.bq_device_check()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for L in Ls:
                    layer_call(L, fused=fused)
            tim = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True)) for _ in Ls]
            gi = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gi, stream=stream):
                for L, t in zip(Ls, tim):
                    layer_call(L, t, fused=fused)
            th0 = time.time()
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            per_replay = (time.time() - th0) / 3
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = max(3, int(2000 / R), int(0.3 / max(per_replay, 1e-6)) + 1)
            tw0 = time.time()
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            tw1 = time.time()
            us_layer = e0.elapsed_time(e1) * 1e3 / (reps * R)
            time.sleep(0.15)
            clk = clocks.stats(tw0, tw1)
            gl = []
            for _ in range(5):
                gi.replay()
                torch.cuda.synchronize()
                gl.append(statistics.mean(a_.elapsed_time(b_) for a_, b_ in tim) * 1e3)
            us_gemv = statistics.median(gl)
            # one cold call: outside any graph, right after writing a buffer twice the L2 size
            cold = []
            for L in Ls[:3]:
                flush.zero_()
                c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                c0.record(stream)
                layer_call(L, fused=fused)
                c1.record(stream)
                torch.cuda.synchronize()
                cold.append(c0.elapsed_time(c1) * 1e3)
            us_cold = statistics.median(cold)
        nb = lb["fused"] if fused else lb["total"]
        line = dict(fmt=fmt, N=N, K=K, M=M, w_bits=w, a_bits=a, path="bq_linear" if fused else "act+gemm",
                    copies=R, us_per_layer=us_layer,
                    gbs=nb / (us_layer * 1e-6) / 1e9, frac_of_peak=nb / (us_layer * 1e-6) / 1e9 / peak,
                    us_gemv=us_gemv, gemv_gbs=lb["gemv"] / (us_gemv * 1e-6) / 1e9,
                    gemv_frac=lb["gemv"] / (us_gemv * 1e-6) / 1e9 / peak, us_cold_single=us_cold,
                    bytes=nb, peak=peak,
                    peak_source=peak_kind, timed_replays=reps, timed_s=round(tw1 - tw0, 3),
                    clocks={"sm_mhz": clk.get("sm_mhz"), "sm_max_mhz": clk.get("sm_max_mhz"),
                            "reasons": clk.get("reasons", []), "samples": clk.get("samples", 0),
                            "power_w_max": clk.get("power_w_max")})
        print(json.dumps(line), flush=True)
        del Ls, g, gi
        torch.cuda.empty_cache()
    clocks.stop()


def run_layer(args) -> None:
    """One layer, a few calls (the target of ncu captures): bq_linear (fused) by default,
    bq_quantize_act + bq_gemv/bq_gemm with --unfused."""
    import torch
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed)
    N, K = (int(v) for v in args.shape.split("x"))
    L = make_layer(args.fmt, N, K, args.M, args.w_bits, args.a_bits, gen, dev)
    for _ in range(args.iters):
        layer_call(L, fused=not args.unfused)
    torch.cuda.synchronize()
    from bit_weight_quantization_b200 import bq
    bq.bq_device_check()
    print(json.dumps(dict(mode="layer", fmt=args.fmt, N=N, K=K, M=args.M, iters=args.iters, ok=True)))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--soak-seconds", type=float, default=1.5,
                    help="untimed replays before the warm-up, while the clocks are sampled")
    ap.add_argument("--timed-seconds", type=float, default=1.0,
                    help="the timed regions (K steps each) repeat until they last about this long")
    ap.add_argument("--mode", default="bench", choices=["bench", "configs", "layer"])
    ap.add_argument("--only", default="")
    ap.add_argument("--fmt", default="bitnet")
    ap.add_argument("--shape", default="11008x4096")
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--w-bits", type=int, default=1)
    ap.add_argument("--a-bits", type=int, default=8)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--unfused", action="store_true", help="bq_quantize_act + bq_gemv/gemm instead of bq_linear")
    ap.add_argument("--no-group", action="store_true", help="bench: one launch per projection (no bq_linear_group)")
    args = ap.parse_args()
    if args.mode == "configs":
        run_configs(args)
    elif args.mode == "layer":
        run_layer(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
