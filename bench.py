#!/usr/bin/env python
"""Benchmark of the fused encoder layer: forward + backward tokens/s.

Workload: the BERT-Large layer of the "DeepSpeed Transformer Kernel usage
guide" (Step 1: hidden 1024, 16 heads, sequence 128, batch 64), fp16 storage,
attention and hidden dropout 0.1, pre-LN, no padding; synthetic seeded inputs
(weights N(0, 0.02), x and dY N(0, 1)).  One step = layer_forward +
layer_backward of one layer over one batch, inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 it runs under torchrun, one rank per GPU, each rank a data-parallel
replica on its own batch (weak scaling) whose step ends with one NCCL
all-reduce of the float32 gradients; the time is the max over ranks.
Rank 0 prints one JSON line.  `--impl reference` times the float64 oracle
(the reference arm) on the host cores instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from transformer_layer_pre_b200.synthetic import WORKLOADS, make_inputs  # noqa: E402

METRIC = "fwd+bwd tokens/s per BERT-Large layer (B64,S128,fp16); % of tensor peak"
WORKLOAD = "bert-large-f16"
L2_FLUSH_BYTES = 256 << 20   # > 126 MB of L2

# ---------------------------------------------------------------- algorithmic work
def linear_flops_per_token(h: int, f: int) -> float:
    """Forward + backward FLOPs of the four Linear layers per token: forward
    2*(4H^2 + 2HF) (QKV 3H^2, out-proj H^2, FFN 2HF), backward twice that."""
    return 3.0 * 2.0 * (4 * h * h + 2 * h * f)


def attn_flops_per_token(s: int, h: int) -> float:
    """Forward + backward attention FLOPs per token: forward Q K^T and P V are
    2*S*d each per head (4*S*H per token), backward four such products."""
    return 3.0 * 4.0 * s * h


def class_work(cls: str, w, tokens: int, elem: int) -> tuple[float, str]:
    """(algorithmic work per step, unit) of a kernel class of the step."""
    h, f, s = w.hidden, w.ffn, w.seq
    th = tokens * h * elem
    if cls == "gemm":
        return linear_flops_per_token(h, f) * tokens, "flop"
    if cls == "attn_fwd":
        return 4.0 * s * h * tokens, "flop"
    if cls == "attn_bwd":
        return 8.0 * s * h * tokens, "flop"
    if cls == "ln_fwd":      # two LayerNorms: read x, write y
        return 2 * (2 * th), "byte"
    if cls == "ln_bwd":      # two LayerNorm backwards: read dy, x, residual grad; write dx (+ dropout copy once)
        return 2 * (4 * th) + th, "byte"
    # dropout backward of dY (read, write) + bias-gradient column sums of dU and dQKV
    return 2 * th + tokens * f * elem + 3 * th, "byte"


GEMM_PROFILE = os.path.join(ROOT, "profiles", "gemm_tc_pair_bert-large-f16.txt")
GEMM_SOURCES = ("gemm_tc.cu", "epilogue.cuh", "sm100.cuh", "common.cuh", "kernels.h", "dispatch.cu", "layer.cu")


def gemm_sources_digest() -> str:
    h = hashlib.sha256()
    for n in GEMM_SOURCES:
        with open(os.path.join(ROOT, "transformer_layer_pre_b200", "csrc", n), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_gemm_traffic(workload: str) -> float | None:
    """DRAM bytes (read + write) per GEMM launch from the committed ncu summary
    of this workload, or None when there is none or the GEMM kernel sources
    (or the layer code that decides which GEMM launches a step makes) have
    changed since it was captured."""
    if workload != WORKLOAD or not os.path.exists(GEMM_PROFILE):
        return None
    with open(GEMM_PROFILE) as fh:
        text = fh.read()
    t = re.search(r"^TRAFFIC_BYTES_PER_LAUNCH (\d+)", text, re.M)
    d = re.search(r"^KERNEL_SOURCES_SHA256 ([0-9a-f]{64})", text, re.M)
    if not (t and d) or d.group(1) != gemm_sources_digest():
        return None
    return float(t.group(1))


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm_gbs": d["hbm_gbs"], "tflops": d["bf16_tflops"], "tflops_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "tflops": 1590.0, "tflops_sustained": 1400.0, "source": "fallback"}


def full_clock(clocks: dict | None) -> bool:
    """Whether the timed region ran at full SM clock: no power or thermal cap
    among the sampled reasons and a median within 3 % of the maximum."""
    if not clocks or not clocks.get("sm_mhz") or not clocks.get("sm_max_mhz"):
        return True
    capped = any(r in ("sw_power_cap", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                       "hw_power_brake_slowdown")
                 for r in clocks.get("reasons", []))
    return not capped and clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"]


def alu_peak_tflops(sm_mhz: float, sms: int = 148) -> float:
    """float32 FMA peak: 128 FP32 lanes per SM x 2 FLOP x SM clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


# ---------------------------------------------------------------- distributed helpers
def dist_env() -> tuple[int, int, int]:
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def reduce_max(value: float) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the GPU's SM clock and clock-event (throttle) reasons through
    NVML (read-only queries; no setting is touched): on a background thread
    every 0.2 ms, and from the main thread through `sample()` while it waits
    for the timed steps to finish.  Samples taken while `timed` is set form
    the timed-region summary."""

    # every clock-event reason NVML reports (read-only), under nvidia-smi's names
    REASONS = (("nvmlClocksEventReasonGpuIdle", "gpu_idle"),
               ("nvmlClocksEventReasonApplicationsClocksSetting", "applications_clocks_setting"),
               ("nvmlClocksEventReasonSwPowerCap", "sw_power_cap"),
               ("nvmlClocksEventReasonHwSlowdown", "hw_slowdown"),
               ("nvmlClocksEventReasonSyncBoost", "sync_boost"),
               ("nvmlClocksEventReasonSwThermalSlowdown", "sw_thermal_slowdown"),
               ("nvmlClocksEventReasonHwThermalSlowdown", "hw_thermal_slowdown"),
               ("nvmlClocksEventReasonHwPowerBrakeSlowdown", "hw_power_brake_slowdown"),
               ("nvmlClocksEventReasonDisplayClockSetting", "display_clock_setting"))

    def __init__(self, index: int, period_s: float = 0.0002):
        self.index, self.period = index, period_s
        self.timed = False
        self.rows: list = []
        self.smax = None
        self._stop = None
        self._thread = None
        self._query = None

    def _handle(self, pynvml):
        """The NVML handle of CUDA device `index`, matched by PCI address
        (NVML numbers every GPU of the machine, CUDA only the visible ones)."""
        try:
            p = torch.cuda.get_device_properties(self.index)
            return pynvml.nvmlDeviceGetHandleByPciBusId(
                f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0".encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._handle(pynvml)
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:   # no NVML: no clock record
            return self
        masks = [(getattr(pynvml, n), name) for n, name in self.REASONS if hasattr(pynvml, n)]
        self._stop = threading.Event()

        def query():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((float(sm), [name for m, name in masks if r & m]))
            except Exception:
                pass
        self._query = query

        def loop():
            while not self._stop.wait(self.period):
                if self.timed:
                    query()

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def sample(self) -> None:
        """One sample now (from the calling thread), if inside the timed region."""
        if self.timed and self._query is not None:
            self._query()

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self) -> dict | None:
        if not self.rows:
            return None
        reasons = sorted({n for _, rs in self.rows for n in rs})
        return {"sm_mhz": statistics.median(sm for sm, _ in self.rows), "sm_max_mhz": self.smax,
                "reasons": reasons, "samples": len(self.rows),
                "source": "NVML queries 0.2 ms apart over the timed regions (a sampling thread, and the "
                          "main thread while it waits for the last timed step)"}


# ---------------------------------------------------------------- oracle (reference arm / CPU baseline)
def oracle_step(w, inp, nseq: int) -> float:
    """Runs the float64 oracle forward + backward on the first nseq sequences
    of the workload; returns seconds."""
    import oracle
    from transformer_layer_pre_b200.synthetic import to_f64
    cfg = oracle.LayerConfig(batch=nseq, seq=w.seq, hidden=w.hidden, heads=w.heads, ffn=w.ffn,
                             attn_dropout=float(np.float32(w.attn_dropout)),
                             hidden_dropout=float(np.float32(w.hidden_dropout)),
                             pre_layer_norm=w.pre_layer_norm, seed=w.seed, storage=w.dtype)
    idx = np.arange(nseq)
    wt = {n: to_f64(inp.weights[0][n]) for n in oracle.WEIGHT_NAMES}
    x = to_f64(inp.x)[:nseq]
    dy = to_f64(inp.dy)[:nseq]
    t0 = time.perf_counter()
    oracle.layer_forward_backward(cfg, x, None, wt, dy, seq_index=idx)
    return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def size_sample(w, inp, target_s: float) -> tuple[int, float]:
    t1 = oracle_step(w, inp, 1)
    nseq = int(max(1, min(w.batch, round(target_s / max(t1, 1e-3)))))
    return nseq, t1


def cpu_baseline(w, inp, target_s: float = 15.0) -> dict:
    nseq, _ = size_sample(w, inp, target_s)
    t = oracle_step(w, inp, nseq)
    reps = 1
    # the whole batch can take less than the target: repeat it (at most 4 times)
    while t < 0.67 * target_s and reps < 4:
        t += oracle_step(w, inp, nseq)
        reps += 1
    return {"value": reps * nseq * w.seq / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"float64 oracle forward+backward of {nseq} of the {w.batch} sequences "
                      f"({nseq * w.seq} tokens) x {reps}, {t:.1f} s"}


def run_reference(args) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    nseq, _ = size_sample(w, inp, 3.0)
    for _ in range(args.warmup):
        oracle_step(w, inp, nseq)
    times = [oracle_step(w, inp, nseq) for _ in range(args.steps)]
    tot = sum(times)
    value = args.steps * nseq * w.seq / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: float64 oracle forward+backward of {nseq} of the {w.batch} "
                                   f"sequences ({nseq * w.seq} tokens)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w) -> dict:
    return {"workload": w.name, "batch": w.batch, "seq": w.seq, "hidden": w.hidden, "heads": w.heads,
            "ffn": w.ffn, "attn_dropout": w.attn_dropout, "hidden_dropout": w.hidden_dropout,
            "layer_norm": "pre" if w.pre_layer_norm else "post", "padding": w.lengths is not None,
            "l2": "flushed (256 MiB write) between timed steps", "parallelism": "data-parallel replicas"}


# ---------------------------------------------------------------- GPU arm
class StepRunner:
    """One forward + backward of the layer on fixed device buffers, replayed
    as a captured CUDA graph of the library's launches (or eagerly)."""

    def __init__(self, layer, x, mask, wt, dy, y, dx, grads, use_graph: bool):
        self.layer, self.x, self.mask, self.wt, self.dy = layer, x, mask, wt, dy
        self.y, self.dx, self.grads = y, dx, grads
        self.graph = None
        if use_graph:
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                self.eager()
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph):
                self.eager()
            torch.cuda.synchronize()

    def eager(self):
        self.layer.forward(self.x, self.mask, self.wt, y=self.y)
        self.layer.backward(self.x, self.dy, self.wt, grads=self.grads, dx=self.dx)

    def __call__(self):
        if self.graph is not None:
            self.graph.replay()
        else:
            self.eager()


def run_ours(args) -> None:
    import transformer_layer_pre_b200 as tlp
    from transformer_layer_pre_b200 import Layer, WEIGHT_NAMES
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    dt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[w.dtype]
    elem = 2 if w.dtype != "f32" else 4
    inp = make_inputs(w)
    T = w.tokens
    layer = Layer(w.batch, w.seq, w.hidden, w.heads, w.ffn, w.attn_dropout, w.hidden_dropout, w.pre_layer_norm,
                  w.seed, dtype=dt, gelu_checkpoint=w.gelu_checkpoint, stochastic_mode=args.stochastic_mode)
    wt = {n: inp.weights[0][n].to(dev) for n in WEIGHT_NAMES}
    mask = None if inp.mask is None else inp.mask.to(dev)
    # gradients are views of one flat buffer: data-parallel ranks average it with one all-reduce
    from transformer_layer_pre_b200.dp import FlatGrads, allreduce_mean
    flat = FlatGrads(w.hidden, w.ffn, dev)
    grads = flat.as_dict()

    def exchange():
        if world > 1:
            allreduce_mean(flat)
    # two buffer sets, so the end-to-end run can overlap one step's copies with the other's compute
    xs = [inp.x.to(dev) for _ in range(2)]
    dys = [inp.dy.to(dev) for _ in range(2)]
    ys = [torch.empty_like(xs[0]) for _ in range(2)]
    dxs = [torch.empty_like(xs[0]) for _ in range(2)]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    # launches per step, counted on one eager step
    l0 = tlp.launch_count()
    layer.forward(xs[0], mask, wt, y=ys[0])
    layer.backward(xs[0], dys[0], wt, grads=grads, dx=dxs[0])
    launches_per_step = tlp.launch_count() - l0
    torch.cuda.synchronize()
    runners = [StepRunner(layer, xs[i], mask, wt, dys[i], ys[i], dxs[i], grads, not args.no_graph) for i in range(2)]

    with ClockSampler(local) as clk:
        for _ in range(args.warmup):
            runners[0]()
            exchange()
        tlp.device_check()
        # ---- timed region: per-step events, L2 flushed between steps (outside the events)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        # let the sampling thread take the interpreter lock often during the
        # few milliseconds of the timed region (the default is every 5 ms)
        switch = sys.getswitchinterval()
        sys.setswitchinterval(1e-4)
        clk.timed = True
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            runners[0]()
            exchange()
            b.record(stream)
        # the steps run on the device meanwhile: sample the clocks until the last one ends
        while not evs[-1][1].query():
            clk.sample()
            time.sleep(2e-4)
        torch.cuda.synchronize()
        clk.timed = False
        sys.setswitchinterval(switch)
        barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = reduce_max(sum(step_ms) / len(step_ms))
    tlp.device_check()
    value = world * T / (ms / 1e3)
    launches = launches_per_step * args.steps

    # ---- kernel-class breakdown (same steps, eager, library event profiler on)
    tlp.profile_enable(True)
    for _ in range(args.steps):
        flush.zero_()
        runners[0].eager()
    prof = tlp.profile_read()
    tlp.profile_enable(False)
    peaks = load_peaks()
    clocks = clk.summary()
    classes = {}
    for c, (cms, n) in prof.items():
        if n == 0:
            continue
        work, unit = class_work(c, w, T, elem)
        per_step_ms = cms / args.steps
        classes[c] = {"ms_per_step": per_step_ms, "launch_groups_per_step": n / args.steps,
                      "achieved": (work / (per_step_ms / 1e3)) / (1e12 if unit == "flop" else 1e9),
                      "unit": "TFLOP/s" if unit == "flop" else "GB/s"}
    dom = max(classes, key=lambda c: classes[c]["ms_per_step"])
    d = classes[dom]
    if d["unit"] == "TFLOP/s":
        tensor = dom == "gemm" or tlp_uses_tensor_attention(dom, w)
        if tensor:
            # the burst figure while the timed region ran at full clock; the
            # sustained one once the power cap held the clock down
            if full_clock(clocks):
                bound, peak, src = "tensor", peaks["tflops"], f"{peaks['source']} bf16 burst (fp16:bf16 = 1:1)"
            else:
                bound, peak, src = ("tensor", peaks["tflops_sustained"],
                                    f"{peaks['source']} bf16 sustained (fp16:bf16 = 1:1; clock held below max)")
        else:
            mhz = (clocks or {}).get("sm_mhz") or 1965.0
            bound, peak, src = "alu", alu_peak_tflops(mhz), f"148 SMs x 128 FP32 lanes x 2 x {mhz:.0f} MHz"
    else:
        bound, peak, src = "hbm", peaks["hbm_gbs"], f"{peaks['source']} copy bandwidth"
    roofline = {"bound": bound, "kernel": dom, "achieved": d["achieved"], "peak": peak, "unit": d["unit"],
                "frac": d["achieved"] / peak,
                "traffic": recorded_gemm_traffic(args.workload) if dom == "gemm" else None,
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, mean over one step's GEMM "
                                  "launches (profiles/gemm_tc_pair_bert-large-f16.txt)", "peak_source": src,
                "launches_per_step": d["launch_groups_per_step"]}
    if bound == "tensor":
        roofline["frac_of_burst_peak"] = d["achieved"] / peaks["tflops"]
        roofline["frac_of_sustained_peak"] = d["achieved"] / peaks["tflops_sustained"]
    step_flops = (linear_flops_per_token(w.hidden, w.ffn) + attn_flops_per_token(w.seq, w.hidden)) * T
    tensor_frac_burst = (step_flops / (ms / 1e3)) / (peaks["tflops"] * 1e12)
    tensor_frac_sustained = (step_flops / (ms / 1e3)) / (peaks["tflops_sustained"] * 1e12)
    tensor_frac = tensor_frac_burst if full_clock(clocks) else tensor_frac_sustained

    # ---- end to end through the public API: every step copies its inputs in
    # from pinned host memory and its results (y, dx) back; copies run on
    # their own streams so step i+1's input copy and step i-1's output copy
    # overlap step i's compute (double-buffered device tensors)
    hx, hdy = inp.x.pin_memory(), inp.dy.pin_memory()
    hys = [torch.empty(xs[0].shape, dtype=dt).pin_memory() for _ in range(2)]
    hdxs = [torch.empty(xs[0].shape, dtype=dt).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    done = [torch.cuda.Event() for _ in range(2)]
    outd = [torch.cuda.Event() for _ in range(2)]
    for e_ in done + outd:
        e_.record(stream)
    torch.cuda.synchronize()

    def e2e_run(nsteps: int, eager: bool) -> float:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(nsteps):
            bsel = i & 1
            ready = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                s_in.wait_event(done[bsel])     # compute of step i-2 is done with this buffer set
                xs[bsel].copy_(hx, non_blocking=True)
                dys[bsel].copy_(hdy, non_blocking=True)
                ready.record(s_in)
            stream.wait_event(ready)
            stream.wait_event(outd[bsel])       # results of step i-2 have left this buffer set
            if eager:
                runners[bsel].eager()           # layer_forward + layer_backward through the C ABI
            else:
                runners[bsel]()
            exchange()
            done[bsel].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[bsel])
                hys[bsel].copy_(ys[bsel], non_blocking=True)
                hdxs[bsel].copy_(dxs[bsel], non_blocking=True)
                outd[bsel].record(s_out)
        s_in.wait_stream(s_out)
        s_in.wait_stream(stream)
        t1.record(s_in)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(args.warmup, True)
    e2e = reduce_max(e2e_run(args.steps, True) / args.steps)
    e2e_run(args.warmup, False)
    e2e_graph = reduce_max(e2e_run(args.steps, False) / args.steps)
    io = T * w.hidden * elem

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, inp)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,0.02) weights, N(0,1) x and dY)",
            "config": workload_config(w), "graph": not args.no_graph, "stochastic_mode": args.stochastic_mode,
            "tensor_peak_frac": tensor_frac,
            "tensor_peak_frac_of_burst": tensor_frac_burst,
            "tensor_peak_frac_of_sustained": tensor_frac_sustained,
            "roofline": roofline, "kernel_classes": classes, "cpu_baseline": cpu,
            "e2e": {"value": world * T / (e2e / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": 2 * io,
                    "d2h_bytes_per_step": 2 * io, "ms_per_step": e2e,
                    "note": "every step: pinned host x, dY in, layer_forward + layer_backward called through "
                            "the C ABI, y, dx out; copies on their own streams overlap neighbouring steps",
                    "graph_replay": {"value": world * T / (e2e_graph / 1e3), "ms_per_step": e2e_graph,
                                     "note": "the same, the two API calls replayed from a captured CUDA graph"}},
            "gpu_launches": launches, "launches_per_step": launches_per_step, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    del runners
    layer.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def tlp_uses_tensor_attention(cls: str, w) -> bool:
    """Attention runs on tensor cores when the library's tensor-core attention
    serves this shape (16-bit storage); the SIMT kernels otherwise."""
    import transformer_layer_pre_b200 as tlp
    return bool(getattr(tlp, "attention_uses_tensor_cores", lambda *a: False)(w.dtype, w.heads, w.hidden // w.heads,
                                                                              w.seq))


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every kernel eagerly instead of replaying a CUDA graph")
    ap.add_argument("--stochastic-mode", action="store_true",
                    help="relaxed determinism: bias, LayerNorm and split-K weight gradients summed with atomics")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
