#!/usr/bin/env python
"""Benchmark of the gated delta rule library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  A step is one prefill call over the
Qwen3.8-27B-shaped DeltaNet layer workload (B=1, T=8192, 16 QK / 48 V heads,
head dim 128, bf16 q/k/v, fp32 g/beta, fp32 state, zero initial state, final
state returned), captured once in a CUDA graph and replayed; the same call
launched eagerly is reported beside it (``eager``).  ``value`` is prefill
throughput in Mtok/s with the inputs resident in HBM, L2 flushed between timed
steps.  The same line carries:
  roofline     the prefill call against the tensor-core roofline (algorithmic
               flops / CUDA-event time over the measured bf16 peak), with the
               HBM fractions for fp32 o and for bf16 o beside it;
  prefill_long262k, prefill_varlen32
               the prefill on the long-context (262,144 tokens, slow decay,
               nonzero initial state updated in place) and the variable-length
               (32 packed sequences) workloads, each with its own roofline;
  decode       the batched decode workload (B=64, 1000 steps, fp32 state of
               201 MB updated in place): state GB/s against HBM peak;
  decode_tokens  the same batch with 4 tokens per sequence per call through the
               multi-token decode over a state pool: tokens/s, GB/s against HBM peak;
  prefill_raw_inputs
               the same step from raw projections (normalisation and gates
               folded into the kernels), with the prepared-input time and the
               time with a separate PyTorch prologue for context;
  prefill_backward
               the backward pass of the same step (gradients for q, k, v, g,
               beta and the initial state; CUDA cores, fp32);
  decode_bf16_state, decode_tokens_bf16_state
               the same with the state pool at rest in bf16 (fp32 arithmetic,
               100 MB of state), 1 and 4 tokens per call;
  e2e          prefill through the public API with inputs copied from pinned
               host memory and o / final state copied back, every step;
  cpu_baseline the fp64 oracle on the host cores (rank 0, N=1 only);
  clocks       SM clocks and throttle reasons sampled during the timed region.
With --gpus N under torchrun each rank runs its own independent workload
(weak scaling, no collective on the data path); timings are the max over
ranks.  ``--impl reference`` times the fp64 oracle instead, on the host.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Algorithmic work per token of one DeltaNet layer at Hqk=16, Hv=48, D=128, chunk 64.
#   flops: per (chunk, V head): QK^T 1.05M + KK^T 1.05M (both shared by the 3 V heads
#   of a QK head) + W 1.05M + U~ 1.05M + W S0^T 2.10M + Q S0^T 2.10M + P U 1.05M +
#   state 2.10M  ->  7,602,176 flop per token over the layer.
#   bytes: q 4096 + k 4096 + v 12288 (bf16) + o 24576 (fp32) + g 192 + beta 192
#   = 45,440 per token.
FLOP_PER_TOKEN = 7_602_176
BYTES_PER_TOKEN = 45_440
# The same with o in bf16 (the input dtype): o 12288 B/token instead of 24576.
BYTES_PER_TOKEN_BF16_O = 33_152
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--decode-steps", type=int, default=1000)
    p.add_argument("--no-backward", action="store_true", help="skip the backward-pass leg")
    p.add_argument("--backward-tokens", type=int, default=0,
                   help="run the backward leg on the first N tokens of the workload (small "
                        "profiling captures); 0 = all")
    p.add_argument("--no-long", action="store_true",
                   help="skip the long262k and varlen32 prefill legs (~20 GB of device memory)")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args(argv)


# ---------------------------------------------------------------- distributed
class Dist:
    """Rank bookkeeping; torch.distributed only for barriers and max-over-ranks."""

    def __init__(self, backend=None):
        import torch.distributed as dist

        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.dist = dist if self.world > 1 else None
        if self.dist is not None and not dist.is_initialized():
            import datetime

            dist.init_process_group(backend=backend or "nccl",
                                    timeout=datetime.timedelta(seconds=120))

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x: float, device=None) -> float:
        if self.dist is None:
            return float(x)
        import torch

        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None and self.dist.is_initialized():
            self.dist.destroy_process_group()


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent workload (weak scaling)."""
    return base + 1000 * rank


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, max clock and throttle reasons of one GPU every
    `period_s` (NVML) while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device_index=0, period_s=0.005):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self._stop = None

    def __enter__(self):
        import threading

        try:
            import pynvml

            pynvml.nvmlInit()
            uuid = self.idx if isinstance(self.idx, str) else None
            self.h = (pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else
                      pynvml.nvmlDeviceGetHandleByIndex(int(self.idx)))
            self.nv = pynvml
        except Exception:
            self.nv = None
            return self
        self._stop = threading.Event()

        def loop():
            nv = self.nv
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    mx = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
                    get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                        nv.nvmlDeviceGetCurrentClocksThrottleReasons
                    rs = get_reasons(self.h)
                    self.samples.append((sm, mx, rs))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._t = threading.Thread(target=loop, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)
        return False

    def summary(self):
        if not self.samples:
            return None
        sm = [x[0] for x in self.samples]
        reasons = sorted({name for _, _, r in self.samples for name, bit in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": reasons, "samples": len(sm), "source": "nvml"}


def gpu_uuid(torch, dev):
    """NVML identifier of the torch device: its UUID string, else its index."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return dev.index or 0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def sources_sha(source_files) -> str:
    h = hashlib.sha256()
    for path in ([source_files] if isinstance(source_files, str) else source_files):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_entry(kernel_key: str, source_files):
    """The committed ncu figures of a kernel (profiles/traffic.json), or None
    when a source changed after the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            ent = json.load(f)[kernel_key]
        return ent if ent.get("source_sha") == sources_sha(source_files) else None
    except (OSError, ValueError, KeyError):
        return None


def kernel_traffic(kernel_key: str, source_files):
    """DRAM bytes per launch (per step for a multi-launch entry) from a
    committed ncu summary, or None when a source changed since."""
    ent = traffic_entry(kernel_key, source_files)
    return None if ent is None else ent["dram_bytes_per_launch"]


CSRC = os.path.join(ROOT, "gated_deltanet_recurrence_rule_b200", "csrc")
PREFILL_SOURCES = [os.path.join(CSRC, n) for n in
                   ("gdn_common.cuh", "gdn_twophase.cuh", "gdn_chunk_ops.cuh", "gdn_sm100.cuh",
                    "gdn_wy_prep.cu", "gdn_state_pass.cu")]
DECODE_SOURCES = [os.path.join(CSRC, n) for n in ("gdn_common.cuh", "gdn_decode.cu")]


# ---------------------------------------------------------------- oracle (CPU)
def oracle_prefill_timed(inp, ntok, num_threads=0):
    """Time the fp64 oracle on the first ``ntok`` tokens (all heads) of a
    single-sequence prefill workload; returns (seconds, threads used)."""
    import numpy as np

    import oracle

    lib = oracle.load()
    sl = {n: inp[n][:ntok] for n in ("q", "k", "v", "g", "beta")}
    arrs = {n: np.ascontiguousarray(sl[n].double().numpy()) for n in sl}
    cu = np.array([0, ntok], dtype=np.int64)
    Hv = arrs["v"].shape[1]
    threads = num_threads if num_threads > 0 else (os.cpu_count() or 1)
    threads = min(threads, Hv)
    t0 = time.perf_counter()
    oracle.prefill(arrs["q"], arrs["k"], arrs["v"], arrs["g"], arrs["beta"], cu_seqlens=cu,
                   num_threads=threads, want_final=True, lib=lib)
    return time.perf_counter() - t0, threads


# ---------------------------------------------------------------- main arms
def workload_desc(w):
    return (f"{w.name}: B={len(w.lengths)} T={w.total_tokens} Hqk={w.Hqk} Hv={w.Hv} D={w.D} "
            f"{w.dtype} q/k/v, fp32 g/beta, fp32 o, fp32 state "
            f"{'zero init' if w.init_std == 0 else 'N(0,%g) init' % w.init_std}, final state returned")


def run_reference(args, D):
    """The fp64 oracle timed on the host cores (rank 0 only)."""
    import torch

    from gated_deltanet_recurrence_rule_b200 import inputs

    w = inputs.WORKLOADS["prefill8k"]
    if D.rank != 0:
        return None
    inp = inputs.workload_inputs(w)
    ntok = 1024
    secs = []
    threads = 1
    for i in range(args.warmup + args.steps):
        s, threads = oracle_prefill_timed(inp, ntok)
        if i >= args.warmup:
            secs.append(s)
    total = sum(secs)
    value = ntok * len(secs) / total / 1e6
    return {
        "impl": "reference",
        "metric": "GDN prefill Mtok/s (H=16/48,D=128) and decode-step state GB/s vs HBM peak",
        "value": value, "unit": "Mtok/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total / len(secs) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "global_batch": 1, "seq_len": w.total_tokens,
                   "parallelism": "host threads over (sequence, V head)",
                   "sample": f"first {ntok} tokens, all 48 V heads, per step"},
        "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {ntok} of 8192 tokens, all 48 V heads, per step"},
        "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ours(args, D):
    import torch

    from gated_deltanet_recurrence_rule_b200 import api, inputs

    dev = torch.device("cuda", D.local_rank)
    torch.cuda.set_device(dev)
    api.load()
    w = inputs.WORKLOADS["prefill8k"]
    inp = inputs.prefill_inputs(w.lengths, w.Hqk, w.Hv, w.D, dtype=w.dtype,
                                seed=rank_seed(w.seed, D.rank))
    T = w.total_tokens
    x = {n: t.to(dev) for n, t in inp.items() if t is not None}
    o = torch.empty((T, w.Hv, w.D), dtype=torch.float32, device=dev)
    fin = torch.empty((1, w.Hv, w.D, w.D), dtype=torch.float32, device=dev)
    ws = torch.zeros(api.prefill_workspace_size(1, T, w.Hqk, w.Hv, w.D, w.D), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2

    def step():
        api.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"],
                    final_state=fin, o=o, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    D.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(gpu_uuid(torch, dev))
    clk.__enter__()  # sampled through the prefill, e2e and decode timed regions
    if True:
        for e0, e1 in evs:
            flush.zero_()              # outside the timed pair: L2 holds nothing of the inputs
            e0.record(stream)
            step()
            e1.record(stream)
        torch.cuda.synchronize()
    D.barrier()
    per_ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    local_ms = sum(per_ms)
    max_ms = D.max(local_ms, dev)
    # The same call captured in a CUDA graph (its 13 launches on two internal
    # streams become graph nodes) and replayed, L2 flushed before each step.
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        step()
    graph.replay()
    torch.cuda.synchronize()
    gevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    D.barrier()
    torch.cuda.synchronize()
    for e0, e1 in gevs:
        flush.zero_()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    D.barrier()
    graph_per_ms = [e0.elapsed_time(e1) for e0, e1 in gevs]
    graph_ms = D.max(sum(graph_per_ms), dev) / args.steps
    del graph
    status = api.get_device_status(ws)
    if status != api.GDN_OK:
        raise RuntimeError(f"device status after timing: {api.status_string(status)}")
    # Headline: the step replayed from the CUDA graph (the same 13 launches with
    # the host's launch and event overhead taken off the GPU's critical path);
    # the eager call is reported beside it.
    eager_ms = max_ms / args.steps
    ms_per_step = graph_ms
    value = D.world * T / (graph_ms / 1e3) / 1e6

    peaks, peak_src = load_peaks()
    kernel_ms = statistics.mean(graph_per_ms)
    launches = api.prefill_launch_count(1, T, w.Hqk, w.Hv, w.D, w.D, ws.numel())
    if _tc_path_available():
        roof = prefill_roofline(T, w.Hv, w.D, kernel_ms, peaks, peak_src, state_io=1)
        # One prefill call is a sequence of launches (plan, then WY prep and
        # state pass per round, on two streams, rounds pipelined): the time is
        # the whole call's, between CUDA events on the caller's stream that
        # bracket every launch of the step.
        ent = traffic_entry("prefill_step", PREFILL_SOURCES)
        roof.update({"kernel": f"prefill step: plan_kernel + wy_prep_kernel and state_pass_kernel "
                               f"per round ({launches} launches, 2 streams, pipelined)",
                     "kernel_ms": kernel_ms,
                     "traffic": None if ent is None else ent["dram_bytes_per_launch"],
                     "dominant": None if ent is None else ent.get("dominant")})
    else:
        # CUDA-core path: 3 fp32 FMAs per state element per token (read, update, output)
        flop = 3 * 2 * w.D * w.D * w.Hv * T
        fp32_peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        achieved = flop / (kernel_ms / 1e3) / 1e12
        roof = {"bound": "alu", "kernel": "prefill_simt_kernel", "achieved": achieved,
                "peak": fp32_peak, "unit": "TFLOP/s", "frac": achieved / fp32_peak,
                "peak_source": "148 SMs x 128 fp32 FMA/clk x 2 x max SM clock",
                "algorithmic": f"3 FMA per state element per token = {flop} flop",
                "traffic": kernel_traffic("prefill_simt", os.path.join(ROOT, "gated_deltanet_recurrence_rule_b200", "csrc", "gdn_prefill_simt.cu"))}

    out = {
        "metric": "GDN prefill Mtok/s (H=16/48,D=128) and decode-step state GB/s vs HBM peak",
        "value": value, "unit": "Mtok/s", "n_gpus": D.world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w), "global_batch": D.world, "seq_len": T,
                   "parallelism": f"replicas{D.world}" if D.world > 1 else "single GPU",
                   "l2": "flushed between timed steps (256 MiB write outside the timed pair)"},
        "roofline": roof,
        "gpu_launches": args.steps * launches,
        "launch": "one gdn_prefill call captured once in a CUDA graph and replayed per step "
                  "(L2 flushed between timed steps)",
        "eager": {"value": D.world * T / (eager_ms / 1e3) / 1e6, "unit": "Mtok/s",
                  "ms_per_step": eager_ms,
                  "how": "the same call launched from the host every step (~80 us of host work per "
                         "call, partly on the GPU's critical path)"},
    }

    out["prefill_raw_inputs"] = _prefill_raw(args, D, dev, x, T, w, ws, fin, o, flush, eager_ms,
                                             launches)

    if not args.no_e2e:
        out["e2e"] = _e2e(args, D, inp, dev, w, ws)

    if not args.no_backward:
        out["prefill_backward"] = _backward(args, D, dev, x, T, w, peaks)
    if not args.no_long:
        out["prefill_long262k"] = _prefill_leg(args, D, dev, peaks, peak_src, "long262k")
        out["prefill_varlen32"] = _prefill_leg(args, D, dev, peaks, peak_src, "varlen32",
                                               single_pass=True)

    if not args.no_decode:
        out["decode"] = _decode(args, D, dev, peaks, peak_src)
        out["decode_tokens"] = _decode_tokens(args, D, dev, peaks, peak_src)
        out["decode_bf16_state"] = _decode_tokens(args, D, dev, peaks, peak_src, tokens=1,
                                                  state_dtype="bf16")
        out["decode_tokens_bf16_state"] = _decode_tokens(args, D, dev, peaks, peak_src,
                                                         state_dtype="bf16")
    clk.__exit__(None, None, None)
    out["clocks"] = clk.summary()

    if not args.no_cpu_baseline and D.rank == 0 and D.world == 1:
        secs, threads = oracle_prefill_timed(inp, T)
        n1 = 1024  # one core, a bounded sample: the first 1024 tokens, all heads
        secs1, _ = oracle_prefill_timed(inp, n1, num_threads=1)
        out["cpu_baseline"] = {"value": T / secs / 1e6, "unit": "Mtok/s", "cores": threads,
                               "kind": "oracle",
                               "sample": f"the whole workload ({T} tokens x {w.Hv} V heads) once, "
                                         f"{secs:.1f} s wall",
                               "single_core": {"value": n1 / secs1 / 1e6, "unit": "Mtok/s",
                                               "sample": f"first {n1} tokens x {w.Hv} V heads, "
                                                         f"1 thread, {secs1:.1f} s wall"}}
    return out


def prefill_roofline(T, Hv, D, ms, peaks, peak_src, state_io):
    """Roofline of one tensor-core prefill call of T tokens taking ``ms``.
    The fraction is tensor-pipe utilisation: algorithmic flops over time
    against the measured bf16 dense (burst) peak.  Beside it the HBM
    fractions for the two readings of the output bytes (fp32 o as written,
    45,440 B/token; bf16 o, 33,152 B/token) plus ``state_io`` states of
    Hv x D x D fp32 per sequence-call (final, or initial and final)."""
    flops = FLOP_PER_TOKEN * T
    state_bytes = state_io * Hv * D * D * 4
    b32 = BYTES_PER_TOKEN * T + state_bytes
    b16 = BYTES_PER_TOKEN_BF16_O * T + state_bytes
    sec = ms / 1e3
    tensor_ach = flops / sec / 1e12
    return {"bound": "tensor", "achieved": tensor_ach, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": tensor_ach / peaks["bf16_tflops"],
            "peak_source": f"{peak_src} bf16_tflops (burst; the call is timed alone)",
            "algorithmic": f"{FLOP_PER_TOKEN} flop/token x {T} tokens",
            "tensor_frac": tensor_ach / peaks["bf16_tflops"],
            "tensor_achieved_tflops": tensor_ach,
            "hbm_frac": b32 / sec / 1e9 / peaks["hbm_gbs"],
            "hbm_algorithmic": f"{BYTES_PER_TOKEN} B/token (fp32 o) x {T} + states",
            "hbm_frac_bf16_o": b16 / sec / 1e9 / peaks["hbm_gbs"],
            "hbm_algorithmic_bf16_o": f"{BYTES_PER_TOKEN_BF16_O} B/token (bf16 o) x {T} + states",
            "floor_us": {"tensor": flops / (peaks["bf16_tflops"] * 1e12) * 1e6,
                         "hbm_fp32_o": b32 / (peaks["hbm_gbs"] * 1e9) * 1e6,
                         "hbm_bf16_o": b16 / (peaks["hbm_gbs"] * 1e9) * 1e6}}


def _tc_path_available():
    from gated_deltanet_recurrence_rule_b200 import api

    return api.prefill_uses_tensor_cores(16, 48, 128, 128)


def _e2e(args, D, inp, dev, w, ws):
    """The prefill through the public API with host buffers: every step copies
    its inputs from pinned host memory to the device and its o and final state
    back.  Consecutive steps are pipelined on three streams (upload of step
    i+1, prefill of step i, download of step i-1) with double-buffered device
    inputs and outputs, so PCIe's two directions and the GPU work overlap."""
    import torch

    from gated_deltanet_recurrence_rule_b200 import api

    names = ("q", "k", "v", "g", "beta", "cu_seqlens")
    host = {n: inp[n].pin_memory() for n in names}
    T = w.total_tokens
    devb = [{n: torch.empty_like(host[n], device=dev) for n in names} for _ in range(2)]
    o = [torch.empty((T, w.Hv, w.D), dtype=torch.float32, device=dev) for _ in range(2)]
    fin = [torch.empty((1, w.Hv, w.D, w.D), dtype=torch.float32, device=dev) for _ in range(2)]
    o_host = [torch.empty((T, w.Hv, w.D), dtype=torch.float32).pin_memory() for _ in range(2)]
    f_host = [torch.empty((1, w.Hv, w.D, w.D), dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host[0].numel() * 4 + f_host[0].numel() * 4
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    ev_in, ev_comp, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    state = {"i": 0}

    def step():
        i = state["i"]
        b = i % 2
        state["i"] += 1
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])           # step i-2 no longer reads devb[b]
            for n in names:
                devb[b][n].copy_(host[n], non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_out[b])          # step i-2's o, final state are on the host
            x = devb[b]
            api.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"],
                        final_state=fin[b], o=o[b], workspace=ws)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            o_host[b].copy_(o[b], non_blocking=True)
            f_host[b].copy_(fin[b], non_blocking=True)
            ev_out[b].record(s_out)

    main = torch.cuda.current_stream(dev)

    def run(n):
        for st in (s_in, s_comp, s_out):
            st.wait_stream(main)
        for _ in range(n):
            step()
        for st in (s_in, s_comp, s_out):
            main.wait_stream(st)

    run(max(args.warmup, 3))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier()
    torch.cuda.synchronize()
    e0.record(main)
    run(args.steps)
    e1.record(main)
    torch.cuda.synchronize()
    D.barrier()
    ms = D.max(e0.elapsed_time(e1), dev)
    return {"value": D.world * T * args.steps / (ms / 1e3) / 1e6, "unit": "Mtok/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / args.steps, "host_buffers": "pinned",
            "pipelined": "upload of step i+1, prefill of step i and download of step i-1 on "
                         "three streams, device buffers doubled"}


def _prefill_raw(args, D, dev, x, T, w, ws, fin, o, flush, prepared_ms, launches):
    """The same prefill step from the layer's raw projections (GDN_INPUT_RAW):
    q, k unnormalised, g and beta as the pre-activations a, b.  The kernels fold
    the normalisation and the gates in; for context, the same inputs prepared by
    separate PyTorch ops (one more pass over q, k, g, beta) before the prepared
    prefill."""
    import torch
    import torch.nn.functional as F

    from gated_deltanet_recurrence_rule_b200 import api

    gen = torch.Generator(device=dev).manual_seed(11)
    scale = lambda t: torch.exp(torch.randn(t.shape[:-1] + (1,), generator=gen, device=dev))
    q = (x["q"].float() * scale(x["q"])).to(x["q"].dtype)
    k = (x["k"].float() * scale(x["k"])).to(x["k"].dtype)
    a = torch.log(torch.expm1(-x["g"].double())).float()     # -softplus(a) = g
    b = torch.log(x["beta"].double() / (1 - x["beta"].double())).float()  # sigmoid(b) = beta

    def fused():
        api.prefill(q, k, x["v"], a, b, cu_seqlens=x["cu_seqlens"], final_state=fin, o=o,
                    workspace=ws, raw_inputs=True)

    def separate():
        qn = F.normalize(q.float(), dim=-1).to(q.dtype)
        kn = F.normalize(k.float(), dim=-1).to(k.dtype)
        api.prefill(qn, kn, x["v"], -F.softplus(a), torch.sigmoid(b), cu_seqlens=x["cu_seqlens"],
                    final_state=fin, o=o, workspace=ws)

    stream = torch.cuda.current_stream(dev)
    res = {}
    for name, fn in (("fused", fused), ("separate", separate)):
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        D.barrier()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        D.barrier()
        res[name] = D.max(sum(e0.elapsed_time(e1) for e0, e1 in evs), dev) / args.steps
    status = api.get_device_status(ws)
    if status != api.GDN_OK:
        raise RuntimeError(f"device status after the raw-input leg: {api.status_string(status)}")
    return {"value": D.world * T / (res["fused"] / 1e3) / 1e6, "unit": "Mtok/s",
            "workload": "prefill8k from raw projections (q, k unnormalised; g, beta as the "
                        "pre-activations of -softplus and sigmoid)",
            "ms_per_step": res["fused"], "prepared_inputs_ms_per_step_eager": prepared_ms,
            "separate_torch_prologue_ms_per_step": res["separate"],
            "l2": "flushed between timed steps", "gpu_launches": args.steps * launches}


def _prefill_leg(args, D, dev, peaks, peak_src, name, single_pass=False):
    """The prefill on another named workload: long262k (one 262,144-token
    sequence, slow decay, nonzero initial state returned as the final state in
    place) or varlen32 (32 packed sequences of 1k to 32k tokens with their own
    initial states, final states returned).  Unlike prefill8k, varlen32 gives
    the state pass many chains at once, so it shows what the two phases cost in
    SM time; there the single-pass kernel (chosen by a header-only workspace) is
    timed beside it.  Inputs are larger than L2, so no flush is needed."""
    import torch

    from gated_deltanet_recurrence_rule_b200 import api, inputs

    w = inputs.WORKLOADS[name]
    inp = inputs.prefill_inputs(w.lengths, w.Hqk, w.Hv, w.D, dtype=w.dtype,
                                seed=rank_seed(w.seed, D.rank), g_mu=w.g_mu, init_std=w.init_std)
    x = {n: t.to(dev) for n, t in inp.items() if t is not None}
    del inp
    T, N = w.total_tokens, len(w.lengths)
    o = torch.empty((T, w.Hv, w.D), dtype=torch.float32, device=dev)
    # the final state overwrites the initial state in place (a resumable prefill)
    state = x["initial_state"]
    full = torch.zeros(api.prefill_workspace_size(N, T, w.Hqk, w.Hv, w.D, w.D), dtype=torch.uint8,
                       device=dev)
    header = torch.zeros(256, dtype=torch.uint8, device=dev)  # selects the single-pass kernel
    steps = max(1, min(args.steps, 3))
    stream = torch.cuda.current_stream(dev)

    def timed(ws):
        def step():
            api.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"],
                        initial_state=state, final_state=state, o=o, workspace=ws)

        for _ in range(2):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        D.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        D.barrier()
        if api.get_device_status(ws) != api.GDN_OK:
            raise RuntimeError(f"device status after the {name} leg")
        return D.max(e0.elapsed_time(e1), dev) / steps

    ms = timed(full)
    out = {"value": D.world * T / (ms / 1e3) / 1e6, "unit": "Mtok/s", "ms_per_step": ms,
           "workload": workload_desc(w) + ", final state written over the initial state",
           "roofline": prefill_roofline(T, w.Hv, w.D, ms, peaks, peak_src, state_io=2 * N),
           "gpu_launches": steps * api.prefill_launch_count(N, T, w.Hqk, w.Hv, w.D, w.D,
                                                            full.numel()),
           "warmup": 2, "steps": steps, "l2": "inputs larger than L2"}
    if single_pass:
        ms_single = timed(header)
        out["single_pass"] = {"value": D.world * T / (ms_single / 1e3) / 1e6, "unit": "Mtok/s",
                              "ms_per_step": ms_single,
                              "how": "the same call with a 256-byte workspace: one CTA per "
                                     "(sequence, value head) runs all its chunks"}
    return out


# Algorithmic flops of the chunk-form backward per (64-token chunk, value head)
# at head dim D (an FMA counts 2; the solve of the 64 x 64 triangular system,
# the elementwise work and the 3-term split of every tensor-core product are
# not counted).  Each term is one matrix product of the algebra:
#   prep         Q K^T, K K^T, W = Tm (.) K, U~ = Tm (.) V          4 x 64.64.D
#   forward      U = U~ - W S0^T, S1 = g S0 + U^T (.) K             2 x 64.D.D
#   reverse      P^T dO', K dS1^T, dO'^T (.) Q, dU^T W              64.64.D + 3 x 64.D.D
#   state grads  dO' S0, dU S0, U dS1                               3 x 64.D.D
#   local grads  dO' U^T, dW K^T, dU V^T, Tm^T dW, Tm^T dU,
#                (dP.E) K, (dP.E)^T Q, (B + B^T) K                  8 x 64.64.D
#                dT Tm^T, Tm^T Z                                    2 x 64.64.64
def backward_chunk_flops(D: int, C: int = 64) -> int:
    return 2 * (13 * C * C * D + 8 * C * D * D + 2 * C * C * C)


def _backward(args, D, dev, x, T, w, peaks):
    """Backward pass of the prefill step on the same workload: d_o and
    dL/dS_final random fp32, gradients for q, k, v, g, beta and the initial
    state.  The leg's value is the chunk form (gdn_prefill_backward with its
    full workspace, tf32 tensor-core products with a 3-term split); the
    sequential CUDA-core form (gdn_prefill_backward_sequential) is timed
    beside it."""
    import torch

    from gated_deltanet_recurrence_rule_b200 import api

    if 0 < args.backward_tokens < T:
        T = args.backward_tokens
        x = {n: (t[:T] if n in ("q", "k", "v", "g", "beta") else t) for n, t in x.items()}
        x["cu_seqlens"] = torch.tensor([0, T], dtype=torch.int32, device=dev)
    gen = torch.Generator(device=dev).manual_seed(12)
    d_o = torch.randn((T, w.Hv, w.D), generator=gen, device=dev)
    d_sf = torch.randn((1, w.Hv, w.D, w.D), generator=gen, device=dev) * 0.1
    steps = max(1, min(args.steps, 3))
    stream = torch.cuda.current_stream(dev)

    def timed(sequential):
        ws = torch.zeros(api.prefill_backward_workspace_size(1, T, w.Hqk, w.Hv, w.D, w.D,
                                                             sequential=sequential),
                         dtype=torch.uint8, device=dev)

        def step():
            return api.prefill_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d_o,
                                        cu_seqlens=x["cu_seqlens"], d_final_state=d_sf,
                                        workspace=ws, sequential=sequential)

        for _ in range(2):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        D.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        D.barrier()
        ms = D.max(e0.elapsed_time(e1), dev) / steps
        status = api.get_device_status(ws)
        if status != api.GDN_OK:
            raise RuntimeError(f"device status after the backward leg: {api.status_string(status)}")
        del ws
        return ms

    ms = timed(False)
    ms_seq = timed(True)
    units = -(-T // 64) * w.Hv
    flop = backward_chunk_flops(w.D) * units
    # tf32 dense peak from the measured bf16 GEMM and the nominal tf32 : bf16 ratio (1.1 : 2.25)
    tf32_peak = peaks["bf16_tflops"] * 1.1 / 2.25
    achieved = flop / (ms / 1e3) / 1e12
    # the sequential form: 18 D^2 fp32 flop per token and value head on CUDA cores
    seq_flop = 18 * w.D * w.D * w.Hv * T
    fp32_peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    seq_ach = seq_flop / (ms_seq / 1e3) / 1e12
    bwd_sources = [os.path.join(CSRC, n) for n in ("gdn_common.cuh", "gdn_chunk_ops.cuh", "gdn_sm100.cuh",
                                                   "gdn_twophase.cuh", "gdn_backward_chunked.cu")]
    return {"value": D.world * T / (ms / 1e3) / 1e6, "unit": "Mtok/s",
            "workload": f"backward of prefill8k: T={T} Hqk={w.Hqk} Hv={w.Hv} D={w.D} bf16 inputs, "
                        "fp32 d_o and dL/dS_final, zero initial state",
            "ms_per_step": ms,
            "roofline": {"bound": "tensor", "kernel": "chunk form: plan, prep, both chains (one launch), "
                                                      "state grads, local grads (dq, dk summed in it)",
                         "achieved": achieved, "peak": tf32_peak, "unit": "TFLOP/s",
                         "frac": achieved / tf32_peak,
                         "peak_source": "measured bf16_tflops x nominal tf32/bf16 (1.1/2.25); products "
                                        "at about fp32 accuracy: state gradients on tcgen05 (bf16 "
                                        "hi/lo, 3 MMAs per step), the rest warp-level (m16n8k16 "
                                        "bf16 with an exact input operand, 2 MMAs per step; "
                                        "m16n8k8 tf32 hi/lo, 3 per step)",
                         "algorithmic": f"{backward_chunk_flops(w.D)} flop per (64-token chunk, value head)"
                                        f" x {units} = {flop} flop",
                         "traffic": kernel_traffic("prefill_backward_chunked", bwd_sources)},
            "sequential": {"ms_per_step": ms_seq, "value": D.world * T / (ms_seq / 1e3) / 1e6,
                           "unit": "Mtok/s",
                           "roofline": {"bound": "alu", "achieved": seq_ach, "peak": fp32_peak,
                                        "unit": "TFLOP/s", "frac": seq_ach / fp32_peak,
                                        "peak_source": "148 SMs x 128 fp32 FMA/clk x 2 x max SM clock",
                                        "algorithmic": f"18 D^2 flop per token and value head = {seq_flop} flop"},
                           "gpu_launches": 5 * steps},
            "gpu_launches": 5 * steps}  # plan, prep, chains, state grads, local grads


def _decode(args, D, dev, peaks, peak_src):
    import torch

    from gated_deltanet_recurrence_rule_b200 import api, inputs

    w = inputs.WORKLOADS["decode64"]
    steps = args.decode_steps
    d = inputs.decode_inputs(w.batch, w.Hqk, w.Hv, w.D, steps=steps, dtype=w.dtype,
                             seed=rank_seed(w.seed, D.rank), init_std=w.init_std)
    x = {n: d[n].to(dev) for n in ("q", "k", "v", "g", "beta")}
    S = d["state"].to(dev)
    o = torch.empty((w.batch, w.Hv, w.D), dtype=torch.float32, device=dev)

    def run(n):
        for s in range(n):
            api.decode_step(x["q"][s], x["k"][s], x["v"][s], x["g"][s], x["beta"][s], S, o=o)

    run(min(steps, 10))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    D.barrier()
    ms = D.max(e0.elapsed_time(e1), dev)
    # The same steps replayed from a CUDA graph of 100 steps (launches with
    # their programmatic-dependent-launch edges captured; fresh inputs per step).
    chunk = min(100, steps)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        run(1)  # warm the binding on the capture stream
    stream.wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        for s_ in range(chunk):
            api.decode_step(x["q"][s_], x["k"][s_], x["v"][s_], x["g"][s_], x["beta"][s_], S, o=o)
    graph.replay()
    torch.cuda.synchronize()
    reps = max(1, steps // chunk)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier()
    torch.cuda.synchronize()
    g0.record(stream)
    for _ in range(reps):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize()
    D.barrier()
    ms_graph = D.max(g0.elapsed_time(g1), dev) / (reps * chunk)
    del graph
    state_bytes = w.batch * w.Hv * w.D * w.D * 4
    # q, k (bf16) + v (bf16) + o (fp32) + g, beta (fp32)
    io_bytes = w.batch * (2 * w.Hqk * w.D * 2 + w.Hv * w.D * 2 + w.Hv * w.D * 4 + 2 * w.Hv * 4)
    per_step = 2 * state_bytes + io_bytes
    us = ms * 1e3 / steps
    gbs = D.world * per_step * steps / (ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    traffic = kernel_traffic("decode", DECODE_SOURCES)
    note = None
    if traffic:
        note = (f"ncu counts {traffic / 1e6:.1f} MB of DRAM traffic per launch against "
                f"{per_step / 1e6:.1f} MB algorithmic: back to back, L2 still holds part of the "
                f"state written by the previous step, so part of this fraction is L2 residency")
    return {"value": gbs, "unit": "GB/s", "workload": f"decode64: B={w.batch} x 1 token, Hqk={w.Hqk} "
            f"Hv={w.Hv} D={w.D} bf16, fp32 state {state_bytes} B in place, {steps} steps",
            "us_per_step": us, "steps_per_s": steps / (ms / 1e3),
            "us_per_step_cuda_graph": ms_graph * 1e3,
            "value_cuda_graph": D.world * per_step / (ms_graph / 1e3) / 1e9,
            "roofline": {"bound": "hbm", "kernel": "decode_step_kernel", "achieved": gbs / D.world,
                         "peak": peak, "unit": "GB/s", "frac": gbs / D.world / peak,
                         "peak_source": f"{peak_src} hbm_gbs",
                         "algorithmic": f"{per_step} B per step (state read+write {2 * state_bytes} + io {io_bytes})",
                         "traffic": traffic, "note": note},
            "gpu_launches": steps}


def _decode_tokens(args, D, dev, peaks, peak_src, tokens=4, state_dtype="fp32"):
    """Multi-token decode (gdn_decode_tokens): the decode64 batch with ``tokens``
    new tokens per sequence per call, states updated in place in a 64-slot pool
    kept in ``state_dtype`` (fp32, or bf16 at rest with fp32 arithmetic)."""
    import torch

    from gated_deltanet_recurrence_rule_b200 import api, inputs

    w = inputs.WORKLOADS["decode64"]
    calls = max(args.decode_steps // tokens, 4)
    d = inputs.decode_inputs(w.batch, w.Hqk, w.Hv, w.D, steps=calls * tokens, dtype=w.dtype,
                             seed=rank_seed(w.seed, D.rank), init_std=w.init_std)

    def per_call(t):  # [calls*tokens, B, ...] -> [calls, B, tokens, ...]
        t = t.view(calls, tokens, *t.shape[1:])
        return t.transpose(1, 2).contiguous().to(dev)

    x = {n: per_call(d[n]) for n in ("q", "k", "v", "g", "beta")}
    sdt = {"fp32": torch.float32, "bf16": torch.bfloat16}[state_dtype]
    S = d["state"].to(sdt).to(dev)
    o = torch.empty((w.batch, tokens, w.Hv, w.D), dtype=torch.float32, device=dev)

    def run(n):
        for c in range(n):
            api.decode_tokens(x["q"][c], x["k"][c], x["v"][c], x["g"][c], x["beta"][c], S, o=o)

    run(min(calls, 4))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    run(calls)
    e1.record(stream)
    torch.cuda.synchronize()
    D.barrier()
    ms = D.max(e0.elapsed_time(e1), dev)
    state_bytes = w.batch * w.Hv * w.D * w.D * S.element_size()
    io_bytes = tokens * w.batch * (2 * w.Hqk * w.D * 2 + w.Hv * w.D * 2 + w.Hv * w.D * 4 + 2 * w.Hv * 4)
    per_call_bytes = 2 * state_bytes + io_bytes
    gbs = D.world * per_call_bytes * calls / (ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    kernel = ("decode_tokens_kernel" if state_dtype == "fp32" else
              "decode_one_bf16s_kernel" if tokens == 1 else "decode_tokens_bf16s_kernel")
    traffic_key = "decode_tokens" + ("" if tokens > 1 else "_1") + ("_bf16" if state_dtype == "bf16" else "")
    return {"value": D.world * w.batch * tokens * calls / (ms / 1e3), "unit": "tokens/s",
            "workload": f"decode64 with {tokens} tokens per sequence per call: B={w.batch}, "
                        f"Hqk={w.Hqk} Hv={w.Hv} D={w.D} bf16, {state_dtype} state pool of {w.batch} "
                        f"slots in place, {calls} calls",
            "state_dtype": state_dtype,
            "us_per_call": ms * 1e3 / calls,
            "roofline": {"bound": "hbm", "kernel": kernel, "achieved": gbs / D.world,
                         "peak": peak, "unit": "GB/s", "frac": gbs / D.world / peak,
                         "peak_source": f"{peak_src} hbm_gbs",
                         "algorithmic": f"{per_call_bytes} B per call (state read+write {2 * state_bytes} + io {io_bytes})",
                         "traffic": kernel_traffic(traffic_key, DECODE_SOURCES)},
            "gpu_launches": calls}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        # the oracle runs on the host; only rank 0 works, other ranks exit 0
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        D = Dist.__new__(Dist)
        D.rank, D.world, D.local_rank, D.dist = 0, 1, 0, None
        out = run_reference(args, D)
        print(json.dumps(out), flush=True)
        return 0
    D = Dist()
    try:
        out = run_ours(args, D)
        if D.rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        D.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
