#!/usr/bin/env python
"""Selective-scan (S6) layer-core throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl axon|reference]
                    [--workload NAME]

One step = one pass of the whole hot path over one batch of synthetic input:
the prefill (conv1d + SiLU + dt + selective recurrence + C/D epilogue + SiLU(z)
gate, returning the (conv_cache, ssm_state) pair) of the long-sequence workload
(B1 L65536 E2048 N16 K4, bf16 io, fp32 state: the largest of the five measured
workloads that fits one GPU), followed by one cached decode step on the
returned caches.  Throughput is counted in token x channel units: B*(L+1)*E
per step.  The other workloads' prefills are measured beside it (key
``workloads``), each with its own roofline fraction.

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent
sequences (different seeds); the path has no data exchange, so there is no
collective on the data path; the elapsed time is the max over ranks and the
value counts the units of all ranks (weak scaling).

Rank 0 prints ONE JSON line.  `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload instead (rank 0 only; other ranks exit 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from selective_state_space_52_b200 import workloads as W  # noqa: E402

METRIC = "selective-scan throughput (G token·channel/s) and % of HBM roofline, 1 B200"
UNIT = "G token·channel/s"
# Transcendental (MUFU) evaluations per token x channel: 16 decays exp(dt*A_n),
# SiLU(xc) (exp + reciprocal), softplus (exp + log), SiLU(z) (exp + reciprocal).
MUFU_PER_TOKEN_CH = 16 + 6
MUFU_LANES_PER_SM_CLK = 16
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# --------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def reduce_max(value: float, device) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def rank_seed(base: int, rank: int, k: int = 0) -> int:
    """Seeds of the independent per-rank problems (rank 0 == the single-GPU run)."""
    return base + 7919 * rank + 104729 * k


def rank_units(units_per_rank: int, world: int) -> int:
    return units_per_rank * world


# --------------------------------------------------------------- peaks / model
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "bf16_tflops": float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "source": "fallback"}


# float32 operations per token x channel of the layer core (conv 4 FMA, dt*u
# and 16 (dt A) products, 16 (dt u) B products, 16 state FMAs, 16 C.h FMAs,
# D u and the gate product): the FMA side of the combined roofline
FP32_OPS_PER_TOKEN_CH = 70


def measure_peaks_in_run(dev) -> dict:
    """The roofline's denominators measured in this run: the HBM copy rate
    (1 GiB copied, read + write bytes, best of 5), and the MUFU exp2 and float32
    FMA rates of this library's throughput probes (axon_peak_probe: 8 blocks of
    256 threads per SM, 8 independent chains per thread, best of 5)."""
    from selective_state_space_52_b200 import axon_ssm
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks = sms * 8
    out = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def best(fn, reps=5):
        fn()
        torch.cuda.synchronize(dev)
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream); fn(); b.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b) / 1e3)
        return min(ts)

    res = {"source": "measured in this run (bench.py measure_peaks_in_run)"}
    for kind, name, iters in ((0, "mufu_gops", 4096), (1, "ffma_gops", 16384)):
        secs = best(lambda: axon_ssm.axon_peak_probe(kind, out, blocks, iters))
        res[name] = blocks * 256 * 8 * iters / secs / 1e9
    src = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    secs = best(lambda: dst.copy_(src))
    res["hbm_copy_gbs"] = 2 * src.numel() / secs / 1e9
    del src, dst
    # the dense bf16 tensor rate as the library GEMM reaches it (a denominator only)
    n = 8192
    a = torch.randn(n, n, device=dev).to(torch.bfloat16)
    b = torch.randn(n, n, device=dev).to(torch.bfloat16)
    c = torch.empty(n, n, dtype=torch.bfloat16, device=dev)
    secs = best(lambda: torch.matmul(a, b, out=c))
    res["bf16_gemm_tflops"] = 2 * n ** 3 / secs / 1e12
    del a, b, c
    return res


def scan_model(wl) -> dict:
    """Algorithmic bytes and MUFU operations of one prefill launch."""
    s = 2 if wl.io == "bf16" else 4
    T = wl.B * wl.L * wl.E
    bytes_ = (4 * T * s                       # x, z, dt_raw read; y written
              + 2 * wl.B * wl.L * wl.N * s    # B, C read
              + wl.E * (wl.K + 3 + wl.N) * 4  # conv_w, conv_b, dt_bias, D, A_log
              + wl.B * wl.E * wl.N * 4        # ssm_state written
              + wl.B * (wl.K - 1) * wl.E * s)  # conv_cache written
    return {"bytes": bytes_, "mufu": MUFU_PER_TOKEN_CH * T, "token_ch": T}


def step_model(wl) -> dict:
    """Algorithmic bytes of one cached decode step (state and cache read + written)."""
    s = 2 if wl.io == "bf16" else 4
    BE = wl.B * wl.E
    bytes_ = (BE * (4 * s + 2 * (wl.K - 1) * s + 2 * wl.N * 4)
              + 2 * wl.B * wl.N * s + wl.E * (wl.K + 3 + wl.N) * 4)
    return {"bytes": bytes_, "mufu": MUFU_PER_TOKEN_CH * BE, "token_ch": BE}


# The sources each profiled kernel is built from: its own headers and the
# translation unit that plans and launches it.  A committed ncu figure counts
# only while these files are unchanged.
KERNEL_SOURCES = {
    "scan": ("axon_ssm.cu", "device_math.cuh", "scan_chunked.cuh", "scan_octo.cuh", "scan_qsplit.cuh",
             "scan_quad.cuh", "scan_seq.cuh"),
    "step": ("axon_ssm.cu", "device_math.cuh", "step.cuh"),
    "ssd": ("axon_ssd.cu", "device_math.cuh", "scan_chunked.cuh", "ssd.cuh", "tc_ops.cuh"),
    "gemm": ("axon_block.cu", "gemm_pair.cuh", "gemm_tc.cuh", "tc_ops.cuh"),
}


def kernel_source_hash(kernel_key: str = "scan") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_52_b200", "csrc")
    for fn in sorted(KERNEL_SOURCES[kernel_key]):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str, workload: str, units: int):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu summary,
    or None when no capture exists for the current kernel source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    ent = d.get(kernel_key, {}).get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel_key):
        return None
    per_unit = ent["dram_bytes"] / ent["units"]
    return per_unit * units


# --------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU during the timed region (NVML)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    self.h = h
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as ex:  # no NVML: report no samples rather than guess
            self.nv = None
            self.error = repr(ex)

    def _run(self):
        nv = self.nv
        while True:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception as ex:
                self.error = repr(ex)
            if self._stop.wait(self.period):
                break

    def start(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self) -> dict:
        if self._thr is not None:
            self._stop.set()
            self._thr.join()
        med = statistics.median(self.samples) if self.samples else None
        out = {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
               "samples": len(self.samples), "source": "nvml"}
        if self.error and not self.samples:
            out["error"] = self.error
        return out


# --------------------------------------------------------------- CPU oracle
def time_oracle(wl, inp, budget_s: float, block: int = 256, parallel: bool = False):
    """Time the fp64 oracle on the first channels of the workload until the
    budget is spent; returns (token_ch/s, token_ch done, seconds, channels,
    threads).  ``parallel`` runs the OpenMP build of the same source on all
    host cores (blocks of ``block`` channels per thread)."""
    import oracle
    threads = oracle.threads(parallel)
    blk = block * threads
    done_ch, t_total = 0, 0.0
    E = wl.E
    while done_ch < E and t_total < budget_s:
        e0, e1 = done_ch, min(E, done_ch + blk)
        sl = slice(e0, e1)
        args = [inp["x"][:, :, sl].contiguous(), inp["z"][:, :, sl].contiguous(),
                inp["dt_raw"][:, :, sl].contiguous(), inp["B"], inp["C"],
                inp["conv_w"][sl], inp["conv_b"][sl], inp["dt_bias"][sl], inp["A_log"][sl],
                inp["D"][sl]]
        t0 = time.perf_counter()
        oracle.scan_fwd(*args, parallel=parallel)
        t_total += time.perf_counter() - t0
        done_ch = e1
    units = done_ch * wl.B * wl.L
    return units / t_total, units, t_total, done_ch, threads


def cpu_baselines(wl, inp, budget_s: float) -> dict:
    """The oracle on one host core and (its OpenMP build) on all of them."""
    import oracle
    oracle.build()
    oracle.build(openmp=True)
    rate1, _, secs1, ch1, _ = time_oracle(wl, inp, budget_s, block=64)
    rate, _, secs, ch, thr = time_oracle(wl, inp, budget_s, block=16, parallel=True)
    return {"value": rate / 1e9, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{ch} of {wl.E} channels x {wl.L} tokens (prefill), {secs:.1f} s, fp64 C oracle, "
                      f"OpenMP build over channels on {thr} host threads",
            "single_core": {"value": rate1 / 1e9, "unit": UNIT, "cores": 1,
                            "sample": f"{ch1} of {wl.E} channels x {wl.L} tokens (prefill), {secs1:.1f} s, "
                                      "fp64 C oracle, single thread"}}


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = W.make_inputs(wl)
    import oracle
    oracle.build(openmp=True)
    per_step_budget = max(0.5, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    channels = None
    threads = 1
    rates = []
    for i in range(args.warmup + args.steps):
        rate, units, secs, ch, threads = time_oracle(wl, inp, per_step_budget, block=16, parallel=True)
        channels = ch
        if i >= args.warmup:
            rates.append((units, secs))
    units = sum(u for u, _ in rates)
    secs = sum(s for _, s in rates)
    value = units / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * secs / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(wl), "sample": f"first {channels} channels x {wl.L} tokens per step"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{channels} of {wl.E} channels x {wl.L} tokens per step, "
                                   f"fp64 C oracle, OpenMP build over channels on {threads} host threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_decode(dev, steps: int = 512, distinct: int = 8) -> dict:
    """Cached decode on the decode workload's shapes (64 sequences, E=7680, bf16):
    per-step time cold (L2 flushed before every step, events around each step)
    and warm (all steps back to back in one CUDA graph; the 34 MB of state and
    cache may then stay in the 126 MB L2)."""
    from selective_state_space_52_b200 import axon_ssm
    wl = W.WORKLOAD_BY_NAME["decode"]
    params = {k: v.to(dev) for k, v in W.make_params(wl).items()}
    st = {k: v.to(dev) for k, v in W.make_state(wl).items()}
    toks = {k: v.to(dev) for k, v in W.make_decode_inputs(wl, distinct).items()}
    cache = (st["conv_cache"], st["ssm_state"])
    y = torch.empty(wl.B, wl.E, dtype=wl.torch_io, device=dev)
    model = step_model(wl)
    stream = torch.cuda.current_stream(dev)

    def one(i):
        axon_ssm.step(*(toks[k][i % distinct] for k in ("x", "z", "dt_raw", "B", "C")), params, cache, y=y)

    for i in range(8):
        one(i)
    # read (not write) a buffer twice the L2 size before every step: the L2 then
    # holds clean lines only, so the step does not pay for another buffer's write-back
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    cold = []
    for i in range(32):
        flush.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream); one(i); b.record(stream)
        torch.cuda.synchronize(dev)
        cold.append(a.elapsed_time(b))
    cold_ms = statistics.median(cold[4:])
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        one(0)
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    with torch.cuda.graph(g):
        for i in range(steps):
            one(i)
    g.replay()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream); g.replay(); b.record(stream)
    torch.cuda.synchronize(dev)
    warm_ms = a.elapsed_time(b) / steps
    del g
    peaks = measured_peaks()
    return {"workload": "decode: B64 E7680 N16 K4, bf16 io, fp32 state",
            "algorithmic_bytes": model["bytes"],
            "cold_us": cold_ms * 1e3, "cold_gbs": model["bytes"] / (cold_ms / 1e3) / 1e9,
            "cold_frac_hbm": model["bytes"] / (cold_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "warm_us": warm_ms * 1e3, "warm_gbs": model["bytes"] / (warm_ms / 1e3) / 1e9,
            "warm_note": f"{steps} steps in one CUDA graph; state + cache (34 MB) can stay in L2",
            "token_ch_per_s_warm": wl.B * wl.E / (warm_ms / 1e3) / 1e9}


def bench_zoh_prefill(wl, sets, params, out, ws, dev, launches: int = 20) -> dict:
    """The same prefill with the exact zero-order-hold discretisation (the
    Axon-SSM page's ZOH form): mean event time of `launches` prefill calls."""
    from selective_state_space_52_b200 import axon_ssm
    stream = torch.cuda.current_stream(dev)
    n_sets = len(sets)

    def run(i):
        s = sets[i % n_sets]
        axon_ssm.scan_fwd(s["x"], s["z"], s["dt_raw"], s["B"], s["C"], params, None, out=out,
                          workspace=ws, discretization="zoh")

    for i in range(3):
        run(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
    torch.cuda.synchronize(dev)
    for i, (a, b) in enumerate(ev):
        a.record(stream); run(i); b.record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    T = wl.B * wl.L * wl.E
    return {"kernel_ms": ms, "value": T / (ms / 1e3) / 1e9, "unit": UNIT, "launches": launches}


def bench_block(dev, launches: int = 50, warmup: int = 20) -> dict:
    """The whole Axon-SSM layer (input projection, conv stage, projection to
    dt/B/C, fused scan, output projection; axon_ssm_block_fwd) on the Bit-Axon
    layer (B1 L2048 D2560 E7680, bf16): mean (and median) event time of
    `launches` calls after `warmup` untimed ones (a call is about 0.6 ms: the
    warm-up also brings the clocks up when the layer runs alone)."""
    from selective_state_space_52_b200 import axon_ssm
    bw = W.BLOCK_WORKLOAD_BY_NAME["bit_axon_block"]
    inp = {k: v.to(dev) for k, v in W.make_block_inputs(bw).items()}
    weights = {k: inp[k] for k in axon_ssm.WEIGHT_KEYS}
    params = {k: inp[k] for k in axon_ssm.PARAM_KEYS}
    M, Dm, E, N = bw.B * bw.L, bw.Dm, bw.E, bw.N
    out = torch.empty(bw.B, bw.L, Dm, dtype=torch.bfloat16, device=dev)
    cc = torch.empty(bw.B, bw.K - 1, E, dtype=torch.bfloat16, device=dev)
    ss = torch.empty(bw.B, E, N, dtype=torch.float32, device=dev)
    ws = torch.empty(axon_ssm.axon_ssm_block_workspace_bytes(bw.B, bw.L, Dm, E, N, bw.K), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def call():
        axon_ssm.block_fwd(inp["X"], weights, params, None, out=(out, cc, ss), workspace=ws, check=False)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(launches):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream); call(); b.record(stream)
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b))
        if axon_ssm.block_error_flag(ws) != 0:
            raise RuntimeError("axon_ssm_block_fwd: a wait of a projection GEMM gave up")
    ms = statistics.mean(times)
    ms_median = statistics.median(times)
    flops = 2 * M * (Dm * 2 * E + E * (E + 2 * N) + E * Dm)
    peaks = measured_peaks()
    return {"workload": "Axon-SSM layer: B1 L2048 D2560 E7680 N16 K4, bf16, weights and input resident",
            "ms": ms, "ms_median": ms_median, "calls": launches, "tokens_per_s": M / (ms / 1e3),
            "gemm_flops": flops, "gemm_tflops_over_layer_time": flops / (ms / 1e3) / 1e12,
            "bf16_peak_tflops": peaks.get("bf16_tflops"),
            "note": "three bf16 GEMM launches on this library's tcgen05 kernels (x|z, dt|B|C, out; fp32 "
                    "accumulate; CTA pairs, the last two with the stream-K split) + conv stage + fused scan"}


def bench_time_split(wl, s, params, dev, P: int = 4, launches: int = 10) -> dict:
    """The time-split protocol (shard.py) on the bench workload's sequence cut
    into P slices, all on this one GPU: the whole protocol, and one rank's own
    work (slice 1: scan from a zero state + dt sum, then fold + scan again),
    which is what each of P GPUs would run besides the two small exchanges."""
    from selective_state_space_52_b200 import shard
    L = wl.L
    cut = [L * r // P for r in range(P + 1)]
    slices = [{k: s[k][:, cut[r]:cut[r + 1]].contiguous() for k in ("x", "z", "dt_raw", "B", "C")}
              for r in range(P)]
    ops = shard.cuda_ops()
    K = wl.K
    stream = torch.cuda.current_stream(dev)

    def whole():
        shard.sliced_scan_local(slices, params, None, ops)

    tails = [shard.slice_tail(sl["x"], K) for sl in slices]
    firsts = [shard.first_pass(r, sl, params, tails[r - 1] if r else None, None, ops) for r, sl in enumerate(slices)]
    h_all = torch.stack([f[2] for f in firsts])
    dts_all = torch.stack([f[3] for f in firsts])

    def one_rank():
        shard.first_pass(1, slices[1], params, tails[0], None, ops)
        shard.second_pass(1, slices[1], params, tails[0], h_all, dts_all, ops)

    res = {}
    for name, fn in (("protocol_ms", whole), ("one_rank_ms", one_rank)):
        for _ in range(2):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(launches):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = a.elapsed_time(b) / launches
    exch = P * (wl.B * wl.E * (wl.N + 1) * 4 + wl.B * (wl.K - 1) * wl.E * 2)
    return {"workload": f"prefill of B{wl.B} L{L} E{wl.E} N{wl.N} K{wl.K} {wl.io}, cut into {P} slices "
                        f"of {L // P} tokens", "slices": P,
            **res, "exchange_bytes_per_rank": exch,
            "note": "all slices on one GPU (one GPU per call here); on P GPUs each rank runs one_rank_ms "
                    "of work plus two all-gathers of the listed bytes"}


def bench_ssd(dev, launches: int = 20) -> dict:
    """The Mamba-2 (SSD) layer core (axon_ssd_scan_fwd) on the Mamba-2 block's
    heads: B1 L4096, 64 heads of 64, d_state 128, bf16; mean event time, with
    its HBM and tensor-core rooflines."""
    from selective_state_space_52_b200 import axon_ssm
    sw = W.SSD_WORKLOAD_BY_NAME["mamba2_ssd"]
    inp = {k: v.to(dev) for k, v in W.make_ssd_inputs(sw).items()}
    params = {k: inp[k] for k in ("dt_bias", "A_log", "D")}
    y = torch.empty_like(inp["x"])
    h = torch.empty(sw.B, sw.H, sw.P, sw.N, dtype=torch.float32, device=dev)
    ws = torch.empty(max(axon_ssm.axon_ssd_workspace_bytes(sw.B, sw.L, sw.H, sw.P, sw.N), 16),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call():
        axon_ssm.ssd_scan(inp["x"], inp["dt_raw"], inp["B"], inp["C"], params, None, out=(y, h), workspace=ws,
                          check=False)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    times = []
    for _ in range(launches):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream); call(); b.record(stream)
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b))
        if axon_ssm.ssd_error_flag(ws) != 0:
            raise RuntimeError("axon_ssd_scan_fwd: a wait for a tensor-core product gave up")
    ms = statistics.median(times)
    Q, P, N, H, L, B = 128, sw.P, sw.N, sw.H, sw.L, sw.B     # Q: tokens per chunk of the kernels
    nC = (L + Q - 1) // Q
    # per chunk: C B^T once; per chunk and head: exp(acum) C S_in, the causal
    # half of the masked Gram times x, and x^T (w B)
    flops = B * nC * (2 * Q * Q * N + H * (2 * Q * N * P + Q * Q * P + 2 * P * N * Q))
    nbytes = B * L * H * P * 2 * 2 + B * L * (H * 2 + 2 * N * 2) + B * H * P * N * 4
    peaks = measured_peaks()
    hbm = nbytes / (ms / 1e3) / 1e9
    tfl = flops / (ms / 1e3) / 1e12
    return {"workload": "Mamba-2 (SSD) core: B1 L4096, 64 heads x 64, d_state 128, bf16; L2 flushed",
            "ms": ms, "algorithmic_bytes": nbytes, "flops": flops,
            "hbm": {"achieved": hbm, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": hbm / peaks["hbm_gbs"]},
            "tensor": {"achieved": tfl, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                       "frac": tfl / peaks["bf16_tflops"],
                       "note": "bf16 tcgen05 MMAs (M = 128, float32 accumulators in tensor memory); the "
                               "carried-state product runs twice (hi and lo parts) and C B^T once per head, "
                               "both counted once"},
            "token_head_per_s": B * L * H / (ms / 1e3)}


def bench_prefill_workload(wl, dev, launches: int = 20) -> dict:
    """One workload's prefill alone (the library's own plan, inputs resident):
    CUDA-event mean over `launches` calls with the L2 flushed (a buffer of
    twice its size written) before each, and its MUFU and HBM rooflines."""
    from selective_state_space_52_b200 import axon_ssm
    inp = {k: v.to(dev) for k, v in W.make_inputs(wl).items()}
    params = {k: inp[k] for k in axon_ssm.PARAM_KEYS}
    io_code = axon_ssm.AXON_BF16 if wl.io == "bf16" else axon_ssm.AXON_F32
    y = torch.empty(wl.B, wl.L, wl.E, dtype=wl.torch_io, device=dev)
    cc = torch.empty(wl.B, wl.K - 1, wl.E, dtype=wl.torch_io, device=dev)
    ss = torch.empty(wl.B, wl.E, wl.N, dtype=torch.float32, device=dev)
    ws = torch.empty(max(axon_ssm.axon_ssm_scan_workspace_bytes(wl.B, wl.L, wl.E, wl.N, wl.K, io_code), 16),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call():
        axon_ssm.scan_fwd(inp["x"], inp["z"], inp["dt_raw"], inp["B"], inp["C"], params, None,
                          out=(y, cc, ss), workspace=ws)

    for _ in range(3):
        call()
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    times = []
    for _ in range(launches):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream); call(); b.record(stream)
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b))
    ms = statistics.mean(times)
    peaks = measured_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mufu_peak = sms * MUFU_LANES_PER_SM_CLK * peaks["sm_max_mhz"] * 1e6 / 1e9
    m = scan_model(wl)
    mufu = m["mufu"] / (ms / 1e3) / 1e9
    hbm = m["bytes"] / (ms / 1e3) / 1e9
    return {"shape": f"B{wl.B} L{wl.L} E{wl.E} {wl.io}", "prefill_us": ms * 1e3,
            "value": m["token_ch"] / (ms / 1e3) / 1e9, "unit": UNIT,
            "mufu_frac": mufu / mufu_peak, "hbm_gbs": hbm, "hbm_frac": hbm / peaks["hbm_gbs"],
            "launches": axon_ssm.axon_ssm_scan_launch_count(wl.B, wl.L, wl.E, wl.N, wl.K, io_code),
            "note": "L2 flushed before every call; mufu_frac = 22 transcendentals per token x channel "
                    "over the MUFU peak"}


def run_single_kernel(args, wl, dev) -> dict:
    """The prefill of `wl` (library plan) or one projection GEMM, 3 warm-up
    calls and one timed call: a short program for profiling one kernel."""
    from selective_state_space_52_b200 import axon_ssm
    stream = torch.cuda.current_stream(dev)
    if args.gemm_only:
        M, N, K = (int(v) for v in args.gemm_only.split(","))
        g = torch.Generator().manual_seed(M + N + K)
        A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(dev)
        Wt = (torch.randn(K, N, generator=g) / K ** 0.5).to(torch.bfloat16).to(dev)
        C = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        gws = torch.empty(axon_ssm.axon_gemm_workspace_bytes(), dtype=torch.uint8, device=dev)

        def call():
            # the automatic tiling with the stream-K scratch, as the layer runs it
            axon_ssm.gemm_bf16(A, Wt, out=C, check=False, workspace=gws)
        what = {"kernel": "axon_gemm_bf16_plan (automatic, with stream-K scratch)", "M": M, "N": N, "K": K}
        flops = 2 * M * N * K
    else:
        inp = {k: v.to(dev) for k, v in W.make_inputs(wl).items()}
        params = {k: inp[k] for k in axon_ssm.PARAM_KEYS}
        out = (torch.empty_like(inp["x"]), torch.empty(wl.B, wl.K - 1, wl.E, dtype=wl.torch_io, device=dev),
               torch.empty(wl.B, wl.E, wl.N, dtype=torch.float32, device=dev))
        io_code = axon_ssm.AXON_BF16 if wl.io == "bf16" else axon_ssm.AXON_F32
        ws = torch.empty(max(axon_ssm.axon_ssm_scan_workspace_bytes(wl.B, wl.L, wl.E, wl.N, wl.K, io_code), 16),
                         dtype=torch.uint8, device=dev)

        def call():
            axon_ssm.scan_fwd(inp["x"], inp["z"], inp["dt_raw"], inp["B"], inp["C"], params, None, out=out,
                              workspace=ws)
        what = {"kernel": "prefill", "workload": workload_desc(wl)}
        flops = None
    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream); call(); b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b)
    what["us"] = ms * 1e3
    if flops:
        what["tflops"] = flops / (ms / 1e3) / 1e12
    return what


def workload_desc(wl) -> str:
    return (f"{wl.name}: B{wl.B} L{wl.L} E{wl.E} N{wl.N} K{wl.K}, {wl.io} io, fp32 state; "
            "step = prefill + 1 cached decode token")


# --------------------------------------------------------------- GPU arm
def run_axon(args, wl):
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU for --impl axon")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    from selective_state_space_52_b200 import axon_ssm

    io = wl.torch_io
    io_code = axon_ssm.AXON_BF16 if wl.io == "bf16" else axon_ssm.AXON_F32
    B, L, E, N, K = wl.B, wl.L, wl.E, wl.N, wl.K

    # inputs: several independent sets so that consecutive steps do not hit in L2
    params_cpu = W.make_params(wl, g=torch.Generator().manual_seed(rank_seed(wl.seed, rank)))
    params = {k: v.to(dev) for k, v in params_cpu.items()}
    set_bytes = 3 * B * L * E * io.itemsize
    n_sets = max(2, math.ceil(2 * L2_BYTES / max(1, set_bytes)) + 1)
    n_sets = min(n_sets, 8)
    sets = []
    for k in range(n_sets):
        g = torch.Generator().manual_seed(rank_seed(wl.seed + 1000, rank, k))
        sets.append({kk: v.to(dev) for kk, v in W.make_sequence(wl, g=g).items()})
    tok = {kk: v[0].to(dev) for kk, v in W.make_decode_inputs(
        wl, 1, g=torch.Generator().manual_seed(rank_seed(wl.seed + 3000, rank))).items()}

    y = torch.empty(B, L, E, dtype=io, device=dev)
    cc = torch.empty(B, K - 1, E, dtype=io, device=dev)
    ss = torch.empty(B, E, N, dtype=torch.float32, device=dev)
    y_tok = torch.empty(B, E, dtype=io, device=dev)
    ws_bytes = axon_ssm.axon_ssm_scan_workspace_bytes(B, L, E, N, K, io_code)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    scan_launches = axon_ssm.axon_ssm_scan_launch_count(B, L, E, N, K, io_code)
    stream = torch.cuda.current_stream(dev)

    def one_step(s):
        axon_ssm.scan_fwd(s["x"], s["z"], s["dt_raw"], s["B"], s["C"], params, None,
                          out=(y, cc, ss), workspace=ws)
        axon_ssm.step(tok["x"], tok["z"], tok["dt_raw"], tok["B"], tok["C"], params, (cc, ss), y=y_tok)

    for i in range(args.warmup):
        one_step(sets[i % n_sets])
    torch.cuda.synchronize(dev)

    # ---- device-resident timed region: exactly K steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    barrier(dev)
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start.record(stream)
    for i in range(args.steps):
        s = sets[i % n_sets]
        e0, e1, e2 = ev[i]
        e0.record(stream)
        axon_ssm.scan_fwd(s["x"], s["z"], s["dt_raw"], s["B"], s["C"], params, None,
                          out=(y, cc, ss), workspace=ws)
        e1.record(stream)
        axon_ssm.step(tok["x"], tok["z"], tok["dt_raw"], tok["B"], tok["C"], params, (cc, ss), y=y_tok)
        e2.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(dev)
    ms_local = t_start.elapsed_time(t_end)
    ms = reduce_max(ms_local, dev)
    scan_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    step_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)

    units_step = B * (L + 1) * E
    value = rank_units(units_step, world) * args.steps / (ms / 1e3) / 1e9

    # ---- end to end through the public API with host buffers (pinned).  The
    # steps are pipelined the way a serving loop runs them: step i's upload
    # (its own stream) overlaps step i-1's compute and download (another
    # stream); device inputs, outputs and caches are double-buffered.
    host = {k: v.cpu().pin_memory() for k, v in sets[0].items()}
    host_tok = {k: v.cpu().pin_memory() for k, v in tok.items()}
    nbuf = 2
    dev_in = [{k: torch.empty_like(v) for k, v in sets[0].items()} for _ in range(nbuf)]
    dev_tok = [{k: torch.empty_like(v) for k, v in tok.items()} for _ in range(nbuf)]
    y_dev = [y] + [torch.empty_like(y) for _ in range(nbuf - 1)]
    ytok_dev = [y_tok] + [torch.empty_like(y_tok) for _ in range(nbuf - 1)]
    caches = [(cc, ss)] + [(torch.empty_like(cc), torch.empty_like(ss)) for _ in range(nbuf - 1)]
    y_host = [torch.empty(y.shape, dtype=io).pin_memory() for _ in range(nbuf)]
    ytok_host = [torch.empty(y_tok.shape, dtype=io).pin_memory() for _ in range(nbuf)]
    h2d = sum(v.numel() * v.element_size() for v in host.values()) + \
        sum(v.numel() * v.element_size() for v in host_tok.values())
    d2h = y_host[0].numel() * y_host[0].element_size() + ytok_host[0].numel() * ytok_host[0].element_size()
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {name: [torch.cuda.Event() for _ in range(nbuf)] for name in ("in_ready", "in_free", "out_ready", "out_free")}

    def e2e_step(i):
        k = i % nbuf
        with torch.cuda.stream(up):
            up.wait_event(ev["in_free"][k])          # step i-2's compute is done with these buffers
            for kk in host:
                dev_in[k][kk].copy_(host[kk], non_blocking=True)
            for kk in host_tok:
                dev_tok[k][kk].copy_(host_tok[kk], non_blocking=True)
            ev["in_ready"][k].record(up)
        stream.wait_event(ev["in_ready"][k])
        stream.wait_event(ev["out_free"][k])         # step i-2's download has read y_dev[k]
        d, t = dev_in[k], dev_tok[k]
        axon_ssm.scan_fwd(d["x"], d["z"], d["dt_raw"], d["B"], d["C"], params, None,
                          out=(y_dev[k], *caches[k]), workspace=ws)
        axon_ssm.step(t["x"], t["z"], t["dt_raw"], t["B"], t["C"], params, caches[k], y=ytok_dev[k])
        ev["in_free"][k].record(stream)
        ev["out_ready"][k].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev["out_ready"][k])
            y_host[k].copy_(y_dev[k], non_blocking=True)
            ytok_host[k].copy_(ytok_dev[k], non_blocking=True)
            ev["out_free"][k].record(down)

    e2e_steps = max(3, min(args.steps, 50))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(ev["out_free"][(e2e_steps - 1) % nbuf])   # the last download is inside the region
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(a.elapsed_time(b), dev)
    e2e_value = rank_units(units_step, world) * e2e_steps / (e2e_ms / 1e3) / 1e9

    # ---- roofline of the dominant kernel (the prefill scan)
    peaks = measured_peaks()
    sm = scan_model(wl)
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    mufu_peak = sms * MUFU_LANES_PER_SM_CLK * peaks["sm_max_mhz"] * 1e6 / 1e9   # Gop/s
    mufu_ach = sm["mufu"] / (scan_ms / 1e3) / 1e9
    hbm_ach = sm["bytes"] / (scan_ms / 1e3) / 1e9
    traffic = ncu_traffic("scan", wl.name, sm["token_ch"])
    stm = step_model(wl)
    pin = measure_peaks_in_run(dev)
    # the combined roofline with this run's peaks: the slowest of the bytes,
    # the MUFU ops and the float32 ops at their measured rates
    t_roof = {"hbm": sm["bytes"] / (pin["hbm_copy_gbs"] * 1e9),
              "mufu": sm["mufu"] / (pin["mufu_gops"] * 1e9),
              "fp32": FP32_OPS_PER_TOKEN_CH * sm["token_ch"] / (pin["ffma_gops"] * 1e9)}
    bound_in_run = max(t_roof, key=t_roof.get)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": workload_desc(wl), "io_dtype": wl.io,
                   "l2": f"{n_sets} rotating input sets of {set_bytes / 1e6:.0f} MB "
                         f"({n_sets * set_bytes / 1e6:.0f} MB > 126 MB L2)",
                   "parallelism": f"dp{world} (independent sequences per GPU, no collective)"},
        "roofline": {"bound": "alu", "achieved": mufu_ach, "peak": mufu_peak, "unit": "Gop/s",
                     "frac": mufu_ach / mufu_peak, "traffic": traffic,
                     "kernel": "prefill scan (MUFU transcendentals: 22 per token x channel)",
                     "peak_source": f"{sms} SMs x {MUFU_LANES_PER_SM_CLK} MUFU/clk x "
                                    f"{peaks['sm_max_mhz']:.0f} MHz",
                     "kernel_ms": scan_ms, "algorithmic_bytes": sm["bytes"],
                     "hbm": {"achieved": hbm_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": hbm_ach / peaks["hbm_gbs"],
                             "peak_source": peaks["source"]},
                     "in_run": {"bound": bound_in_run, "frac": t_roof[bound_in_run] / (scan_ms / 1e3),
                                "roofline_us": {k: v * 1e6 for k, v in t_roof.items()},
                                "note": "max(algorithmic bytes / HBM copy, 22 MUFU ops / MUFU rate, "
                                        f"{FP32_OPS_PER_TOKEN_CH} FP32 ops / FFMA rate) per token x channel, "
                                        "each rate measured in this run (peaks_in_run)"}},
        "peaks_in_run": pin,
        "decode_step": {"us": step_ms * 1e3, "algorithmic_bytes": stm["bytes"],
                        "hbm_gbs": stm["bytes"] / (step_ms / 1e3) / 1e9},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipeline": "pinned host buffers; step i's upload overlaps step i-1's compute and "
                            "download (separate streams, two device buffer sets)"},
        "clocks": clk,
        "gpu_launches": args.steps * (scan_launches + 1),
    }

    if not args.no_workloads and world == 1:
        line["workloads"] = {w.name: bench_prefill_workload(w, dev) for w in W.WORKLOADS
                             if w.name not in ("tiny_f32", wl.name)}
    if not args.no_decode_bench:
        line["decode"] = bench_decode(dev)
        line["decode"]["cold_frac_hbm_copy_in_run"] = (line["decode"]["algorithmic_bytes"] /
                                                       (line["decode"]["cold_us"] / 1e6) / 1e9 /
                                                       pin["hbm_copy_gbs"])
        line["prefill_zoh"] = bench_zoh_prefill(wl, sets, params, (y, cc, ss), ws, dev)
    if not args.no_block_bench and world == 1:
        line["block"] = bench_block(dev)
        line["block"]["gemm_frac_of_bf16_gemm_in_run"] = (line["block"]["gemm_tflops_over_layer_time"] /
                                                          pin["bf16_gemm_tflops"])
        line["time_split"] = bench_time_split(wl, sets[0], params, dev)
        line["ssd"] = bench_ssd(dev)
        line["ssd"]["tensor"]["frac_of_bf16_gemm_in_run"] = (line["ssd"]["tensor"]["achieved"] /
                                                             pin["bf16_gemm_tflops"])
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = {**params_cpu, **{k: v.cpu() for k, v in sets[0].items()}}
        line["cpu_baseline"] = cpu_baselines(wl, inp_cpu, args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier(dev)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["axon", "reference"], default="axon")
    ap.add_argument("--workload", default="long_seq", choices=[w.name for w in W.WORKLOADS])
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode-bench", action="store_true",
                    help="skip the separate cached-decode measurement (decode workload shapes)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the prefills of the other measured workloads")
    ap.add_argument("--no-block-bench", action="store_true",
                    help="skip the whole-layer measurement (input/output projections around the scan)")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the cached-decode measurement and print it as one JSON line "
                         "(for profiling the step kernel alone)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the workload's prefill (library plan): 3 warm-up calls and one timed call, "
                         "printed as one JSON line (for profiling the prefill kernel alone)")
    ap.add_argument("--gemm-only", default=None, metavar="M,N,K",
                    help="run only the projection GEMM (axon_gemm_bf16) on random bf16 operands of this shape: "
                         "3 warm-up calls and one timed call (for profiling it alone)")
    ap.add_argument("--ssd-only", action="store_true",
                    help="run only the Mamba-2 (SSD) layer-core measurement and print it as one JSON line "
                         "(for profiling its kernels alone)")
    ap.add_argument("--block-only", action="store_true",
                    help="run only the whole-layer measurement (key block) and print it as one JSON line "
                         "(for profiling the layer's kernels alone)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)     # at least 3 untimed warm-up steps
    wl = W.WORKLOAD_BY_NAME[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.decode_only:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA GPU for --decode-only")
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps({"decode": bench_decode(dev)}), flush=True)
        return 0
    if args.prefill_only or args.gemm_only:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA GPU for --prefill-only / --gemm-only")
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps(run_single_kernel(args, wl, dev)), flush=True)
        return 0
    if args.ssd_only:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA GPU for --ssd-only")
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps({"ssd": bench_ssd(dev)}), flush=True)
        return 0
    if args.block_only:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA GPU for --block-only")
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps({"block": bench_block(dev)}), flush=True)
        return 0
    return run_axon(args, wl)


if __name__ == "__main__":
    sys.exit(main())
