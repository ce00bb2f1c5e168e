"""Throughput of the ConvRot W8A8 INT8 linear on B200.

One step = one whole pass of the hot path over one batch: rotate + quantise
the bf16 activations, int8 GEMM, dequantise with bias to bf16 (the weights
are packed once, offline, as the pages' checkpoints are).  The headline
workload is the full 768p projection, M = 38656 tokens, K = N = 5376,
Hadamard block 128.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The default run prints one JSON line: the headline (K back-to-back steps),
each kernel of the step timed in its own back-to-back loop, a sustained leg
(the same step for at least two seconds, under the power cap), the end-to-end
leg through host buffers, the oracle's CPU baseline, and -- on one GPU -- a
`configs` object with the other workloads (the tiny and 4096-token
projections, the 768p MLP pair, the 42-head Q K^T GEMM and int8 attention),
each with its roofline fraction and its own CPU baseline.

Multi-GPU (torchrun): every rank runs its own full batch (token rows are
independent; no collective on the data path), value = all ranks' work / the
slowest rank's time.  `--impl reference` times the CPU oracle on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ConvRot W8A8 linear TOPS at M=38656,K=N=5376 and % of B200 INT8 peak"
UNIT = "TOPS"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
GEMM_PROFILE = os.path.join(ROOT, "profiles", "linear_fused_proj_m38656_k5376_n5376.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "w8a8_int8_quantized_block_b200", "csrc", f)
                  for f in ("linear_fused.cu", "gemm_core.cuh", "quant_core.cuh", "ptx.cuh", "kernels.h")]
INT8_PER_BF16 = 2.0  # nominal dense ratio of 8-bit to bf16 tensor throughput (4.5 vs 2.25 PFLOP/s)
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_SUSTAINED = 6650.0, 1590.0, 1400.0
L2_FLUSH_BYTES = 256 << 20  # written between timed calls of workloads that fit in the 126 MB L2


REGULAR = 0x10000  # the C ABI's CONVROT_HADAMARD_REGULAR flag on a block value
BLOCK_CHOICES = {"64": 64, "128": 128, "256": 256,
                 "reg16": REGULAR | 16, "reg64": REGULAR | 64, "reg256": REGULAR | 256}


def workload(args):
    """The 768p projection with the chosen rotation (the inputs do not change)."""
    import dataclasses
    from w8a8_int8_quantized_block_b200 import workloads as W
    spec = W.PROJ_768P
    if args.block == "128":
        return spec
    return dataclasses.replace(spec, block=BLOCK_CHOICES[args.block], name=f"{spec.name}_block{args.block}")


def oracle_block(block: int):
    """(b, regular) of a block value, as the oracle takes them."""
    n = block & ~REGULAR
    return (n if n > 1 else 1), bool(block & REGULAR)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-seconds", type=float, default=60.0,
                    help="CPU time budget of the whole --impl reference run (warm-up + timed steps)")
    ap.add_argument("--block", choices=sorted(BLOCK_CHOICES), default="128",
                    help="rotation of the step: Sylvester H_b (64, 128, 256) or the regular H_4^(x)k "
                         "(reg16, reg64, reg256); the headline is 128")
    ap.add_argument("--workload", choices=["proj", "mlp", "attention"], default="proj",
                    help="proj: the 768p projection (the headline); mlp: the 768p MLP, up 5376 -> 21504 with "
                         "GELU, then down, timed by both routes of the activation (see --mlp-route); "
                         "attention: int8 attention over 42 heads of 8192 tokens, head dim 128")
    ap.add_argument("--heads", type=int, default=None,
                    help="attention workload only: number of heads (default 42; fewer for small profiling runs)")
    ap.add_argument("--mlp-route", choices=["prologue", "epilogue"], default="prologue",
                    help="the route the mlp line's value is for: GELU as the down projection's prologue "
                         "(convrot_linear_act) or in the up projection's epilogue; both are timed")
    ap.add_argument("--context-parallel", action="store_true",
                    help="strong scaling: the 38656 tokens split across the ranks, each step the rank's linear "
                         "then an NCCL all-gather of the bf16 rows so every rank holds the whole output")
    ap.add_argument("--rows", type=int, default=None,
                    help="with --kernel-only: only the first ROWS token rows of the projection (a smaller case "
                         "of the same workload, for detailed profiler captures)")
    ap.add_argument("--kernel-only", choices=["fused", "quant", "gemm", "bmm", "mlp-up", "mlp-down", "act"],
                    default=None,
                    help="set up, then launch only this kernel --warmup + --steps times and exit "
                         "(for profiler captures; prints no result line).  bmm: the 42-head Q K^T GEMM "
                         "(--heads for fewer); mlp-up: the MLP's up projection (one kernel, 5376 -> 21504, GELU "
                         "epilogue) on --rows rows; mlp-down: its down projection GEMM (K = 21504); act: the "
                         "GELU prologue quantiser of that projection")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' legs (the configs object of the default line)")
    ap.add_argument("--sustained-seconds", type=float, default=2.0,
                    help="length of the sustained leg (the headline step repeated under the power cap)")
    ap.add_argument("--quant-launches", type=int, default=1000,
                    help="back-to-back launches of the standalone quantiser in its own timed loop")
    return ap.parse_args()


def peaks():
    """(hbm GB/s, bf16 burst TFLOP/s, bf16 sustained TFLOP/s, source)."""
    try:
        p = json.load(open(PEAKS_FILE))
        bf16 = float(p["bf16_tflops"])
        return float(p["hbm_gbs"]), bf16, float(p.get("bf16_tflops_sustained", bf16)), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_SUSTAINED, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the one-kernel linear from the committed ncu
    summary, or None when the kernel sources changed since it was taken."""
    try:
        kv = {}
        for line in open(GEMM_PROFILE):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("kernel_sources_sha256_16") != kernel_hash():
            return None
        return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """Largest value over all ranks (every rank must call it, in the same order)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tops(ops_per_step: float, steps: int, world: int, slowest_rank_s: float) -> float:
    """Whole-job throughput under weak scaling: every rank runs the full
    per-rank workload, so the job does world * ops_per_step * steps in the
    slowest rank's time."""
    return world * ops_per_step * steps / slowest_rank_s / 1e12


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (the
    counters nvidia-smi reads) while the timed region runs."""

    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
             0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, cuda_index: int, period_s: float = 0.02):
        self.cuda_index, self.period, self.samples, self.err = cuda_index, period_s, [], None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._match_handle(pynvml)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception as e:  # no NVML: report it, do not fail the run
            self.err = f"{type(e).__name__}: {e}"
        return self

    def _match_handle(self, nv):
        """NVML handle of the CUDA device (matched by UUID: CUDA_VISIBLE_DEVICES
        may renumber devices)."""
        import torch
        want = str(torch.cuda.get_device_properties(self.cuda_index).uuid).lower().replace("gpu-", "")
        for i in range(nv.nvmlDeviceGetCount()):
            h = nv.nvmlDeviceGetHandleByIndex(i)
            u = nv.nvmlDeviceGetUUID(h)
            u = (u.decode() if isinstance(u, bytes) else u).lower().replace("gpu-", "")
            if u == want:
                return h
        return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _run(self):
        nv, h = self._nv, self._h
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), get_reasons(h),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
            except Exception as e:
                self.err = str(e)
                break
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"error": self.err or "no samples"}
        mask = 0
        for _, r, _ in self.samples:
            mask |= r
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in sorted(self.NAMES.items()) if mask & b],
                "power_w_max": round(max(s[2] for s in self.samples), 1), "samples": len(self.samples),
                "source": "NVML during the timed region"}


# ---------------------------------------------------------------------------- CPU oracle


def oracle_sample(x_bits, qw, sw, bias, rows: int, block: int):
    """The oracle's whole path (quantise, int64 GEMM, fp64 dequant) on `rows`
    token rows; returns seconds."""
    from oracle import oracle as O
    b, reg = oracle_block(block)
    t0 = time.perf_counter()
    qx, sx = O.quantize_act(x_bits[:rows], b, reg)
    acc = O.igemm(qx, qw)
    O.dequant(acc, sx, sw, bias, b)
    return time.perf_counter() - t0


def oracle_pack(w, block: int):
    from oracle import oracle as O
    b, reg = oracle_block(block)
    return O.pack_weight(w, b, reg)


def cpu_baseline(spec, target_s: float = 12.0):
    """Oracle timed on the host cores on a bounded sample of the workload."""
    import numpy as np
    from oracle import oracle as O
    from w8a8_int8_quantized_block_b200 import workloads as W
    x, w, bias = W.linear_inputs(spec)
    xb = O.bf16_bits(x)
    qw, sw = oracle_pack(w.numpy(), spec.block)  # offline on both sides: not timed
    b = bias.numpy().astype(np.float32)
    rows = 16
    t = oracle_sample(xb, qw, sw, b, rows, spec.block)
    while t < 0.5 * target_s and rows < spec.M:  # grow the sample until it takes about target_s
        rows = int(min(spec.M, max(2 * rows, round(rows * target_s / max(t, 1e-3)))))
        t = oracle_sample(xb, qw, sw, b, rows, spec.block)
    ops = 2.0 * rows * spec.N * spec.K
    return {"value": ops / t / 1e12, "unit": UNIT, "cores": O.num_threads(), "kind": "oracle",
            "sample": f"{rows} of {spec.M} token rows through the whole path (rotate+quantise, int64 GEMM vs all "
                      f"{spec.N} columns, fp64 dequant) in {t:.1f} s; weight packing excluded on both sides"}


def run_reference(args, rank: int):
    """`--impl reference`: the CPU oracle, as it stands, on this host."""
    from w8a8_int8_quantized_block_b200 import workloads as W
    from oracle import oracle as O
    import numpy as np
    if rank != 0:
        return
    spec = workload(args)
    x, w, bias = W.linear_inputs(spec)
    xb = O.bf16_bits(x)
    qw, sw = oracle_pack(w.numpy(), spec.block)
    b = bias.numpy().astype(np.float32)
    per_step_target = max(0.02, args.reference_seconds / max(1, args.steps + args.warmup))
    t = oracle_sample(xb, qw, sw, b, 8, spec.block)
    rows = int(min(spec.M, max(1, round(8 * per_step_target / max(t, 1e-4)))))
    for _ in range(args.warmup):
        oracle_sample(xb, qw, sw, b, rows, spec.block)
    tot = 0.0
    for _ in range(args.steps):
        tot += oracle_sample(xb, qw, sw, b, rows, spec.block)
    ops = 2.0 * rows * spec.N * spec.K * args.steps
    value = ops / tot / 1e12
    sample = f"each step: {rows} of {spec.M} token rows through the oracle's whole path"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic", "config": config_dict(spec, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": O.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(spec, n, context_parallel=False):
    par = (f"cp{n} (the tokens split across GPUs, then an all-gather of the output rows)" if context_parallel
           else f"dp{n} (independent token batches per GPU)")
    return {"workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "block": spec.block,
            "parallelism": par,
            "l2": "inputs larger than L2: x and y are 415.6 MB each per step; the 28.9 MB packed weights "
                  "stay L2-resident across steps as they do when one layer serves many batches"}


# ---------------------------------------------------------------------------- timing helpers


IDLE_GAP_S = 1.0  # the GPU idles this long before each timed leg, so no leg inherits the power cap of the last


def loop_time(fn, n: int, stream, world: int, clocks: bool = True, gap_s: float = IDLE_GAP_S):
    """n back-to-back calls between two CUDA events on `stream` (a barrier and
    a synchronize on both sides, after `gap_s` seconds of idle GPU); returns
    (slowest rank's seconds per call, NVML clock summary of the region or None)."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    time.sleep(gap_s)
    clk = ClockSampler(torch.cuda.current_device()) if clocks else None
    if clk:
        clk.__enter__()
    try:
        barrier()
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        barrier()
    finally:
        if clk:
            clk.__exit__()
    return max_over_ranks(e0.elapsed_time(e1) / 1e3, world) / n, (clk.summary() if clk else None)


def graph_time(fn, calls: int, reps: int):
    """Device time of one call when `calls` calls are replayed from one CUDA
    graph (no host launch cost between them): fn(stream) enqueues one call."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(calls):
            fn(s)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    e0.record(cur)
    for _ in range(reps):
        g.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / (reps * calls)
    del g
    return t


def cold_time(fn, n: int, stream, flush):
    """Mean device time of one call with the L2 flushed before each (the flush
    is outside the events): for workloads small enough to sit in L2."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize()
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / n / 1e3


def check_status(C, where: str):
    st, code = C.last_device_status()
    if st != C.OK:
        raise RuntimeError(f"device status {st} (code {code}) {where}")


def grow_sample(run, start: int, limit: int, target_s: float):
    """Grow a row sample until one timed oracle pass takes about target_s;
    returns (rows, seconds)."""
    rows = start
    t = run(rows)
    while t < 0.5 * target_s and rows < limit:
        rows = int(min(limit, max(2 * rows, round(rows * target_s / max(t, 1e-3)))))
        t = run(rows)
    return rows, t


# ---------------------------------------------------------------------------- other workloads


def measure_tiny(args, world, stream, flush, peak_i8):
    """The tiny projection (M = 256, K = N = 512): one fused call, latency-bound."""
    import numpy as np
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W
    spec = W.TINY
    x_cpu, w_cpu, b_cpu = W.linear_inputs(spec)
    x, bias = x_cpu.cuda(), b_cpu.cuda()
    pw = C.pack_weight(w_cpu.cuda(), spec.block)
    ws = C.alloc_workspace(spec.M, spec.K)
    import torch
    y = torch.empty(spec.M, spec.N, dtype=torch.bfloat16, device="cuda")
    call = lambda st: C.linear_fused(x, pw, bias, workspace=ws, out=y, stream=st)
    step = lambda: call(stream)
    for _ in range(5):
        step()
    t_cold = cold_time(step, 50, stream, flush)
    t_warm, clk = loop_time(step, 500, stream, world)
    t_graph = graph_time(call, 100, 20)
    check_status(C, "after the tiny projection")
    out = {"workload": spec.name, "us": t_graph * 1e6, "TOPS": spec.ops / t_graph / 1e12,
           "frac_of_int8_peak": spec.ops / t_graph / 1e12 / peak_i8,
           "us_direct_calls": t_warm * 1e6, "us_cold": t_cold * 1e6,
           "bound": "latency: 0.13 GOP is one 256-row panel of two column tiles, so 2 of 74 CTA pairs work and "
                    "the call is the one-kernel path's fill and drain plus the launch",
           "timing": "us: device time per call with 100 calls replayed from one CUDA graph (20 replays); "
                     "us_direct_calls: 500 calls from the host in a row (host launch cost included); "
                     "us_cold: mean of 50 direct calls with the L2 flushed before each",
           "clocks": clk}
    if not args.no_cpu_baseline:
        from oracle import oracle as O
        xb, qw_sw = O.bf16_bits(x_cpu), oracle_pack(w_cpu.numpy(), spec.block)
        b = b_cpu.numpy().astype(np.float32)
        reps, t = 0, 0.0
        while t < 1.0:
            t += oracle_sample(xb, qw_sw[0], qw_sw[1], b, spec.M, spec.block)
            reps += 1
        out["cpu_baseline"] = {"value": reps * spec.ops / t / 1e12, "unit": UNIT, "cores": O.num_threads(),
                               "kind": "oracle", "sample": f"the whole workload ({spec.M} rows), {reps} passes"}
    return out


def measure_proj4k(args, world, stream, flush, peak_i8):
    """The 4096-token projection (K = N = 5376): tensor-bound, fits in L2."""
    import numpy as np
    import torch
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W
    spec = W.PROJ_4K
    x_cpu, w_cpu, b_cpu = W.linear_inputs(spec)
    x, bias = x_cpu.cuda(), b_cpu.cuda()
    pw = C.pack_weight(w_cpu.cuda(), spec.block)
    ws = C.alloc_workspace(spec.M, spec.K)
    y = torch.empty(spec.M, spec.N, dtype=torch.bfloat16, device="cuda")
    step = lambda: C.linear_fused(x, pw, bias, workspace=ws, out=y, stream=stream)
    for _ in range(5):
        step()
    t_cold = cold_time(step, 50, stream, flush)
    t_warm, clk = loop_time(step, 300, stream, world)
    check_status(C, "after the 4096-token projection")
    out = {"workload": spec.name, "us": t_cold * 1e6, "TOPS": spec.ops / t_cold / 1e12,
           "frac_of_int8_peak": spec.ops / t_cold / 1e12 / peak_i8,
           "us_back_to_back": t_warm * 1e6, "TOPS_back_to_back": spec.ops / t_warm / 1e12,
           "bound": "tensor (2 M N K = 236.8 GOP; 16 x 21 tiles of 256 x 256 over 74 CTA pairs)",
           "timing": "us: mean of 50 calls with the L2 flushed before each (x, y and the weights, 117 MB, "
                     "would otherwise stay in the 126 MB L2); back_to_back: 300 calls in a row",
           "clocks": clk}
    if not args.no_cpu_baseline:
        from oracle import oracle as O
        xb = O.bf16_bits(x_cpu)
        qw, sw = oracle_pack(w_cpu.numpy(), spec.block)
        b = b_cpu.numpy().astype(np.float32)
        rows, t = grow_sample(lambda r: oracle_sample(xb, qw, sw, b, r, spec.block), 16, spec.M, 5.0)
        out["cpu_baseline"] = {"value": 2.0 * rows * spec.N * spec.K / t / 1e12, "unit": UNIT,
                               "cores": O.num_threads(), "kind": "oracle",
                               "sample": f"{rows} of {spec.M} token rows through the whole path in {t:.1f} s"}
    return out


MLP_METRIC = "ConvRot W8A8 MLP TOPS at M=38656, K=5376, H=21504 (up + GELU + down)"


def measure_mlp(args, world, stream, peak_i8, steps: int, route_for_clocks: str = "epilogue"):
    """The 768p MLP pair by both routes of its GELU: in the up projection's
    epilogue (then the plain quantiser on the down projection's input), or as
    the down projection's prologue (convrot_linear_act on the plain up
    projection's output)."""
    import numpy as np
    import torch
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W

    spec = W.MLP_768P
    x_cpu, w1_cpu, w2_cpu = W.mlp_inputs(spec)
    x = x_cpu.cuda()
    p1 = C.pack_weight(w1_cpu.cuda(), spec.block)
    p2 = C.pack_weight(w2_cpu.cuda(), spec.block)
    ws1 = C.alloc_workspace(spec.M, spec.K)
    ws2 = C.alloc_workspace(spec.M, spec.H)
    h = torch.empty(spec.M, spec.H, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(spec.M, spec.K, dtype=torch.bfloat16, device="cuda")

    def up(gelu):
        C.linear_fused(x, p1, None, gelu=gelu, workspace=ws1, out=h, stream=stream)

    def down(prologue):
        if prologue:
            C.linear_act(h, C.ACT_GELU, p2, None, workspace=ws2, out=y, stream=stream)
        else:
            C.linear_fused(h, p2, None, workspace=ws2, out=y, stream=stream)

    routes = {"epilogue": (lambda: (up(True), down(False))), "prologue": (lambda: (up(False), down(True)))}
    for r in routes.values():
        for _ in range(2):
            r()
    times, kern, clocks = {}, {}, {}
    for name, fn in routes.items():
        times[name], clocks[name] = loop_time(fn, steps, stream, world)
        nk = min(steps, 20)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nk)]
        torch.cuda.synchronize()
        for i in range(nk):
            ev[i][0].record(stream)
            up(name == "epilogue")
            ev[i][1].record(stream)
            down(name == "prologue")
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        kern[name] = {"up_us": sum(e[0].elapsed_time(e[1]) for e in ev) / nk * 1e3,
                      "down_us": sum(e[1].elapsed_time(e[2]) for e in ev) / nk * 1e3}
    check_status(C, "after the MLP")
    t = times["epilogue"]
    out = {"workload": spec.name, "route": "epilogue (GELU in the up projection's epilogue)",
           "ms_per_step": t * 1e3, "TOPS": spec.ops / t / 1e12, "frac_of_int8_peak": spec.ops / t / 1e12 / peak_i8,
           "bound": "tensor (17.9 TOP per step)",
           "routes": {n: {"TOPS": spec.ops / times[n] / 1e12, "ms_per_step": times[n] * 1e3, **kern[n],
                          "clocks": clocks[n]} for n in times},
           "timing": f"{steps} steps back to back per route (inputs larger than L2: h is 1.66 GB)",
           "clocks": clocks[route_for_clocks]}
    del x, h, y, ws1, ws2, p1, p2
    if not args.no_cpu_baseline:
        from oracle import oracle as O
        xb = O.bf16_bits(x_cpu)
        q1, s1 = O.pack_weight(w1_cpu.numpy(), spec.block)
        q2, s2 = O.pack_weight(w2_cpu.numpy(), spec.block)

        def run(r):
            t0 = time.perf_counter()
            qx, sx = O.quantize_act(xb[:r], spec.block)
            hh = O.dequant(O.igemm(qx, q1), sx, s1, None, spec.block, True)
            hb = O.bf16_bits(torch.from_numpy(hh).to(torch.bfloat16))
            qh, sh = O.quantize_act(hb, spec.block)
            O.dequant(O.igemm(qh, q2), sh, s2, None, spec.block)
            return time.perf_counter() - t0

        rows, t = grow_sample(run, 4, spec.M, 5.0)
        out["cpu_baseline"] = {"value": 4.0 * rows * spec.H * spec.K / t / 1e12, "unit": UNIT,
                               "cores": O.num_threads(), "kind": "oracle",
                               "sample": f"{rows} of {spec.M} token rows through both projections (GELU in "
                                         f"fp64, bf16 between them) in {t:.1f} s"}
    return out


def measure_bmm(args, world, stream, hbm, peak_i8, steps: int):
    """The skinny-K batched GEMM (42 heads, M = N = 8192, K = 128): quantise Q
    and K per row (no rotation), then the GEMM writing 5.64 GB of bf16."""
    import numpy as np
    import torch
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W
    spec = W.QK_BMM
    q_cpu, k_cpu = W.bmm_inputs(spec)
    B, M, N, K = spec.batch, spec.M, spec.N, spec.K
    q, k = q_cpu.cuda().view(B * M, K), k_cpu.cuda().view(B * N, K)
    qa = torch.empty(B * M, K, dtype=torch.int8, device="cuda")
    qb = torch.empty(B * N, K, dtype=torch.int8, device="cuda")
    sa = torch.empty(B * M, device="cuda")
    sb = torch.empty(B * N, device="cuda")
    y = torch.empty(B, M, N, dtype=torch.bfloat16, device="cuda")

    def gemm():
        C.w8a8_bmm(qa.view(B, M, K), sa, qb.view(B, N, K), sb, out=y, stream=stream)

    def step():
        C.quantize_act(q, 0, qa, sa, stream=stream)
        C.quantize_act(k, 0, qb, sb, stream=stream)
        gemm()

    for _ in range(3):
        step()
    t_step, clk = loop_time(step, steps, stream, world)
    t_gemm, clk_g = loop_time(gemm, steps, stream, world)
    t_fill, _ = loop_time(lambda: y.fill_(1.0), steps, stream, world, clocks=False)
    check_status(C, "after the Q K^T GEMM")
    out_bytes = B * M * N * 2
    gemm_bytes = out_bytes + (B * M + B * N) * (K + 4)
    out = {"workload": spec.name, "us": t_step * 1e6, "TOPS": spec.ops / t_step / 1e12,
           "gemm_us": t_gemm * 1e6, "gemm_TOPS": spec.ops / t_gemm / 1e12,
           "gemm_GB/s": gemm_bytes / t_gemm / 1e9, "frac_of_hbm": gemm_bytes / t_gemm / 1e9 / hbm,
           "hbm_peak_gbs": hbm, "algorithmic_bytes_per_launch": gemm_bytes,
           "write_only_ceiling_gbs": out_bytes / t_fill / 1e9,
           "frac_of_write_ceiling": (gemm_bytes / t_gemm) / (out_bytes / t_fill),
           "bound": "HBM store (5.64 GB of bf16 out per step, 2 bytes per 256 ops)",
           "timing": f"{steps} steps back to back (quantise Q, quantise K, GEMM); the GEMM alone likewise; "
                     "write_only_ceiling: torch fill_ of the same 5.64 GB output, back to back",
           "clocks": clk, "clocks_gemm": clk_g}
    del q, k, qa, qb, sa, sb, y
    if not args.no_cpu_baseline:
        from oracle import oracle as O
        qbits = O.bf16_bits(q_cpu[0])
        kbits = O.bf16_bits(k_cpu[0])

        def run(r):
            t0 = time.perf_counter()
            qx, sx = O.quantize_act(qbits[:r], 0)
            kx, sk = O.quantize_act(kbits, 0)
            O.dequant(O.igemm(qx, kx), sx, sk, None, 0)
            return time.perf_counter() - t0

        rows, t = grow_sample(run, 64, M, 5.0)
        out["cpu_baseline"] = {"value": 2.0 * rows * N * K / t / 1e12, "unit": UNIT, "cores": O.num_threads(),
                               "kind": "oracle",
                               "sample": f"{rows} query rows of head 0 against its {N} keys (quantise, int64 "
                                         f"GEMM, fp64 dequant) in {t:.1f} s"}
    return out


ATTN_METRIC = "int8 attention TFLOP/s at 42 heads x 8192 tokens, d=128 (Q K^T int8 + P V bf16)"


def measure_attention(args, world, stream, bf16, steps: int, heads=None):
    """int8 attention on the 42-head, 8192-token workload: the whole entry
    (quantise Q and K, transpose V, attend) and the attention kernel alone.
    Work = 2 H L^2 d int8 ops (Q K^T) + 2 H L^2 d bf16 flops (P V)."""
    import numpy as np
    import torch
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W

    spec = W.QK_BMM
    H, L, d = spec.batch, spec.M, spec.K
    q_cpu, k_cpu = W.bmm_inputs(spec)
    v_cpu = torch.randn(H, L, d, generator=torch.Generator().manual_seed(44)).to(torch.bfloat16)
    if heads is not None:  # a smaller case of the same workload: its first heads
        if not 1 <= heads <= H:
            raise SystemExit(f"--heads must be in [1, {H}]")
        H = heads
        q_cpu, k_cpu, v_cpu = q_cpu[:H].contiguous(), k_cpu[:H].contiguous(), v_cpu[:H].contiguous()
    q, k, v = q_cpu.cuda(), k_cpu.cuda(), v_cpu.cuda()
    Lib = C.load()
    ws = torch.empty((Lib.convrot_attention_workspace_bytes(H, L, L),), dtype=torch.uint8, device="cuda")
    o = torch.empty(H, L, d, dtype=torch.bfloat16, device="cuda")
    r256 = lambda n: (n + 255) // 256 * 256
    off_sq = r256(H * L * d)
    off_kx = off_sq + r256(H * L * 4)
    off_sk = off_kx + r256(H * L * d)
    off_vt = off_sk + r256(H * L * 4)
    qx, sq = ws[:H * L * d].view(torch.int8).view(H, L, d), ws[off_sq:off_sq + H * L * 4].view(torch.float32)
    kx, sk = ws[off_kx:off_kx + H * L * d].view(torch.int8).view(H, L, d), ws[off_sk:off_sk + H * L * 4].view(
        torch.float32)
    vt = ws[off_vt:off_vt + H * d * L * 2].view(torch.bfloat16).view(H, d, L)
    off_part = off_vt + r256(H * d * L * 2)
    part_bytes = C.attention_split_bytes(H, L, L)
    part = ws[off_part:off_part + part_bytes] if part_bytes else None
    # attention launches per call: the units of whole waves, and (when the last
    # wave is split over its keys) the split units and the combine
    units = H * ((L // 128 + 1) // 2)
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    main_units = units - units % sms if part_bytes else units
    attn_launches = (1 if main_units > 0 else 0) + (2 if part_bytes else 0)

    full = lambda: C.attention(q, k, v, workspace=ws, out=o, stream=stream)
    kernel = lambda: C.attention_int8(qx, sq, kx, sk, vt, out=o, stream=stream, split_ws=part)
    for _ in range(3):
        full()
    t_kernel, clk = loop_time(kernel, steps, stream, world)
    t_full, clk_full = loop_time(full, steps, stream, world)
    check_status(C, "after attention")
    int8_peak = bf16 * INT8_PER_BF16
    half = 2.0 * H * L * L * d          # each of the two products
    ops = 2 * half
    t_tensor = half / (int8_peak * 1e12) + half / (bf16 * 1e12)   # both products at their peaks
    mufu = 16 * sms * 1.965e9                                      # 2^x per second (SFU, nominal)
    t_exp = H * L * L / mufu
    out = {"workload": f"attention_h{H}_l{L}_d{d}", "heads": H, "L": L, "d": d,
           "ms": t_full * 1e3, "TFLOP/s": ops / t_full / 1e12,
           "kernel_ms": t_kernel * 1e3, "kernel_TFLOP/s": ops / t_kernel / 1e12,
           "frac_of_tensor_bound": t_tensor / t_kernel, "tensor_bound_ms": t_tensor * 1e3,
           "exp2_bound_ms": t_exp * 1e3, "attn_launches": attn_launches,
           "bound": f"tensor: Q K^T at bf16 burst x {INT8_PER_BF16}, P V at the bf16 burst {bf16} TFLOP/s; the "
                    f"2^x of the softmax alone would take {t_exp * 1e3:.3f} ms on the special-function units "
                    f"(nominal 16/clk/SM at 1965 MHz)",
           "timing": f"{steps} calls back to back (the kernel on quantised inputs; the whole entry)",
           "clocks": clk, "clocks_full": clk_full}
    del q, k, v, ws, o
    if not args.no_cpu_baseline:
        from oracle import oracle as O
        qx0, sq0 = O.quantize_act(O.bf16_bits(q_cpu[0]), 0)
        kx0, sk0 = O.quantize_act(O.bf16_bits(k_cpu[0]), 0)
        vb = O.bf16_bits(v_cpu[:1])

        def run(r):
            t0 = time.perf_counter()
            O.attention_rows(qx0[None], sq0[None], kx0[None], sk0[None], vb, np.zeros(r, dtype=np.int64),
                             np.arange(r), d ** -0.5)
            return time.perf_counter() - t0

        rows, t = grow_sample(run, 4, L, 4.0)
        out["cpu_baseline"] = {"value": 4.0 * rows * L * d / t / 1e12, "unit": "TFLOP/s", "cores": O.num_threads(),
                               "kind": "oracle",
                               "sample": f"{rows} query rows of head 0 over all {L} keys (int64 scores, fp64 "
                                         f"softmax and P V), in {t:.1f} s"}
    return out, ops


def run_attention(args, rank: int, world: int):
    import torch
    import torch.distributed as dist
    stream = torch.cuda.current_stream()
    hbm, bf16, bf16_sus, kind = peaks()
    r, ops = measure_attention(args, world, stream, bf16, args.steps, args.heads)
    if rank == 0:
        value = world * ops / (r["ms"] / 1e3) / 1e12
        line = {
            "metric": ATTN_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8+bf16", "data": "synthetic",
            "config": {"workload": r["workload"], "heads": r["heads"], "Lq": r["L"], "Lk": r["L"], "d": r["d"],
                       "parallelism": f"dp{world} (independent heads and sequences per GPU)",
                       "l2": "Q, K, V and O are 88 MB each at 42 heads (bf16); the score matrix is never stored"},
            "roofline": {"bound": "tensor", "kernel": f"attention_kernel ({r['attn_launches']} launch(es))",
                         "achieved": r["kernel_TFLOP/s"], "peak": ops / (r["tensor_bound_ms"] / 1e3) / 1e12,
                         "unit": "TFLOP/s", "frac": r["frac_of_tensor_bound"], "traffic": None,
                         "peak_source": f"{kind}: {r['bound']}"},
            "kernels": {"attention_kernel_us": r["kernel_ms"] * 1e3,
                        "quantise_transpose_us": (r["ms"] - r["kernel_ms"]) * 1e3},
            "clocks": r["clocks_full"],
            "gpu_launches": (3 + r["attn_launches"]) * args.steps,
        }
        if "cpu_baseline" in r:
            line["cpu_baseline"] = r["cpu_baseline"]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_mlp(args, rank: int, world: int):
    """The MLP line; its value is for --mlp-route."""
    import torch
    import torch.distributed as dist
    from w8a8_int8_quantized_block_b200 import workloads as W
    stream = torch.cuda.current_stream()
    hbm, bf16, bf16_sus, kind = peaks()
    int8_peak = bf16 * INT8_PER_BF16
    r = measure_mlp(args, world, stream, int8_peak, args.steps, args.mlp_route)
    if rank == 0:
        spec = W.MLP_768P
        t = r["routes"][args.mlp_route]["ms_per_step"] / 1e3
        value = job_tops(spec.ops, 1, world, t)
        line = {
            "metric": MLP_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": spec.name, "M": spec.M, "K": spec.K, "H": spec.H, "block": spec.block,
                       "activation": "gelu", "route": args.mlp_route,
                       "parallelism": f"dp{world} (independent token batches per GPU)",
                       "l2": "inputs larger than L2: h is 1.66 GB per step"},
            "pct_of_int8_peak": round(100.0 * value / world / int8_peak, 2),
            "routes": r["routes"],
            "clocks": r["clocks"],
            "gpu_launches": 3 * args.steps,  # up (one kernel), down (quantiser + GEMM)
        }
        if "cpu_baseline" in r:
            line["cpu_baseline"] = r["cpu_baseline"]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def kernel_only(args, spec, x, x_cpu, pw, bias, ws, y, stream):
    """`--kernel-only`: launch one kernel warmup + steps times (profiler captures)."""
    import torch
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W
    which = args.kernel_only
    if which in ("fused", "quant", "gemm"):
        q, s = ws[:spec.M * spec.K].view(torch.int8).view(spec.M, spec.K), torch.empty(spec.M, device="cuda")
        C.quantize_act(x, spec.block, q, s, stream=stream)
        one = {"fused": lambda: C.linear_fused(x, pw, bias, workspace=ws, out=y, stream=stream),
               "quant": lambda: C.quantize_act(x, spec.block, q, s, stream=stream),
               "gemm": lambda: C.w8a8_linear(q, s, pw, bias, out=y, stream=stream)}[which]
    elif which == "bmm":
        bs = W.QK_BMM
        B = bs.batch if args.heads is None else args.heads
        qa = torch.randint(-127, 128, (B, bs.M, bs.K), dtype=torch.int8, device="cuda")
        qb = torch.randint(-127, 128, (B, bs.N, bs.K), dtype=torch.int8, device="cuda")
        sa, sb = torch.rand(B * bs.M, device="cuda"), torch.rand(B * bs.N, device="cuda")
        yb = torch.empty(B, bs.M, bs.N, dtype=torch.bfloat16, device="cuda")
        one = lambda: C.w8a8_bmm(qa, sa, qb, sb, out=yb, stream=stream)
    elif which == "mlp-up":  # the MLP's up projection on the first --rows rows of its workload
        ms = W.MLP_768P
        rows = ms.M if args.rows is None else args.rows
        g = torch.Generator(device="cuda").manual_seed(ms.seed)
        xu = (torch.randn(rows, ms.K, device="cuda", generator=g) * 2.0).to(torch.bfloat16)
        w1 = torch.randn(ms.H, ms.K, device="cuda", generator=g) * ms.w_std
        p1 = C.pack_weight(w1, ms.block)
        del w1
        wsu = C.alloc_workspace(rows, ms.K)
        hu = torch.empty(rows, ms.H, dtype=torch.bfloat16, device="cuda")
        one = lambda: C.linear_fused(xu, p1, None, gelu=True, workspace=wsu, out=hu, stream=stream)
    else:  # the MLP's down projection (K = 21504) on the first --rows rows of its workload
        ms = W.MLP_768P
        rows = ms.M if args.rows is None else args.rows
        g = torch.Generator(device="cuda").manual_seed(ms.seed)
        h = (torch.randn(rows, ms.H, device="cuda", generator=g) * 2.0).to(torch.bfloat16)
        w2 = torch.randn(ms.K, ms.H, device="cuda", generator=g) * ms.w_std
        p2 = C.pack_weight(w2, ms.block)
        del w2
        q2 = torch.empty(rows, ms.H, dtype=torch.int8, device="cuda")
        s2 = torch.empty(rows, device="cuda")
        y2 = torch.empty(rows, ms.K, dtype=torch.bfloat16, device="cuda")
        C.act_quantize(h, C.ACT_GELU, ms.block, q2, s2, stream=stream)
        one = (lambda: C.w8a8_linear(q2, s2, p2, None, out=y2, stream=stream)) if which == "mlp-down" else \
            (lambda: C.act_quantize(h, C.ACT_GELU, ms.block, q2, s2, stream=stream))
    for _ in range(args.warmup + args.steps):
        one()
    torch.cuda.synchronize()
    check_status(C, "after the kernel-only loop")


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)

    import torch
    import torch.distributed as dist
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if args.workload == "attention":
        return run_attention(args, rank, world)
    if args.workload == "mlp":
        return run_mlp(args, rank, world)
    spec = workload(args)
    x_cpu, w_cpu, b_cpu = W.linear_inputs(spec)
    if args.rows is not None and not args.kernel_only:
        raise SystemExit("--rows needs --kernel-only")
    if args.rows is not None and args.kernel_only in ("fused", "quant", "gemm"):
        import dataclasses
        if not 1 <= args.rows <= spec.M:
            raise SystemExit(f"--rows must be in [1, {spec.M}]")
        spec = dataclasses.replace(spec, M=args.rows, name=f"{spec.name}_rows{args.rows}")
        x_cpu = x_cpu[:args.rows].contiguous()
    job = spec  # the whole job's tokens
    if args.context_parallel:
        import dataclasses
        from w8a8_int8_quantized_block_b200 import context_parallel as CP
        lo, hi = CP.token_shard(spec.M, world, rank)
        x_cpu = x_cpu[lo:hi].contiguous()
        spec = dataclasses.replace(spec, M=hi - lo)  # this rank's shard: the per-kernel and end-to-end legs
    x = x_cpu.cuda()
    bias = b_cpu.cuda()
    pw = C.pack_weight(w_cpu.cuda(), spec.block)
    ws = C.alloc_workspace(spec.M, spec.K)
    y = torch.empty(spec.M, spec.N, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    if args.kernel_only:
        return kernel_only(args, spec, x, x_cpu, pw, bias, ws, y, stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    if args.context_parallel:
        y_full = torch.empty(job.M, job.N, dtype=torch.bfloat16, device="cuda")

        def shard_linear(xs, out):
            C.linear_fused(xs, pw, bias, workspace=ws, out=out, stream=stream)

        def step():
            CP.linear_context_parallel(x, job.M, job.N, shard_linear, out=y_full)
    else:
        def step():
            C.linear_fused(x, pw, bias, workspace=ws, out=y, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    barrier()
    check_status(C, "after warm-up")

    # ---- the headline: K steps back to back
    per_step, clk_head = loop_time(step, args.steps, stream, world)
    elapsed_s = per_step * args.steps
    check_status(C, "after the timed region")
    if args.context_parallel:
        value = job.ops * args.steps / elapsed_s / 1e12  # strong scaling: the ranks share one job
    else:
        value = job_tops(spec.ops, args.steps, world, elapsed_s)

    # ---- each kernel of the step in its own back-to-back loop (CUDA events on
    # the launching stream around the loop; x and y are larger than L2)
    q, s = ws[:spec.M * spec.K].view(torch.int8).view(spec.M, spec.K), torch.empty(spec.M, device="cuda")
    fused = lambda: C.linear_fused(x, pw, bias, workspace=ws, out=y, stream=stream)
    quant = lambda: C.quantize_act(x, spec.block, q, s, stream=stream)
    gemm = lambda: C.w8a8_linear(q, s, pw, bias, out=y, stream=stream)
    nk = max(args.steps, 100)
    t_fused, clk_fused = loop_time(fused, nk, stream, world)
    for _ in range(3):
        quant()
    t_quant, clk_quant = loop_time(quant, args.quant_launches, stream, world)
    t_gemm, clk_gemm = loop_time(gemm, nk, stream, world)
    check_status(C, "after the per-kernel loops")

    # ---- sustained: the same step for at least --sustained-seconds, under the power cap
    n_sus = max(args.steps, int(args.sustained_seconds / max(per_step, 1e-6)) + 1)
    t_sus, clk_sus = loop_time(step, n_sus, stream, world)
    check_status(C, "after the sustained leg")

    # ---- end to end through the C ABI with host buffers (copies inside the timed region)
    x_host = x_cpu.pin_memory()
    y_host = torch.empty(spec.M, spec.N, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    e2e = lambda: C.linear_fused_host(x_host, pw, bias, False, x_dev, ws, y, y_host, stream=stream)
    for _ in range(2):
        e2e()
    e2e_per, _ = loop_time(e2e, args.e2e_steps, stream, world, clocks=False)
    e2e_value = job_tops(spec.ops, 1, world, e2e_per)
    check_status(C, "after the end-to-end leg")
    del x_host, y_host, x_dev

    hbm, bf16, bf16_sus, kind = peaks()
    int8_peak = bf16 * INT8_PER_BF16
    int8_sus = bf16_sus * INT8_PER_BF16

    # ---- the other workloads (one GPU)
    configs = None
    if world == 1 and not args.no_configs and not args.context_parallel:
        del q, s
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        configs = {}
        configs["tiny"] = measure_tiny(args, world, stream, flush, int8_peak)
        configs["proj_4k"] = measure_proj4k(args, world, stream, flush, int8_peak)
        del flush
        configs["mlp"] = measure_mlp(args, world, stream, int8_peak, max(5, min(args.steps, 20)))
        torch.cuda.empty_cache()
        configs["qk_bmm"] = measure_bmm(args, world, stream, hbm, int8_peak, max(5, min(args.steps, 20)))
        torch.cuda.empty_cache()
        configs["attention"], _ = measure_attention(args, world, stream, bf16, max(5, min(args.steps, 20)))
        torch.cuda.empty_cache()

    if rank == 0:
        achieved = spec.ops / t_fused / 1e12
        quant_bytes = spec.M * spec.K * 3 + spec.M * 4
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_s / args.steps * 1e3, "higher_is_better": True,
            "scaling": "strong" if args.context_parallel else "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic", "config": config_dict(job, world, args.context_parallel),
            "pct_of_int8_peak": round(100.0 * value / world / int8_peak, 2),
            "roofline": {"bound": "tensor",
                         "kernel": "linear_fused_kernel (rotate + quantise + int8 GEMM + dequant epilogue, one launch)",
                         "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s", "frac": achieved / int8_peak,
                         "traffic": profiled_traffic() if args.block == "128" else None,
                         "peak_source": f"{kind} bf16 burst {bf16} TFLOP/s x {INT8_PER_BF16} (nominal int8:bf16)",
                         "algorithmic_ops_per_launch": spec.ops},
            "kernels": {
                "linear_fused_kernel": {"us": t_fused * 1e6, "TOPS": achieved, "frac_of_int8_peak": achieved / int8_peak,
                                        "launches": nk, "clocks": clk_fused},
                "igemm_pair_kernel (split path)": {"us": t_gemm * 1e6, "TOPS": spec.ops / t_gemm / 1e12,
                                                   "frac_of_int8_peak": spec.ops / t_gemm / 1e12 / int8_peak,
                                                   "launches": nk, "clocks": clk_gemm},
                "rotate_quant_kernel": {"us": t_quant * 1e6, "GB/s": quant_bytes / t_quant / 1e9,
                                        "frac_of_hbm": quant_bytes / t_quant / 1e9 / hbm, "hbm_peak_gbs": hbm,
                                        "algorithmic_bytes_per_launch": quant_bytes,
                                        "launches": args.quant_launches, "clocks": clk_quant,
                                        "timing": "back-to-back launches between two CUDA events"},
            },
            "sustained": {"ms_per_step": t_sus * 1e3, "steps": n_sus, "seconds": t_sus * n_sus,
                          "TOPS": job_tops(spec.ops, 1, world, t_sus),
                          "frac": spec.ops / t_sus / 1e12 / int8_sus, "peak": int8_sus,
                          "peak_source": f"{kind} bf16 sustained {bf16_sus} TFLOP/s x {INT8_PER_BF16}",
                          "clocks": clk_sus},
            "clocks": clk_head,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": spec.M * spec.K * 2,
                    "d2h_bytes_per_step": spec.M * spec.N * 2, "steps": args.e2e_steps,
                    "path": "convrot_linear_fused_host (pinned host x -> device -> linear -> pinned host y)"},
            "gpu_launches": args.steps,  # one linear_fused_kernel per step (plus a memset node of its counters)
        }
        if configs is not None:
            line["configs"] = configs
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(spec)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
