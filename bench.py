"""Throughput of the ConvRot W8A8 INT8 linear on B200.

One step = one whole pass of the hot path over one batch: rotate + quantise
the bf16 activations, int8 GEMM, dequantise with bias to bf16 (the weights
are packed once, offline, as the pages' checkpoints are).  The workload is
the full 768p projection, M = 38656 tokens, K = N = 5376, Hadamard block 128.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

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
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


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
    ap.add_argument("--kernel-only", choices=["fused", "quant", "gemm"], default=None,
                    help="set up, then launch only this kernel --warmup + --steps times and exit "
                         "(for profiler captures; prints no result line)")
    return ap.parse_args()


def peaks():
    try:
        p = json.load(open(PEAKS_FILE))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


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


# ---------------------------------------------------------------------------- GPU path


ATTN_METRIC = "int8 attention TFLOP/s at 42 heads x 8192 tokens, d=128 (Q K^T int8 + P V bf16)"


def run_attention(args, rank: int, world: int):
    """int8 attention on the 42-head, 8192-token workload: the whole entry
    (quantise Q and K, transpose V, attend) and the attention kernel alone.
    Work = 2 H L^2 d int8 ops (Q K^T) + 2 H L^2 d bf16 flops (P V)."""
    import torch
    import torch.distributed as dist
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W

    spec = W.QK_BMM
    H, L, d = spec.batch, spec.M, spec.K
    q_cpu, k_cpu = W.bmm_inputs(spec)
    v_cpu = torch.randn(H, L, d, generator=torch.Generator().manual_seed(44)).to(torch.bfloat16)
    if args.heads is not None:  # a smaller case of the same workload: its first heads
        if not 1 <= args.heads <= H:
            raise SystemExit(f"--heads must be in [1, {H}]")
        H = args.heads
        q_cpu, k_cpu, v_cpu = q_cpu[:H].contiguous(), k_cpu[:H].contiguous(), v_cpu[:H].contiguous()
    q, k, v = q_cpu.cuda(), k_cpu.cuda(), v_cpu.cuda()
    Lib = C.load()
    ws = torch.empty((Lib.convrot_attention_workspace_bytes(H, L, L),), dtype=torch.uint8, device="cuda")
    o = torch.empty(H, L, d, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
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

    def full():
        C.attention(q, k, v, workspace=ws, out=o, stream=stream)

    def kernel():
        C.attention_int8(qx, sq, kx, sk, vt, out=o, stream=stream, split_ws=part)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        full()
    barrier()
    times = {}
    clk_summary = None
    for name, fn in (("kernel", kernel), ("full", full)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device()) as clk:
            barrier()
            e0.record(stream)
            for _ in range(args.steps):
                fn()
            e1.record(stream)
            barrier()
        times[name] = max_over_ranks(e0.elapsed_time(e1) / 1e3, world) / args.steps
        if name == "kernel":
            clk_summary = clk.summary()
    st, code = C.last_device_status()
    if st != C.OK:
        raise RuntimeError(f"device status {st} (code {code})")
    if rank == 0:
        hbm, bf16, kind = peaks()
        int8_peak = bf16 * INT8_PER_BF16
        half = 2.0 * H * L * L * d          # each of the two products
        ops = 2 * half
        t_tensor = half / (int8_peak * 1e12) + half / (bf16 * 1e12)   # both products at their peaks
        mufu = 16 * 148 * 1.965e9                                      # 2^x per second (SFU, nominal)
        t_exp = H * L * L / mufu
        value = world * ops / times["full"] / 1e12
        line = {
            "metric": ATTN_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": times["full"] * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8+bf16", "data": "synthetic",
            "config": {"workload": f"attention_h{H}_l{L}_d{d}", "heads": H, "Lq": L, "Lk": L, "d": d,
                       "parallelism": f"dp{world} (independent heads and sequences per GPU)",
                       "l2": f"Q, K, V are {H * L * d * 2 / 1e6:.0f} MB each (bf16), O the same"
                             f"{'' if 4 * H * L * d * 2 > 126e6 else ' (together below L2: a small profiling case)'}; the score "
                             f"matrix ({H * L * L * 2 / 1e9:.1f} GB as bf16) is never stored"},
            "roofline": {"bound": "tensor",
                         "kernel": f"attention_kernel (Q K^T, softmax, P V; {attn_launches} launch"
                                   f"{'es: whole units, split units, combine' if attn_launches > 1 else ''})",
                         "achieved": ops / times["kernel"] / 1e12, "peak": ops / t_tensor / 1e12,
                         "unit": "TFLOP/s", "frac": t_tensor / times["kernel"], "traffic": None,
                         "peak_source": f"{kind}: Q K^T at bf16 burst x {INT8_PER_BF16}, P V at the bf16 burst "
                                        f"{bf16} TFLOP/s; the 2^x of the softmax alone would take "
                                        f"{t_exp * 1e3:.3f} ms on the special-function units (nominal 16/clk/SM)"},
            "kernels": {"attention_kernel_us": times["kernel"] * 1e6,
                        "quantise_transpose_us": (times["full"] - times["kernel"]) * 1e6},
            "clocks": clk_summary,
            "gpu_launches": (3 + attn_launches) * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


MLP_METRIC = "ConvRot W8A8 MLP TOPS at M=38656, K=5376, H=21504 (up + GELU + down)"


def run_mlp(args, rank: int, world: int):
    """The 768p MLP step by both routes of its GELU: in the up projection's
    epilogue (then the plain quantiser on the down projection's input), or as
    the down projection's prologue (convrot_linear_act on the plain up
    projection's output).  The line's value is for --mlp-route."""
    import torch
    import torch.distributed as dist
    from w8a8_int8_quantized_block_b200 import convrot as C
    from w8a8_int8_quantized_block_b200 import workloads as W

    spec = W.MLP_768P
    x_cpu, w1_cpu, w2_cpu = W.mlp_inputs(spec)
    x = x_cpu.cuda()
    p1 = C.pack_weight(w1_cpu.cuda(), spec.block)
    p2 = C.pack_weight(w2_cpu.cuda(), spec.block)
    del w1_cpu, w2_cpu
    ws1 = C.alloc_workspace(spec.M, spec.K)
    ws2 = C.alloc_workspace(spec.M, spec.H)
    h = torch.empty(spec.M, spec.H, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(spec.M, spec.K, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def up(gelu):
        C.linear_fused(x, p1, None, gelu=gelu, workspace=ws1, out=h, stream=stream)

    def down(prologue):
        if prologue:
            C.linear_act(h, C.ACT_GELU, p2, None, workspace=ws2, out=y, stream=stream)
        else:
            C.linear_fused(h, p2, None, workspace=ws2, out=y, stream=stream)

    routes = {"epilogue": (lambda: (up(True), down(False))), "prologue": (lambda: (up(False), down(True)))}

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for r in routes.values():
        for _ in range(max(3, args.warmup)):
            r()
    barrier()
    times, kern = {}, {}
    clk_summary = None
    for name in ("epilogue", "prologue"):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device()) as clk:
            barrier()
            e0.record(stream)
            for _ in range(args.steps):
                routes[name]()
            e1.record(stream)
            barrier()
        times[name] = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
        if name == args.mlp_route:
            clk_summary = clk.summary()
        # per launch: up projection, then the down projection's two kernels
        nk = min(args.steps, 50)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nk)]
        barrier()
        for i in range(nk):
            ev[i][0].record(stream)
            up(name == "epilogue")
            ev[i][1].record(stream)
            down(name == "prologue")
            ev[i][2].record(stream)
        barrier()
        kern[name] = {"up_us": sum(e[0].elapsed_time(e[1]) for e in ev) / nk * 1e3,
                      "down_us": sum(e[1].elapsed_time(e[2]) for e in ev) / nk * 1e3}
    st, code = C.last_device_status()
    if st != C.OK:
        raise RuntimeError(f"device status {st} (code {code})")
    if rank == 0:
        hbm, bf16, kind = peaks()
        int8_peak = bf16 * INT8_PER_BF16
        t = times[args.mlp_route]
        value = job_tops(spec.ops, args.steps, world, t)
        line = {
            "metric": MLP_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": spec.name, "M": spec.M, "K": spec.K, "H": spec.H, "block": spec.block,
                       "activation": "gelu", "route": args.mlp_route,
                       "parallelism": f"dp{world} (independent token batches per GPU)",
                       "l2": "inputs larger than L2: h is 1.66 GB per step"},
            "pct_of_int8_peak": round(100.0 * value / world / int8_peak, 2),
            "routes": {n: {"TOPS": job_tops(spec.ops, args.steps, world, times[n]),
                           "ms_per_step": times[n] / args.steps * 1e3, **kern[n]} for n in times},
            "clocks": clk_summary,
            "gpu_launches": 3 * args.steps,  # up (one kernel), down (prologue quantiser + GEMM)
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


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
    if args.rows is not None:
        import dataclasses
        if not args.kernel_only or not 1 <= args.rows <= spec.M:
            raise SystemExit(f"--rows needs --kernel-only and 1 <= ROWS <= {spec.M}")
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
    q, s = ws[:spec.M * spec.K].view(torch.int8).view(spec.M, spec.K), torch.empty(spec.M, device="cuda")
    stream = torch.cuda.current_stream()

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

    if args.kernel_only:
        C.quantize_act(x, spec.block, q, s, stream=stream)
        one = {"fused": step,
               "quant": lambda: C.quantize_act(x, spec.block, q, s, stream=stream),
               "gemm": lambda: C.w8a8_linear(q, s, pw, bias, out=y, stream=stream)}[args.kernel_only]
        for _ in range(args.warmup + args.steps):
            one()
        torch.cuda.synchronize()
        st, code = C.last_device_status()
        if st != C.OK:
            raise RuntimeError(f"device status {st} (code {code})")
        return

    for _ in range(max(3, args.warmup)):
        step()
    barrier()
    st, code = C.last_device_status()
    if st != C.OK:
        raise RuntimeError(f"device status {st} (code {code}) after warm-up")

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
    elapsed_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    st, code = C.last_device_status()
    if st != C.OK:
        raise RuntimeError(f"device status {st} (code {code}) after the timed region")
    if args.context_parallel:
        value = job.ops * args.steps / elapsed_s / 1e12  # strong scaling: the ranks share one job
    else:
        value = job_tops(spec.ops, args.steps, world, elapsed_s)

    # Per-kernel durations, same stream, CUDA events around each launch: the
    # one-kernel step (its ready-counter memset included), then the two
    # kernels of the split path for comparison.
    nk = min(args.steps, 200)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nk)]
    barrier()
    for i in range(nk):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
        C.quantize_act(x, spec.block, q, s, stream=stream)
        ev[i][2].record(stream)
        C.w8a8_linear(q, s, pw, bias, out=y, stream=stream)
        ev[i][3].record(stream)
    barrier()
    t_fused = sum(e[0].elapsed_time(e[1]) for e in ev) / nk / 1e3
    t_quant = sum(e[1].elapsed_time(e[2]) for e in ev) / nk / 1e3
    t_gemm = sum(e[2].elapsed_time(e[3]) for e in ev) / nk / 1e3

    # End to end through the C ABI with host buffers (copies inside the timed region).
    x_host = x_cpu.pin_memory()
    y_host = torch.empty(spec.M, spec.N, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    for _ in range(2):
        C.linear_fused_host(x_host, pw, bias, False, x_dev, ws, y, y_host, stream=stream)
    barrier()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        C.linear_fused_host(x_host, pw, bias, False, x_dev, ws, y, y_host, stream=stream)
    e1.record(stream)
    barrier()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    e2e_value = job_tops(spec.ops, args.e2e_steps, world, e2e_s)
    st, code = C.last_device_status()
    if st != C.OK:
        raise RuntimeError(f"device status {st} (code {code}) after the end-to-end leg")

    if rank == 0:
        hbm, bf16, kind = peaks()
        int8_peak = bf16 * INT8_PER_BF16
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
                "linear_fused_kernel": {"us": t_fused * 1e6, "TOPS": achieved, "frac_of_int8_peak": achieved / int8_peak},
                "igemm_pair_kernel (split path)": {"us": t_gemm * 1e6, "TOPS": spec.ops / t_gemm / 1e12,
                                                   "frac_of_int8_peak": spec.ops / t_gemm / 1e12 / int8_peak},
                "rotate_quant_kernel (split path)": {"us": t_quant * 1e6, "GB/s": quant_bytes / t_quant / 1e9,
                                 "frac_of_hbm": quant_bytes / t_quant / 1e9 / hbm, "hbm_peak_gbs": hbm,
                                 "algorithmic_bytes_per_launch": quant_bytes},
            },
            "clocks": clk.summary(),
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": spec.M * spec.K * 2,
                    "d2h_bytes_per_step": spec.M * spec.N * 2, "steps": args.e2e_steps,
                    "path": "convrot_linear_fused_host (pinned host x -> device -> linear -> pinned host y)"},
            "gpu_launches": args.steps,  # one linear_fused_kernel per step (plus a 604-byte memset node)
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(spec)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
