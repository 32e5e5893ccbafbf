#!/usr/bin/env python
"""Benchmark of the MXFP4 expert-FFN MoE layer on B200.

A step is one pass of the layer's hot path over one batch: top-k routing of the
router logits, then the expert layer (permute, gather, gate_up grouped GEMM with
clamped SwiGLU, down grouped GEMM with bias and routing weight, combine), all
through the library's C ABI.  The default workload is the gpt-oss-20b-shaped
prefill layer (T=4096 tokens, hidden 2880, intermediate 2880, 32 experts, top-4,
MXFP4 weights) with seeded synthetic inputs.  Secondary measurements (standalone
dequant, decode, gpt-oss-120b-shaped skewed layers) ride in the same JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank runs an independent replica of the layer
(the path has no cross-GPU exchange); value = all tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

DEFAULT_WORKLOAD = "20b_prefill_T4096"
# DRAM bytes (read + write) of one gate_up launch of the default workload, measured by
# ncu (dram__bytes_read.sum + dram__bytes_write.sum) on the kernel whose source has the
# SHA-256 prefix below; reported only while the source still matches, else null.
GATE_UP_DRAM_BYTES = 469.6e6
GATE_UP_SOURCE_SHA = "e44c8fabd3ce3bff"
GATE_UP_SOURCE = os.path.join(ROOT, "mxfp4_expert_ffn_moe_b200", "csrc", "gemm_swap.cuh")


def kernel_source_sha(path: str) -> str:
    import hashlib
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def gate_up_traffic():
    """The captured DRAM bytes per gate_up launch, or None when the kernel's source has
    changed since the capture."""
    try:
        return GATE_UP_DRAM_BYTES if kernel_source_sha(GATE_UP_SOURCE) == GATE_UP_SOURCE_SHA else None
    except OSError:
        return None
METRIC = "MoE layer tokens/s (prefill)"
# algorithmic weight bytes of one gpt-oss-20b/120b expert (gate_up + down: packed
# codes, E8M0 scales, fp32 biases)
EXPERT_BYTES_2880 = (5760 * 1440 + 5760 * 90 + 5760 * 4) + (2880 * 1440 + 2880 * 90 + 2880 * 4)
# the NVFP4 variant: E4M3 scales per 16 elements, plus three fp32 weight_scale_2
NVFP4_EXPERT_BYTES_2880 = (5760 * 1440 + 5760 * 180 + 5760 * 4) + (2880 * 1440 + 2880 * 180 + 2880 * 4) + 12


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while it runs."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        # raw samples go to a temporary file; the summary rides in the JSON line
        self.path = os.path.join(tempfile.gettempdir(), f"moe_bench_clocks_{os.getpid()}.csv")
        self.window = None

    def mark(self, t0: float, t1: float):
        """Wall-clock bounds (time.time()) of the timed region."""
        self.window = (t0, t1)

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.device_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        import datetime
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        n_all = 0
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                vals = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            n_all += 1
            if self.window and not (self.window[0] - 0.05 <= ts <= self.window[1] + 0.05):
                continue
            sm.append(vals[0])
            smax.append(vals[1])
            power.append(vals[2])
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"no samples in the timed "
                                                                     f"window ({n_all} outside)"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "power_w_max": float(max(power)), "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- device layer

class DeviceLayer:
    def __init__(self, layer, device):
        import torch
        self.layer = layer
        self.device = device

        def d(a, dtype=None):
            if a is None:
                return None
            t = torch.from_numpy(np.ascontiguousarray(a))
            return (t.view(dtype) if dtype is not None else t).to(device)

        self.x = d(layer.x_bits, torch.bfloat16)
        self.logits = d(layer.logits)
        self.gu_blocks, self.gu_scales = d(layer.gate_up.blocks), d(layer.gate_up.scales)
        self.gu_bias = d(layer.gate_up_bias)
        self.d_blocks, self.d_scales = d(layer.down.blocks), d(layer.down.scales)
        self.d_bias = d(layer.down_bias)
        self.nv = layer.fmt == "nvfp4"
        self.gu_s2, self.d_s2 = d(layer.gate_up.scale2), d(layer.down.scale2)
        L = layer
        import mxfp4_expert_ffn_moe_b200 as moe
        self.moe = moe
        self.ws = torch.empty(moe.moe_mxfp4_workspace_size(L.T, L.H, L.I, L.E, L.k),
                              dtype=torch.uint8, device=device)
        self.ids = torch.empty((L.T, L.k), dtype=torch.int32, device=device)
        self.w = torch.empty((L.T, L.k), dtype=torch.float32, device=device)
        self.out = torch.empty((L.T, L.H), dtype=torch.bfloat16, device=device)
        self.flags = moe.MOE_FLAG_WEIGHT_ON_INPUT if L.weight_on_input else 0

    def step(self, x=None, logits=None, out=None):
        L, moe = self.layer, self.moe
        out = self.out if out is None else out
        moe.moe_route(self.logits if logits is None else logits, L.k, ids=self.ids, weights=self.w)
        if self.nv:
            moe.moe_nvfp4_forward_ex(self.x if x is None else x, self.ids, self.w, self.gu_blocks,
                                     self.gu_scales, self.gu_s2, self.gu_bias, self.d_blocks,
                                     self.d_scales, self.d_s2, self.d_bias, alpha=L.alpha,
                                     limit=L.limit, out=out, flags=self.flags, workspace=self.ws)
            return out
        moe.moe_mxfp4_forward_ex(self.x if x is None else x, self.ids, self.w, self.gu_blocks,
                                 self.gu_scales, self.gu_bias, self.d_blocks, self.d_scales,
                                 self.d_bias, alpha=L.alpha, limit=L.limit, out=out,
                                 flags=self.flags, workspace=self.ws)
        return out


def distinct_experts(logits, k):
    # count of distinct experts among the top-k of each row (workload statistic)
    top = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    return int(np.unique(top).size)


def time_steps(fn, steps, stream, flush=None):
    """Device time (ms) of `steps` calls of fn, with optional L2 flush outside the events."""
    import torch
    if flush is None:
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)
    total = 0.0
    evs = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    for a, b in evs:
        total += a.elapsed_time(b)
    return total


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its device time and all get the
    max (NCCL on the GPUs; any backend whose tensors live on `device`)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time (weak scaling:
    each replica runs the full workload)."""
    return world * tokens_per_rank * steps / (ms_max * 1e-3)


def graph_of(fn, stream):
    """fn captured into a CUDA graph (the library's launches, programmatic dependent
    launch edges included), or None with the reason when capture is not possible."""
    import torch
    try:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()                                  # warm the host-side caches outside capture
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g, None
    except Exception as exc:                      # noqa: BLE001 - reported, eager timing stays
        try:
            torch.cuda.synchronize()
        except Exception:                         # noqa: BLE001
            pass
        return None, f"{type(exc).__name__}: {exc}"[:200]


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The CPU oracle, timed on this host's cores, on bounded samples of the workload."""
    import oracle
    from mxfp4_expert_ffn_moe_b200.workloads import workload
    oracle.build()
    layer = workload(args.workload)
    threads = oracle.num_threads()

    def one_step(n_tok, offset):
        tokens = (np.arange(n_tok, dtype=np.int64) + offset) % layer.T
        ids, w = oracle.route(layer.logits[tokens], layer.k)
        sub_x = layer.x_bits[tokens]
        oracle.forward_tokens(sub_x, ids, w, layer.gate_up.blocks, layer.gate_up.scales,
                              layer.gate_up_bias, layer.down.blocks, layer.down.scales,
                              layer.down_bias, alpha=layer.alpha, limit=layer.limit)

    t0 = time.perf_counter()
    one_step(threads, 0)
    t_threads = time.perf_counter() - t0                   # wall time of `threads` tokens
    budget = 150.0 / max(1, args.steps + args.warmup)      # seconds per step
    n_tok = max(1, min(threads * 4, int(threads * budget / max(t_threads, 1e-6))))
    for i in range(args.warmup):
        one_step(n_tok, 7 * i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one_step(n_tok, 131 * i + 1)
    dt = time.perf_counter() - t0
    value = n_tok * args.steps / dt
    cores = min(threads, n_tok)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "T": layer.T, "H": layer.H, "I": layer.I,
                   "E": layer.E, "k": layer.k},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_tok} tokens of the {args.workload} layer per step "
                                   f"(route + forward, decode-on-the-fly double precision)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm

def cpu_baseline_leg(layer, name):
    import oracle
    oracle.build()
    threads = oracle.num_threads()
    n_tok = 3 * threads
    tokens = np.linspace(0, layer.T - 1, n_tok).astype(np.int64)
    t0 = time.perf_counter()
    ids, w = oracle.route(layer.logits[tokens], layer.k)
    oracle.forward_tokens(layer.x_bits[tokens], ids, w, layer.gate_up.blocks, layer.gate_up.scales,
                          layer.gate_up_bias, layer.down.blocks, layer.down.scales, layer.down_bias,
                          alpha=layer.alpha, limit=layer.limit)
    dt = time.perf_counter() - t0
    return {"value": n_tok / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_tok} of the {layer.T} tokens of {name} (route + forward), {dt:.1f} s"}


def extra_measurements(device, stream, peaks):
    """Standalone dequant, decode and the gpt-oss-120b-shaped layers (secondary)."""
    import torch
    import mxfp4_expert_ffn_moe_b200 as moe
    from mxfp4_expert_ffn_moe_b200.workloads import make_dequant_bank, make_nvfp4_dequant_bank, workload
    res = {}
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    flush_read = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    flush_sink = torch.empty((), dtype=torch.float32, device=device)

    def flush():
        # write 256 MB (evicts every line), then read another 256 MB: the L2 (126 MB) ends
        # up holding clean lines of neither the inputs nor the flush writes, so the timed
        # kernel neither finds its data in L2 nor pays for writing the flush back
        flush_buf.fill_(1)
        torch.sum(flush_read, dim=0, out=flush_sink)

    # standalone dequant of the gpt-oss-20b expert bank (both projections)
    gu, dn = make_dequant_bank(seed=0)
    banks = []
    nbytes = 0
    for bank in (gu, dn):
        E, N, K = bank.shape
        b = torch.from_numpy(bank.blocks).to(device)
        s = torch.from_numpy(bank.scales).to(device)
        o = torch.empty((E, N, K), dtype=torch.bfloat16, device=device)
        banks.append((b, s, o))
        nbytes += bank.blocks.nbytes + bank.scales.nbytes + E * N * K * 2

    def deq():
        for b, s, o in banks:
            moe.mxfp4_dequantize(b, s, out=o)

    for _ in range(3):
        deq()
    moe.moe_profile_read()
    moe.moe_profile_enable(True)
    ms = time_steps(deq, 10, stream, flush) / 10
    prof = moe.moe_profile_read()
    moe.moe_profile_enable(False)
    kms = prof["dequant"][0] / max(1, prof["dequant"][1]) * 2
    res["dequant_20b_bank"] = {
        "GB/s": nbytes / (ms * 1e-3) / 1e9, "ms": ms, "bytes": nbytes,
        "kernel_GB/s": nbytes / (kms * 1e-3) / 1e9,
        "hbm_frac_of_measured": nbytes / (kms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "hbm_frac_of_8TBps": nbytes / (kms * 1e-3) / 1e9 / 8000.0}
    del banks
    torch.cuda.empty_cache()

    # standalone dequant of the NVFP4 bank of the same shapes (E4M3 per 16, weight_scale_2)
    gu, dn = make_nvfp4_dequant_bank(seed=0)
    banks = []
    nbytes = 0
    for bank in (gu, dn):
        E, N, K = bank.shape
        b = torch.from_numpy(bank.blocks).to(device)
        s = torch.from_numpy(bank.scales).to(device)
        s2 = torch.from_numpy(bank.scale2).to(device)
        o = torch.empty((E, N, K), dtype=torch.bfloat16, device=device)
        banks.append((b, s, s2, o))
        nbytes += bank.blocks.nbytes + bank.scales.nbytes + bank.scale2.nbytes + E * N * K * 2

    def deq_nv():
        for b, s, s2, o in banks:
            moe.nvfp4_dequantize(b, s, s2, out=o)

    for _ in range(3):
        deq_nv()
    moe.moe_profile_read()
    moe.moe_profile_enable(True)
    ms = time_steps(deq_nv, 10, stream, flush) / 10
    prof = moe.moe_profile_read()
    moe.moe_profile_enable(False)
    kms = prof["dequant"][0] / max(1, prof["dequant"][1]) * 2
    res["nvfp4_dequant_20b_bank"] = {
        "GB/s": nbytes / (ms * 1e-3) / 1e9, "ms": ms, "bytes": nbytes,
        "kernel_GB/s": nbytes / (kms * 1e-3) / 1e9,
        "hbm_frac_of_measured": nbytes / (kms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del banks
    torch.cuda.empty_cache()

    # dequant-on-copy from host memory: the gpt-oss-20b down bank in page-locked host
    # memory, decoded by the kernel through its device mapping, against a plain
    # copy-engine transfer of the same packed bytes (the host link's rate)
    _, dn = make_dequant_bank(seed=0)
    E, N, K = dn.shape
    hb = torch.from_numpy(dn.blocks).pin_memory()
    hs = torch.from_numpy(dn.scales).pin_memory()
    o = torch.empty((E, N, K), dtype=torch.bfloat16, device=device)
    db = torch.empty(dn.blocks.shape, dtype=torch.uint8, device=device)
    ds = torch.empty(dn.scales.shape, dtype=torch.uint8, device=device)

    def from_host():
        moe.mxfp4_dequantize_from_host(hb, hs, out=o)

    def copy_packed():
        db.copy_(hb, non_blocking=True)
        ds.copy_(hs, non_blocking=True)

    for _ in range(2):
        from_host()
        copy_packed()
    ms_h = time_steps(from_host, 5, stream) / 5
    ms_c = time_steps(copy_packed, 5, stream) / 5
    packed = dn.blocks.nbytes + dn.scales.nbytes
    res["dequant_from_host_20b_down"] = {
        "ms": ms_h, "packed_bytes": packed, "bf16_bytes_written": E * N * K * 2,
        "host_link_GB/s": packed / (ms_h * 1e-3) / 1e9,
        "copy_engine_GB/s_same_bytes": packed / (ms_c * 1e-3) / 1e9,
        "frac_of_copy_engine": ms_c / ms_h}
    del hb, hs, o, db, ds
    torch.cuda.empty_cache()

    # router linear layer fused with routing (tensor-core GEMM + top-k epilogue)
    from mxfp4_expert_ffn_moe_b200.workloads import router_workload
    for name in ("router_20b_T8", "router_20b_T4096", "router_120b_T8192"):
        r = router_workload(name)
        T, H = r.x_bits.shape
        E = r.w_bits.shape[0]
        x = torch.from_numpy(r.x_bits).view(torch.bfloat16).to(device)
        w = torch.from_numpy(r.w_bits).view(torch.bfloat16).to(device)
        b = torch.from_numpy(r.bias).to(device)
        ids = torch.empty((T, r.k), dtype=torch.int32, device=device)
        wt = torch.empty((T, r.k), dtype=torch.float32, device=device)

        def rr():
            moe.moe_router_route(x, w, b, r.k, ids=ids, weights=wt)

        for _ in range(3):
            rr()
        ms_eager = time_steps(rr, 20, stream, flush) / 20
        g, why = graph_of(rr, stream)
        ms = time_steps(g.replay, 20, stream, flush) / 20 if g is not None else ms_eager
        nbytes = 2 * T * H + 2 * E * H + 4 * E + 8 * T * r.k
        res[name] = {"us": ms * 1e3, "tokens/s": T / (ms * 1e-3), "GB/s": nbytes / (ms * 1e-3) / 1e9,
                     "TFLOP/s": 2.0 * T * E * H / (ms * 1e-3) / 1e12, "bytes": nbytes,
                     "timed": "CUDA graph replay" if g is not None else "eager (graph capture failed)",
                     "us_eager_calls": ms_eager * 1e3}
        if why:
            res[name]["graph_error"] = why
        del g, x, w, b, ids, wt
    torch.cuda.empty_cache()

    for name, steps, do_flush in [("20b_decode_T1", 50, True), ("20b_decode_T8", 50, True),
                                  ("20b_decode_T64", 30, True), ("120b_zipf_T256", 20, True),
                                  ("120b_zipf_T8192", 5, False), ("nvfp4_20b_decode_T8", 50, True),
                                  ("nvfp4_20b_prefill_T4096", 20, False)]:
        layer = workload(name)
        dl = DeviceLayer(layer, device)
        for _ in range(3):
            dl.step()
        # the step as it runs (kernels overlapping under programmatic dependent launch),
        # replayed from a CUDA graph so that the host's per-call work (argument marshalling,
        # tensor-map encoding, launches) does not stand in for device time on these short
        # steps; the eager figure rides beside it; then a second, eager pass with every
        # stage bracketed by events for the breakdown
        ms_eager = time_steps(dl.step, steps, stream, flush if do_flush else None) / steps
        g, why = graph_of(dl.step, stream)
        ms = time_steps(g.replay, steps, stream, flush if do_flush else None) / steps if g is not None else ms_eager
        moe.moe_profile_read()
        moe.moe_profile_enable(True)
        time_steps(dl.step, steps, stream, flush if do_flush else None)
        prof = moe.moe_profile_read()
        moe.moe_profile_enable(False)
        touched = distinct_experts(layer.logits, layer.k)
        wbytes = touched * (NVFP4_EXPERT_BYTES_2880 if layer.fmt == "nvfp4" else EXPERT_BYTES_2880)
        entry = {"tokens/s": layer.T / (ms * 1e-3), "ms": ms, "touched_experts": touched,
                 "weight_GB/s": wbytes / (ms * 1e-3) / 1e9,
                 "hbm_frac_of_measured": wbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                 "stage_ms": {k: v[0] / steps for k, v in prof.items() if v[1]},
                 "timed": "CUDA graph replay" if g is not None else "eager (graph capture failed)",
                 "ms_eager_calls": ms_eager}
        if why:
            entry["graph_error"] = why
        del g
        flops = 2.0 * layer.T * layer.k * layer.H * 3 * layer.I
        entry["tflops"] = flops / (ms * 1e-3) / 1e12
        res[name] = entry
        del dl
        torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    from mxfp4_expert_ffn_moe_b200 import build as moe_build
    if rank == 0:
        moe_build.build()
    if world > 1:
        dist.barrier()
    import mxfp4_expert_ffn_moe_b200 as moe
    from mxfp4_expert_ffn_moe_b200.workloads import workload
    moe.load_library()

    peaks = measured_peaks()
    layer = workload(args.workload)
    L = layer
    dl = DeviceLayer(layer, device)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    with ClockSampler(uuid) as clocks:
        time.sleep(0.5)                      # let nvidia-smi start sampling
        for _ in range(args.warmup):
            dl.step()
        torch.cuda.synchronize()
        moe.moe_profile_read()
        barrier()
        torch.cuda.synchronize()
        # the timed region: K steps as a user runs them, no events between kernels
        # (consecutive kernels overlap under programmatic dependent launch)
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        wall0 = time.time()
        ev0.record(stream)
        for _ in range(args.steps):
            dl.step()
        ev1.record(stream)
        torch.cuda.synchronize()
        clocks.mark(wall0, time.time())
        launches = moe.moe_profile_read()
        barrier()
        # the same K steps again with events around the dominant kernel only, for the
        # roofline: an event pair between two kernels keeps them from overlapping, so
        # this pass runs a little slower and its time is reported apart
        moe.moe_profile_enable_stages(["gate_up"])
        ev2 = torch.cuda.Event(enable_timing=True)
        ev3 = torch.cuda.Event(enable_timing=True)
        ev2.record(stream)
        for _ in range(args.steps):
            dl.step()
        ev3.record(stream)
        torch.cuda.synchronize()
        moe.moe_profile_enable(False)
        time.sleep(0.2)
    barrier()
    ms_total = ev0.elapsed_time(ev1)
    ms_profiled = ev2.elapsed_time(ev3)
    prof = moe.moe_profile_read()
    ms_total = max_over_ranks(ms_total, world, device)
    value = job_throughput(L.T, args.steps, world, ms_total)
    gpu_launches = sum(v[1] for v in launches.values())

    # end to end through the public API: pinned host inputs -> device -> layer -> host.
    # Every step copies its x and logits in and its output out (full bytes each step);
    # the copies of neighbouring steps overlap the layer on two copy streams, with two
    # device buffer slots (step i uses slot i % 2).
    x_host = torch.from_numpy(L.x_bits).view(torch.bfloat16).pin_memory()
    lg_host = torch.from_numpy(L.logits).pin_memory()
    out_host = [torch.empty((L.T, L.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(dl.x) for _ in range(2)]
    lg_dev = [torch.empty_like(dl.logits) for _ in range(2)]
    out_dev = [torch.empty_like(dl.out) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of the slot copied in
    ev_done = [torch.cuda.Event() for _ in range(2)]    # layer finished with the slot
    ev_out = [torch.cuda.Event() for _ in range(2)]     # output of the slot copied out

    def e2e_run(n, ev_start=None, ev_end=None):
        if ev_start is not None:
            ev_start.record(s_in)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[b])
                x_dev[b].copy_(x_host, non_blocking=True)
                lg_dev[b].copy_(lg_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])
            with torch.cuda.stream(stream):
                dl.step(x=x_dev[b], logits=lg_dev[b], out=out_dev[b])
                ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                ev_out[b].record(s_out)
        if ev_end is not None:
            ev_end.record(s_out)

    # as many steps as the device-timed region, so that both run in the same clock state
    # (a short pass after a power-capped region runs at recovered clocks)
    e2e_steps = max(3, args.steps)
    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    moe.moe_profile_read()
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    e2e_value = job_throughput(L.T, e2e_steps, world, e2e_ms)

    # roofline of the dominant kernel (gate_up grouped GEMM), from the live events
    gu_ms, gu_n = prof["gate_up"]
    gu_avg = gu_ms / max(1, gu_n)
    gu_flops = 2.0 * L.T * L.k * L.H * (2 * L.I)
    achieved = gu_flops / (gu_avg * 1e-3) / 1e12
    # the burst peak fits a kernel running at full clocks; once the clocks sampled in the
    # timed window sit below them (the 1 kW power cap, or a region longer than a second)
    # the sustained peak is the one that matches
    clk = clocks.summary()
    capped = (clk.get("sm_mhz") is not None and clk.get("sm_max_mhz") and
              clk["sm_mhz"] < 0.95 * clk["sm_max_mhz"])
    long_region = ms_total > 1000.0 or bool(capped)
    peak = peaks["bf16_tflops_sustained"] if long_region else peaks["bf16_tflops"]
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": gate_up_traffic(), "kernel": "gate_up grouped GEMM",
                "peak_kind": f"{peaks['source']} bf16 {'sustained' if long_region else 'burst'}",
                "frac_of_2250_spec": achieved / 2250.0,
                "frac_of_burst": achieved / peaks["bf16_tflops"],
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "flops_per_launch": gu_flops, "avg_launch_ms": gu_avg,
                "measured_in": "a second pass of the same steps with events around each gate_up launch",
                "ms_per_step_of_that_pass": ms_profiled / args.steps}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; MXFP4 codes uniform, E8M0 118..126, N(0,1) activations)",
        "config": {"workload": args.workload, "T": L.T, "H": L.H, "I": L.I, "E": L.E, "k": L.k,
                   "global_batch": world * L.T, "parallelism": f"replicas x{world}",
                   "l2": "inputs exceed L2 (424 MB of resident expert weights per step)"},
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(L.x_bits.nbytes + L.logits.nbytes),
                "d2h_bytes_per_step": int(L.T * L.H * 2)},
        "gpu_launches": int(gpu_launches),
        "stage_ms_per_step": {k: v[0] / args.steps for k, v in prof.items() if v[0]},
        "roofline": roofline,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_extra:
        line["extra"] = extra_measurements(device, stream, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(layer, args.workload)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference(args)
        return
    run_ours(args)


if __name__ == "__main__":
    main()
