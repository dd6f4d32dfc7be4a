"""Benchmark of the anti-quant weight GEMM (W4A16, per-group g=128, m=k=n=4096) on B200.

One step = phase 1 (host: validate + plan) and phase 2 (the GEMM kernel) of
wqmm_get_workspace_size / wqmm_run on one batch of synthetic, seeded input,
with the weight pre-packed (the packing is weight preparation, done once).

  value     : TFLOP/s (2*m*n*k / device time), inputs resident in HBM, L2
              flushed before every timed step (a 512 MB write, outside the
              timed interval), CUDA events on the launching stream, max over ranks.
  e2e       : the same metric through the same C-ABI calls with HOST buffers:
              every step copies its inputs from pinned host memory and reads
              the output back, all inside the timed interval.
  roofline  : the GEMM kernel against its bound: the measured dense bf16 peak
              (anti-quant and non-quantised GEMMs: bf16/f16 MMAs), the int8
              peak measured in this run (the int8 GEMM), or the measured HBM
              bandwidth, whichever roofline time is larger for the workload.
  cpu_baseline / --impl reference : the CPU oracle timed on a bounded sample.

N > 1 (torchrun): N independent replicas (one problem per GPU, no collective on
the data path), weak scaling; value = all ranks' FLOPs / max rank time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE = "w4a16_g128_bf16_4096x4096x4096"
METRIC = "anti-quant GEMM TFLOP/s & % of roofline (W4A16 g128, m=k=n=4096), 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["weight_quantized_gemm_anti_b200/csrc/kernels_wqmm.cu",
                  "weight_quantized_gemm_anti_b200/csrc/kernels_smallm.cu",
                  "weight_quantized_gemm_anti_b200/csrc/wqmm_common.cuh",
                  "weight_quantized_gemm_anti_b200/csrc/ptx.cuh",
                  "weight_quantized_gemm_anti_b200/csrc/kernels_qmm.cu",
                  "weight_quantized_gemm_anti_b200/csrc/kernels_aux.cu"]


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments and with whitespace collapsed, so that
    the hash follows the code, not its documentation."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    """Identifies the kernel code a profile was taken on (comments ignored)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def load_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, only if it was taken
    on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ schedule
def wqmm_schedule(m: int, n: int, k: int, sms: int, nonquant: bool = False) -> dict:
    """The anti-quant GEMM's schedule as the library's phase 1 chooses it with
    no tuning overrides (a restatement of its planner, checked against the
    library's workspace sizes in the CPU tests): m tile, stream-K or whole
    tiles, and whether a fix-up kernel follows the GEMM.  ``nonquant``: a
    16-bit weight of the x1 dtype, which always runs on the general kernel."""
    bn = 16 if m <= 16 else 32 if m <= 32 else 64 if m <= 64 else 128 if m <= 128 else 256
    num_nb = -(-n // 128)
    if 256 < m <= 512 and -(-m // 256) * num_nb < sms and -(-m // 128) * num_nb <= sms:
        bn = 128  # the 128-row split is cheaper than the 256-row one here
    kt = -(-k // 64)
    tiles = -(-m // bn) * num_nb
    out = {"bn": bn, "stream_k": False, "inline": False, "partial_bytes": 0, "flag_bytes": 0,
           "kernel": "smallm" if bn <= 32 and not nonquant else "general", "grid": min(tiles, sms)}
    if k == 0:
        return out
    if bn <= 32 and not nonquant:
        # small-m kernel: stream-K over every tile, >= 16 k steps per CTA
        unit = 2 if kt % 2 == 0 else 1
        T = tiles * kt // unit
        grid = max(1, min(sms, -(-(T * unit) // 16)))
        owner = lambda s: ((s + 1) * grid - 1) // T
        ms = max(owner((r * kt + kt - 1) // unit) - owner(r * kt // unit) + 1 for r in range(tiles))
        out.update(stream_k=True, inline=ms <= 4, grid=grid)
        if ms > 1:
            out.update(partial_bytes=tiles * ms * bn * 128 * 4, flag_bytes=tiles * ms * 8 if ms <= 4 else 0)
        return out
    if kt < 2:
        return out
    rem = tiles % sms
    if tiles < sms:
        dp = 0
    elif bn < 128 and rem > 0 and rem * 100 <= 85 * sms:
        dp = tiles - rem
    else:
        return out
    unit = 2 if (bn >= 128 and kt % 2 == 0) else 1
    split = tiles - dp
    T = split * kt // unit
    grid = sms if dp > 0 else min(T, sms)
    skg = min(T, grid)
    owner = lambda s: ((s + 1) * skg - 1) // T
    ms = max(owner((r * kt + kt - 1) // unit) - owner(r * kt // unit) + 1 for r in range(split))
    out.update(stream_k=True, inline=ms <= 4, partial_bytes=split * ms * bn * 128 * 4,
               flag_bytes=split * ms * 8 if ms <= 4 else 0, grid=grid)
    return out


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self):
        self.proc = None
        self.path = None
        self.skip = 0

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # the timed region starts once the sampler is writing (at most 5 s)
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None and os.path.getsize(self.path) == 0:
            time.sleep(0.02)
        self.skip = sum(1 for _ in open(self.path))  # samples taken before the timed region

    def stop(self, gpu_index: int):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            lines = f.readlines()

        def parse(rows):
            sm, mx, reasons = [], 0.0, set()
            for line in rows:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9 or not parts[0].isdigit() or int(parts[0]) != gpu_index:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
            return sm, mx, reasons

        # samples taken during the timed region; a region shorter than the
        # sampling interval falls back to the samples taken just before it
        sm, mx, reasons = parse(lines[self.skip:])
        if not sm:
            sm, mx, reasons = parse(lines)
        os.unlink(self.path)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workload labels
def describe_weight(case) -> str:
    """Human-readable weight/quantisation label of a workload."""
    if not hasattr(case, "wdt"):
        dq = "per-tensor" if case.dequant_scale.size == 1 else "per-channel"
        pt = " + per-token scale" if case.pertoken_scale is not None else ""
        return f"int8 x int8, {dq} {case.dq_dtype} dequantScale{pt}"
    if case.mode == "none":
        return f"{case.wdt} (non-quantised), no antiquant"
    w = {"i4": "int4", "i8": "int8", "fp8": "fp8-e4m3"}[case.wdt]
    mode = {"tensor": "per-tensor", "channel": "per-channel", "group": f"per-group g={case.group_size}"}[case.mode]
    off = " + offset" if case.offset is not None else ""
    return f"{w} packed, {mode} scale{off}"


def arithmetic_dtype(case) -> str:
    """The type the MMAs compute in: the activation type, or int8."""
    return "i8" if not hasattr(case, "wdt") else case.act


def roofline_bound(flops: float, nbytes: float, tensor_peak_tflops: float, hbm_gbs: float) -> str:
    """'tensor' when the tensor-core time of the FLOPs exceeds the HBM time of
    the algorithmic bytes, else 'hbm'."""
    return "tensor" if flops / (tensor_peak_tflops * 1e12) >= nbytes / (hbm_gbs * 1e9) else "hbm"


def measure_int8_peak(device: str, iters: int = 20):
    """Dense int8 tensor throughput measured on this GPU: torch._int_mm (the
    vendor library) and this library's int8 GEMM, both on an 8192^3 problem
    (per-tensor dequantScale, no bias, x3 or per-token scale).  Returns the
    larger, with both figures."""
    import torch
    import workloads as WL
    import weight_quantized_gemm_anti_b200 as W
    from weight_quantized_gemm_anti_b200 import cases as C

    s = 8192
    flops = 2.0 * s * s * s
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(iters):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    out = {"shape": f"{s}x{s}x{s}", "iters": iters}
    a = torch.randint(-127, 128, (s, s), dtype=torch.int8, device=device)
    bt = torch.randint(-127, 128, (s, s), dtype=torch.int8, device=device)
    try:
        ms = timed(lambda: torch._int_mm(a, bt))
        out["torch_int_mm_tops"] = round(flops / (ms * 1e-3) / 1e12, 1)
    except RuntimeError as e:  # no int8 library GEMM for this device / build
        out["torch_int_mm_tops"] = None
        out["torch_int_mm_error"] = str(e).splitlines()[0][:120]
    del a, bt
    case = WL.make_qmm_case(name="int8_peak", x1_shape=(s, s), n=s, out="bf16", bias=False, x3=False,
                            pertoken=False, dq_per_tensor=True, seed=99)
    d = C.qmm_to_device(case, device=device)
    D = W.desc
    descs = (D(d.x1), d.x2_desc, None, None, d.dq_desc, None, None, "sum", 0, 1, D(d.out))
    st, ws, ex = W.qmm_get_workspace_size(*descs)
    W.check(st)
    W.wqmm_executor_destroy(ex)
    wsb = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)

    def own():
        st, ws2, ex2 = W.qmm_get_workspace_size(*descs)
        W.check(st)
        W.check(W.qmm_run(wsb.data_ptr(), ws2, ex2, stream))

    ms = timed(own)
    out["qmm_tops"] = round(flops / (ms * 1e-3) / 1e12, 1)
    del d, wsb
    torch.cuda.empty_cache()
    cands = [v for v in (out["torch_int_mm_tops"], out["qmm_tops"]) if v]
    out["peak_tops"] = max(cands)
    out["peak_from"] = "torch._int_mm" if out["peak_tops"] == out["torch_int_mm_tops"] else "this library's int8 GEMM"
    return out


def workload_roofline(prob, peaks, int8_peak):
    """(bound, peak, unit, peak_source) of a workload's roofline."""
    if prob.int8:
        tpeak = int8_peak["peak_tops"] if int8_peak else 2.0 * peaks["bf16_tflops"]
        tsrc = (f"int8 measured in this run ({int8_peak['peak_from']}, {int8_peak['shape']})" if int8_peak
                else "2 x measured bf16 burst (nominal ratio)")
    else:
        tpeak, tsrc = peaks["bf16_tflops"], "bf16 burst"
    bound = roofline_bound(prob.flops, prob.bytes, tpeak, peaks["hbm_gbs"])
    if bound == "tensor":
        return bound, tpeak, "TFLOP/s", tsrc
    return bound, peaks["hbm_gbs"], "GB/s", "HBM copy"


def algorithmic_bytes(case) -> float:
    """Each input read once plus the output written once (int4 = 0.5 B)."""
    c = case
    if not hasattr(c, "wdt"):
        b = c.m * c.k + c.k * c.n + c.m * c.n * 2
        b += 0 if c.bias is None else 4 * c.n
        b += c.dequant_scale.nbytes + (0 if c.pertoken_scale is None else 4 * c.m)
        b += 0 if c.x3 is None else 2 * c.m * c.n
        return b
    wbytes = {"i4": 0.5, "i8": 1.0, "fp8": 1.0, "f16": 2.0, "bf16": 2.0}[c.wdt]
    b = c.m * c.k * 2 + c.k * c.n * wbytes + c.m * c.n * 2
    b += (0 if c.scale is None else c.scale.nbytes) + (0 if c.offset is None else c.offset.nbytes)
    b += 0 if c.bias is None else 2 * c.n
    b += 0 if c.x3 is None else 2 * c.m * c.n
    return b


# ------------------------------------------------------------------ GPU arm
class Problem:
    """One workload resident on the device, with prebuilt ABI descriptors."""

    def __init__(self, name, device):
        import torch
        import workloads as WL
        import weight_quantized_gemm_anti_b200 as W
        from weight_quantized_gemm_anti_b200 import cases as C

        self.W, self.C, self.torch = W, C, torch
        self.name = name
        self.case = WL.workload(name)
        self.int8 = not hasattr(self.case, "wdt")
        if self.int8:
            self.dev = C.qmm_to_device(self.case, device=device)
        else:
            self.dev = C.wqmm_to_device(self.case, device=device)
        torch.cuda.synchronize()
        c = self.case
        self.flops = 2.0 * c.m * c.n * c.k
        self.bytes = algorithmic_bytes(self.case)
        d = self.dev
        D = W.desc
        if self.int8:
            self.descs = (D(d.x1), d.x2_desc, None if d.bias is None else D(d.bias),
                          None if d.x3 is None else D(d.x3), d.dq_desc, None if d.pt is None else D(d.pt),
                          None, "sum", 0, 1, D(d.out))
        else:
            self.descs = (D(d.x1), d.x2_desc, None if d.bias is None else D(d.bias), d.scale_desc, d.offset_desc,
                          None if d.x3 is None else D(d.x3), None, "sum", 0, 1, d.group_size, D(d.out))
        st, ws, ex = self.phase1()
        W.wqmm_executor_destroy(ex)
        self.ws_size = ws
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)

    def phase1(self):
        if self.int8:
            return self.W.qmm_get_workspace_size(*self.descs)
        return self.W.wqmm_get_workspace_size(*self.descs)

    def phase2(self, ex, stream):
        if self.int8:
            return self.W.qmm_run(self.ws.data_ptr(), self.ws_size, ex, stream)
        return self.W.wqmm_run(self.ws.data_ptr(), self.ws_size, ex, stream)

    def launches_per_step(self):
        if self.int8:
            return 1
        c = self.case
        k = c.k
        m = 1
        for d in c.x1_shape[:-1]:
            m *= d
        sched = wqmm_schedule(m, c.n, k, self.torch.cuda.get_device_properties(0).multi_processor_count,
                              nonquant=c.mode == "none")
        # the GEMM, plus the fix-up kernel when split tiles are reduced by one
        return 1 + (1 if sched["stream_k"] and not sched["inline"] else 0)


def time_device(prob: Problem, steps: int, warmup: int, flush_bytes: int):
    """Per-step device time of phase 1 + phase 2 (events on the launching stream,
    L2 flushed before each step outside the timed interval)."""
    torch = prob.torch
    stream = torch.cuda.current_stream()
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device=prob.ws.device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    host_p1 = 0.0
    for i in range(warmup + steps):
        flush.fill_(i & 0xFF)  # > L2: evicts the previous step's inputs and outputs
        t0 = time.perf_counter()
        st, ws, ex = prob.phase1()
        host_p1 += time.perf_counter() - t0 if i >= warmup else 0.0
        prob.W.check(st)
        if i >= warmup:
            evs[i - warmup][0].record(stream)
        prob.W.check(prob.phase2(ex, stream))
        if i >= warmup:
            evs[i - warmup][1].record(stream)
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in evs]
    return times, host_p1 / max(steps, 1)


def time_e2e(prob: Problem, steps: int, warmup: int):
    """The same calls with host buffers: H2D of every input from pinned memory,
    phase 1 + phase 2, D2H of the output, inside one timed interval per step."""
    torch = prob.torch
    d = prob.dev
    stream = torch.cuda.current_stream()
    if prob.int8:
        dev_inputs = [d.x1, d.packed, d.bias, d.dq, d.pt, d.x3]
    else:
        dev_inputs = [d.x1, d.packed, d.scale, d.offset, d.bias, d.x3]
    pairs = []
    for t in dev_inputs:
        if t is None:
            continue
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t if t.is_contiguous() else t.contiguous())
        pairs.append((h, t))
    out_h = torch.empty(d.out.shape, dtype=d.out.dtype, pin_memory=True)
    h2d = sum(h.numel() * h.element_size() for h, _ in pairs)
    d2h = out_h.numel() * out_h.element_size()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    total = 0.0
    for i in range(warmup + steps):
        start.record(stream)
        for h, t in pairs:
            if t.is_contiguous():
                t.copy_(h, non_blocking=True)
            else:
                t.copy_(h.to(t.device, non_blocking=True))
        st, ws, ex = prob.phase1()
        prob.W.check(st)
        prob.W.check(prob.phase2(ex, stream))
        out_h.copy_(d.out, non_blocking=True)
        end.record(stream)
        end.synchronize()
        if i >= warmup:
            total += start.elapsed_time(end)
    return total / steps, h2d, d2h


def cpu_baseline(name: str, rows: int):
    """The oracle as it stands on the host cores, on `rows` output rows of the workload."""
    import numpy as np
    import oracle
    import workloads as WL

    case = WL.workload(name)
    r = np.arange(0, case.m, max(1, case.m // rows))[:rows]
    oracle.build()
    t0 = time.perf_counter()
    if hasattr(case, "wdt"):
        oracle.wqmm(case, rows=r)
    else:
        oracle.qmm(case, rows=r)
    dt = time.perf_counter() - t0
    flops = 2.0 * len(r) * case.n * case.k
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(r)} of {case.m} output rows x all {case.n} columns of {name} ({dt:.1f} s)"}


def max_over_ranks(values, device):
    """Elementwise max of per-rank values over the process group (identity for one rank).
    Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def replica_throughput(flops_per_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s of `world` independent replicas that each ran `steps`
    steps, timed by the slowest rank (max_ms, device time)."""
    return flops_per_step * world * steps / (max_ms * 1e-3) / 1e12


def gpu_arm(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    import weight_quantized_gemm_anti_b200 as W
    W.build()
    peaks, peak_src = load_peaks()
    prob = Problem(args.config, f"cuda:{local}")
    flush_bytes = 512 << 20

    sampler = ClockSampler()
    if rank == 0:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    times, host_p1 = time_device(prob, args.steps, args.warmup, flush_bytes)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop(local) if rank == 0 else None
    max_ms = max_over_ranks([sum(times)], "cuda")[0]
    st, code = W.wqmm_device_error(reset=True)
    if st != 0 or code != 0:
        raise RuntimeError(f"device error word {code}")

    e2e_ms, h2d, d2h = time_e2e(prob, max(3, min(args.steps, 20)), 2)
    e2e_ms = max_over_ranks([e2e_ms], "cuda")[0]

    extra = {}
    int8_peak = None
    if rank == 0 and world == 1 and not args.no_extra:
        import workloads as WL
        int8_peak = measure_int8_peak(f"cuda:{local}")
        for nm in WL.WORKLOAD_NAMES:
            if nm == args.config:
                continue
            p2 = Problem(nm, f"cuda:{local}")
            # launch-latency-sized problems: a larger sample for a stable median
            nsteps = 1000 if p2.flops < 1e8 else max(args.extra_steps, 50)
            tt, _ = time_device(p2, nsteps, 3, flush_bytes)
            tt.sort()
            ms = tt[len(tt) // 2]  # median step
            bound, peak, unit, src = workload_roofline(p2, peaks, int8_peak)
            ent = {"ms_per_step": round(ms, 5), "stat": f"median of {len(tt)} steps",
                   "weight": describe_weight(p2.case), "dtype": arithmetic_dtype(p2.case),
                   "tflops": round(p2.flops / (ms * 1e-3) / 1e12, 2),
                   "gbs": round(p2.bytes / (ms * 1e-3) / 1e9, 1), "launches_per_step": p2.launches_per_step()}
            ach = ent["tflops"] if bound == "tensor" else ent["gbs"]
            ent["roofline"] = {"bound": bound, "achieved": ach, "peak": peak, "unit": unit,
                               "frac": round(ach / peak, 4), "peak_source": src}
            extra[nm] = ent
            del p2
            torch.cuda.empty_cache()

    if rank == 0 and prob.int8 and int8_peak is None:
        int8_peak = measure_int8_peak(f"cuda:{local}")
    if rank == 0:
        ms_step = max_ms / args.steps
        value = replica_throughput(prob.flops, world, args.steps, max_ms)
        bound, peak, unit, src = workload_roofline(prob, peaks, int8_peak)
        achieved = (prob.flops / (ms_step * 1e-3) / 1e12 if bound == "tensor"
                    else prob.bytes / (ms_step * 1e-3) / 1e9)
        traffic = load_traffic(args.config)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": arithmetic_dtype(prob.case),
            "data": "synthetic (seeded; shapes/distributions of the workload)",
            "config": {"workload": args.config, "m": prob.case.m, "k": prob.case.k, "n": prob.case.n,
                       "weight": describe_weight(prob.case), "l2": "flushed before every step "
                       "(512 MB write outside the timed interval)", "parallelism": f"replicas x{world}"},
            "e2e": {"value": round(replica_throughput(prob.flops, world, 1, e2e_ms), 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": prob.launches_per_step() * args.steps,
            "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_source": f"{peak_src} {src}" if "measured in this run" not in src else src},
            "clocks": clocks,
            "host_phase1_us": round(host_p1 * 1e6, 1),
        }
        if extra:
            line["configs_measured"] = extra
        if int8_peak:
            line["int8_peak_measured"] = int8_peak
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.config, args.cpu_rows)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def reference_arm(args):
    """The CPU oracle timed as the reference arm on the same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    import workloads as WL

    case = WL.workload(args.config)
    oracle.build()
    rows_per_step = args.ref_rows
    rng = np.random.default_rng(0)
    total, flops = 0.0, 0.0
    for i in range(args.warmup + args.steps):
        r = np.sort(rng.choice(case.m, size=rows_per_step, replace=False))
        t0 = time.perf_counter()
        oracle.wqmm(case, rows=r) if hasattr(case, "wdt") else oracle.qmm(case, rows=r)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            total += dt
            flops += 2.0 * rows_per_step * case.n * case.k
    value = flops / total / 1e12
    sample = f"{rows_per_step} random output rows x all {case.n} columns of {args.config} per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {"workload": args.config, "m": case.m, "k": case.k, "n": case.n},
            "cpu_baseline": {"kind": "oracle", "cores": oracle.num_threads(), "sample": sample, "value": value,
                             "unit": "TFLOP/s"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="wqmm", choices=["wqmm", "reference"])
    ap.add_argument("--config", default=HEADLINE)
    ap.add_argument("--extra-steps", type=int, default=100)
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads and the int8 peak leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=1024)
    ap.add_argument("--ref-rows", type=int, default=8)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
