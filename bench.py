"""Benchmark: bf16 exact-attention forward + backward TFLOP/s on B200.

One step = one pass of the whole hot path over one batch: ``fa_fwd`` (fused forward) then
``fa_bwd`` (preprocess, fused backward, dQ convert) on the same seeded synthetic inputs.
Default workload: the throughput-sweep shape at N = 4096, H = 16, d = 128, non-causal,
B = 16384 / N = 4 per GPU (the size at which the throughput targets are stated).

FLOP accounting: forward 4*B*H*N^2*d (halved when causal), backward 2.5x the forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --row fwd-d256|bwd-d256|fwd-fp8|decode|varlen [...]   (the further entry points)

With N > 1 launch one process per GPU with torch.distributed.run; each rank runs its own
batch of the same shape (weak scaling, no collective on the data path) and rank 0 prints one
JSON line with the time taken as the maximum over ranks.

``--impl reference`` times the fp64 CPU oracle (the plain definition of attention) on a bounded
sample of the same workload; it is a deliberately slow reference, not a target.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "bf16 attention fwd/bwd TFLOP/s and % of B200 dense BF16 tensor peak"
NOMINAL_PEAK_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
WORKLOADS = {
    "sweep-N4096-H16-d128": lambda: workloads.sweep(4096, 16, 128, False),
    "sweep-N4096-H16-d128-causal": lambda: workloads.sweep(4096, 16, 128, True),
    "sweep-N16384-H16-d128": lambda: workloads.sweep(16384, 16, 128, False),
    "sweep-N4096-H32-d64": lambda: workloads.sweep(4096, 32, 64, False),
    "gpt2-small": workloads.gpt2_small,
    "bert-large-padded": workloads.bert_large_padded,
    # grouped-query attention: 32 query heads over 8 key/value heads
    "gqa-N4096-H32-kv8-d128": lambda: workloads.Workload(
        "gqa non-causal B2 H32 Hkv8 N4096 d128", 2, 32, 4096, 128, False, 1040, H_kv=8),
}
for _N in workloads.SWEEP_N:
    for _H, _d in workloads.SWEEP_HD:
        for _c in (False, True):
            WORKLOADS.setdefault(f"sweep-N{_N}-H{_H}-d{_d}" + ("-causal" if _c else ""),
                                 (lambda N=_N, H=_H, d=_d, c=_c: workloads.sweep(N, H, d, c)))
SWEEP_NAMES = [f"sweep-N{N}-H{H}-d{d}" + ("-causal" if c else "")
               for N in workloads.SWEEP_N for (H, d) in workloads.SWEEP_HD for c in (False, True)]
DEFAULT_WORKLOAD = "sweep-N4096-H16-d128"


def flops_per_step(w: workloads.Workload, seqlens=None) -> tuple[float, float]:
    """(forward, backward) algorithmic FLOPs for one batch; padded keys count as skipped work."""
    if seqlens is not None:
        keys = float(sum(int(x) for x in seqlens))  # effective: sum_b L_b instead of B*N
        fwd = 4.0 * w.H * w.N * keys * w.d
    else:
        fwd = 4.0 * w.B * w.H * w.N * w.N * w.d
    if w.causal:
        fwd /= 2.0
    return fwd, 2.5 * fwd


def tensor_peak(peaks: dict, src: str, timed_s: float, clocks: dict | None) -> tuple[float, str]:
    """The bf16 tensor peak a kernel timed in this run is set against.  The measured burst
    figure (a GEMM timed alone) applies to a timed region shorter than a second whose clock
    record shows no power capping; a longer or power-capped region is set against the
    sustained figure (a seconds-long GEMM loop under the power cap)."""
    reasons = (clocks or {}).get("reasons", [])
    if timed_s < 1.0 and "sw_power_cap" not in reasons:
        return float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])), f"{src} bf16 burst"
    return (float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])),
            f"{src} bf16 sustained")


def roofline_tensor(kernel: str, achieved: float, kernel_ms: float, peaks: dict, src: str,
                    timed_s: float, clocks: dict | None, traffic, scale: float = 1.0) -> dict:
    """Roofline object of a tensor-bound kernel: `frac` against the peak that applies (see
    tensor_peak), plus both measured fractions and the share of the nominal dense peak.
    `scale` multiplies the bf16 peaks (2 for e4m3, the nominal ratio)."""
    peak, which = tensor_peak(peaks, src, timed_s, clocks)
    burst = scale * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sust = scale * float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak *= scale
    source = which + (" (MEASURED_PEAKS.json)" if src == "measured" else " (no MEASURED_PEAKS.json)")
    if scale != 1.0:
        source += f" x {scale:g} (nominal e4m3 / bf16 ratio)"
    return {"kernel": kernel, "bound": "tensor", "achieved": round(achieved, 2),
            "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "peak_source": source,
            "frac_of_burst": round(achieved / burst, 4),
            "frac_of_sustained": round(achieved / sust, 4),
            "pct_of_2250": round(100.0 * achieved / (scale * NOMINAL_PEAK_TFLOPS), 2),
            "kernel_ms": round(kernel_ms, 4), "traffic": traffic}


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "fa_fwd_kernel": ("fa_fwd.cu", "sm100.cuh", "fa_internal.h"),
    "fa_fwd_persist_kernel": ("fa_fwd.cu", "sm100.cuh", "fa_internal.h"),
    "fa_bwd_kernel": ("fa_bwd.cu", "fa_bwd_common.cuh", "sm100.cuh", "fa_internal.h"),
    "fa_bwd_persist_kernel": ("fa_bwd.cu", "fa_bwd_common.cuh", "sm100.cuh", "fa_internal.h"),
    "fa_fwd_d256_kernel": ("fa_fwd_d256.cu", "sm100.cuh", "fa_internal.h"),
    "fa_fwd_fp8_kernel": ("fa_fwd_fp8.cu", "fa_fwd_fp8.h", "sm100.cuh", "fa_internal.h"),
    "fa_bwd_d256_kernel": ("fa_bwd_d256.cu", "fa_bwd_common.cuh", "sm100.cuh", "fa_internal.h"),
    "fa_decode_kernel": ("fa_decode.cu", "fa_decode.h", "sm100.cuh", "fa_internal.h"),
}


def main_kernels(w: workloads.Workload, num_sms: int) -> tuple[str, str]:
    """Names of the fused forward and backward kernels the library launches for `w`: the
    persistent forward for launches without key lengths with more units than SMs and at most
    32 key blocks per tile (causal or not), the persistent backward when every unit costs the
    same (no causal mask either) and is at most 16 query steps long; the one-CTA-per-unit
    kernels otherwise."""
    equal = not w.causal and w.pad_range is None
    fwd_units = -(-w.N // 256) * w.H * w.B
    bwd_units = -(-w.N // 128) * w.kv_heads * w.B
    steps = (w.H // w.kv_heads) * -(-w.N // 128)  # query steps of one backward unit
    fwd = ("fa_fwd_persist_kernel"
           if w.pad_range is None and fwd_units > num_sms and -(-w.N // 128) <= 32
           else "fa_fwd_kernel")
    bwd = ("fa_bwd_persist_kernel" if equal and bwd_units > num_sms and steps <= 16
           else "fa_bwd_kernel")
    return fwd, bwd


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources a kernel is compiled from (a recorded traffic figure is only valid
    for the exact code it was measured on)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "io_aware_exact_16_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dram_traffic(kernel: str, workload: str) -> float | None:
    """Per-launch DRAM bytes of `kernel` at `workload` from the committed ncu summaries
    (profiles/traffic.json, keyed "kernel @ workload"), or None when the kernel's sources have
    changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return None
    entry = data.get(f"{kernel} @ {workload}", {})
    if entry.get("source_hash") != kernel_source_hash(kernel):
        return None
    return float(entry["dram_bytes_per_launch"])


def _pct(sorted_vals, q):
    """q-th percentile (nearest rank) of an ascending list."""
    i = min(len(sorted_vals) - 1, max(0, int(round(q / 100 * (len(sorted_vals) - 1)))))
    return sorted_vals[i]


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = open(f"/tmp/fa_bench_clocks_{os.getpid()}.csv", "w", buffering=1)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
            return self
        # wait (up to 3 s) for the first sample so the timed region is covered
        t0 = time.time()
        while time.time() - t0 < 3.0 and self.proc.poll() is None:
            try:
                if os.path.getsize(self.out.name) > 0:
                    break
            except OSError:
                break
            time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.out is not None:
            self.out.close()

    def summary(self) -> dict | None:
        if self.proc is None or self.out is None:
            return None
        try:
            with open(self.out.name) as f:
                lines = [l.strip() for l in f if l.strip()]
            os.unlink(self.out.name)
        except OSError:
            return None
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(sms)}


def rank_workload(w: workloads.Workload, rank: int) -> workloads.Workload:
    """The batch rank `rank` processes: same shape, its own seed (independent batches)."""
    return workloads.Workload(w.name, w.B, w.H, w.N, w.d, w.causal, w.seed + 7919 * rank, w.std,
                              w.pad_range, H_kv=w.H_kv)


def reduce_max(values: list[float], world: int, device=None) -> list[float]:
    """Element-wise maximum over ranks (the job takes as long as its slowest rank)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def run_ours(args, rank: int, world: int, local_rank: int) -> dict | None:
    import io_aware_exact_16_b200 as fa

    w = WORKLOADS[args.workload]()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    # Each rank draws its own batch (seed offset by rank): weak scaling over independent batches.
    inp = workloads.make_inputs(rank_workload(w, rank))
    sl_cpu = inp.seqlens
    fwd_flops, bwd_flops = flops_per_step(w, sl_cpu)
    step_flops = fwd_flops + bwd_flops

    pinned = {n: getattr(inp, n).pin_memory() for n in ("q", "k", "v", "do")}
    q, k, v, do = (pinned[n].to(dev, non_blocking=True) for n in ("q", "k", "v", "do"))
    sl = sl_cpu.to(dev) if sl_cpu is not None else None
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.forward(q, k, v, causal=w.causal, seqlens=sl, scale=w.scale, out=o, lse=lse)
        fa.backward(q, k, v, o, do, lse, causal=w.causal, seqlens=sl, scale=w.scale,
                    dq=dq, dk=dk, dv=dv, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.check_device_error(dev) != 0:
        raise RuntimeError("device error flag set during warm-up")

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- timed region: per-pass CUDA events on the launching stream, plus events the library
    # records right around the fused forward and fused backward kernels (time_next_kernel)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e in (x for row in kev for x in row):
        e.record(stream)  # creates the CUDA events before the timed region
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            fa.time_next_kernel(kev[s][0], kev[s][1])
            fa.forward(q, k, v, causal=w.causal, seqlens=sl, scale=w.scale, out=o, lse=lse)
            ev[s][1].record(stream)
            fa.time_next_kernel(kev[s][2], kev[s][3])
            fa.backward(q, k, v, o, do, lse, causal=w.causal, seqlens=sl, scale=w.scale,
                        dq=dq, dk=dk, dv=dv, workspace=ws)
            ev[s][2].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    elapsed_ms = start.elapsed_time(end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    step_ms = sorted(e[0].elapsed_time(e[2]) for e in ev)  # per step, for the spread
    fwd_kernel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in kev)
    bwd_kernel_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in kev)
    status = fa.check_device_error(dev)
    if status != 0:
        raise RuntimeError(f"device error flag {status} after the timed region")

    # ---- end-to-end through the public API: every step copies its inputs in from pinned host
    # memory and its results (O, dQ, dK, dV) out to pinned host memory.  The copies run on their
    # own streams over two device buffer sets, so step s+1's inputs travel while step s
    # computes and step s-1's results travel back, as a training input pipeline would do.
    def e2e_leg():
        def device_set():
            return {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
                    "do": torch.empty_like(do), "o": torch.empty_like(o),
                    "lse": torch.empty_like(lse), "dq": torch.empty_like(dq),
                    "dk": torch.empty_like(dk), "dv": torch.empty_like(dv),
                    "ws": torch.empty_like(ws)}

        sets = [device_set(), device_set()]
        outs = ("o", "dq", "dk", "dv")
        host_out = [{n: torch.empty(sets[0][n].shape, dtype=sets[0][n].dtype).pin_memory()
                     for n in outs} for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in pinned.values())
        d2h = sum(host_out[0][n].numel() * host_out[0][n].element_size() for n in outs)
        e2e_steps = max(1, min(args.steps, 10))
        copy_in = torch.cuda.Stream(dev)
        copy_out = torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_done = [ev() for _ in range(e2e_steps)]
        comp_done = [ev() for _ in range(e2e_steps)]
        out_done = [ev() for _ in range(e2e_steps)]
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy_in.wait_event(e0)
        for s_ in range(e2e_steps):
            bset = sets[s_ % 2]
            with torch.cuda.stream(copy_in):
                if s_ >= 2:
                    copy_in.wait_event(comp_done[s_ - 2])  # step s-2 has read this set's inputs
                for n in ("q", "k", "v", "do"):
                    bset[n].copy_(pinned[n], non_blocking=True)
                in_done[s_].record(copy_in)
            stream.wait_event(in_done[s_])
            if s_ >= 2:
                stream.wait_event(out_done[s_ - 2])  # step s-2's results have left this set
            fa.forward(bset["q"], bset["k"], bset["v"], causal=w.causal, seqlens=sl, scale=w.scale,
                       out=bset["o"], lse=bset["lse"])
            fa.backward(bset["q"], bset["k"], bset["v"], bset["o"], bset["do"], bset["lse"],
                        causal=w.causal, seqlens=sl, scale=w.scale, dq=bset["dq"], dk=bset["dk"],
                        dv=bset["dv"], workspace=bset["ws"])
            comp_done[s_].record(stream)
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(comp_done[s_])
                for n in outs:
                    host_out[s_ % 2][n].copy_(bset[n], non_blocking=True)
                out_done[s_].record(copy_out)
        stream.wait_event(out_done[e2e_steps - 1])
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = e0.elapsed_time(e1)
        if fa.check_device_error(dev) != 0:
            raise RuntimeError("device error flag set in the end-to-end leg")
        return e2e_ms, h2d, d2h, e2e_steps

    if args.skip_e2e:
        e2e_ms, h2d, d2h, e2e_steps = 0.0, 0, 0, 0
    else:
        e2e_ms, h2d, d2h, e2e_steps = e2e_leg()

    elapsed_ms, e2e_ms, fwd_ms, bwd_ms, fwd_kernel_ms, bwd_kernel_ms = reduce_max(
        [elapsed_ms, e2e_ms, fwd_ms, bwd_ms, fwd_kernel_ms, bwd_kernel_ms], world, dev)
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    value = step_flops * args.steps * world / (elapsed_ms * 1e-3) / 1e12
    ms_per_step = elapsed_ms / args.steps
    bwd_tflops = bwd_flops / (bwd_ms * 1e-3) / 1e12
    fwd_tflops = fwd_flops / (fwd_ms * 1e-3) / 1e12
    # every backward GEMM (recompute S, dP, dV, dK, dQ) runs in the fused kernel
    bwd_kernel_tflops = bwd_flops / (bwd_kernel_ms * 1e-3) / 1e12
    fwd_kernel_tflops = fwd_flops / (fwd_kernel_ms * 1e-3) / 1e12
    clock_summary = clocks.summary()
    timed_s = elapsed_ms * 1e-3
    wname = args.workload
    fwd_name, bwd_name = main_kernels(w, torch.cuda.get_device_properties(dev).multi_processor_count)
    traffic = dram_traffic(bwd_name, wname)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) draws rounded to bf16)",
        "pct_of_dense_bf16_peak": round(100.0 * value / world / NOMINAL_PEAK_TFLOPS, 2),
        "config": {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.kv_heads, "N": w.N, "d": w.d,
                   "causal": w.causal, "padded": w.pad_range is not None,
                   "per_gpu_batch": w.B, "global_batch": w.B * world,
                   "parallelism": f"independent batches x{world}",
                   "l2": "inputs larger than L2: Q,K,V,O,dO,dQ,dK,dV are %.0f MB each per GPU"
                         % (w.B * w.H * w.N * w.d * 2 / 1e6)},
        "passes": {"fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
                   "fwd_tflops": round(fwd_tflops, 2), "bwd_tflops": round(bwd_tflops, 2),
                   "fwd_pct_of_2250": round(100 * fwd_tflops / NOMINAL_PEAK_TFLOPS, 2),
                   "bwd_pct_of_2250": round(100 * bwd_tflops / NOMINAL_PEAK_TFLOPS, 2),
                   "step_ms_p10_p50_p90": [round(_pct(step_ms, q), 4) for q in (10, 50, 90)]},
        "roofline": roofline_tensor(f"{bwd_name} (fused backward: all five backward GEMMs)",
                                    bwd_kernel_tflops, bwd_kernel_ms, peaks, peak_src, timed_s,
                                    clock_summary, traffic),
        "roofline_fwd": roofline_tensor(fwd_name, fwd_kernel_tflops, fwd_kernel_ms, peaks,
                                        peak_src, timed_s, clock_summary,
                                        dram_traffic(fwd_name, wname)),
        "e2e": {"value": round(step_flops * e2e_steps * world / (max(e2e_ms, 1e-9) * 1e-3) / 1e12, 2),
                "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "copies": "pinned host memory, own streams, overlapped "
                                              "with the neighbouring steps' compute"},
        "gpu_launches": 4 * args.steps,
        "clocks": clock_summary,
    }
    if args.skip_e2e:
        del line["e2e"]
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp, args.cpu_heads)
    return line


def cpu_baseline(w: workloads.Workload, inp, heads: int) -> dict:
    """The oracle as it stands, fwd + bwd on a bounded sample of heads of the same workload."""
    import oracle

    oracle.build()
    total = w.B * w.H
    picks = workloads.seeded_sample(w.seed + 99, total, heads)
    t0 = time.perf_counter()
    flops = 0.0
    for flat in picks:
        b, h = divmod(flat, w.H)
        L = int(inp.seqlens[b]) if inp.seqlens is not None else w.N
        hk = h // (w.H // w.kv_heads)
        oracle.head_bwd(inp.q[b, h], inp.k[b, hk], inp.v[b, hk], inp.do[b, h], w.scale, w.causal,
                        L)
        f = 4.0 * w.N * L * w.d * (0.5 if w.causal else 1.0)
        flops += 3.5 * f
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(),
            "kind": "oracle",
            "sample": f"fp64 C oracle fwd+bwd on {len(picks)} of {total} heads ({dt:.1f} s)"}


def run_reference(args, rank: int, world: int) -> dict | None:
    if rank != 0:
        return None
    import oracle

    oracle.build()
    w = WORKLOADS[args.workload]()
    inp = workloads.make_inputs(w)
    fwd_flops, bwd_flops = flops_per_step(w, inp.seqlens)
    head_flops = (fwd_flops + bwd_flops) / (w.B * w.H)  # one head per step (bounded sample)
    heads = workloads.seeded_sample(w.seed + 99, w.B * w.H, args.warmup + args.steps)

    def one(flat):
        b, h = divmod(flat, w.H)
        L = int(inp.seqlens[b]) if inp.seqlens is not None else w.N
        hk = h // (w.H // w.kv_heads)
        oracle.head_bwd(inp.q[b, h], inp.k[b, hk], inp.v[b, hk], inp.do[b, h], w.scale, w.causal,
                        L)

    for i in range(args.warmup):
        one(heads[i % len(heads)])
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(heads[(args.warmup + i) % len(heads)])
    dt = time.perf_counter() - t0
    value = head_flops * args.steps / dt / 1e12
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.kv_heads, "N": w.N, "d": w.d, "causal": w.causal},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(),
                         "kind": "oracle",
                         "sample": f"one head of {w.B * w.H} per step, fp64 fwd+bwd"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------- further rows
# Each row below is one more entry point of the path, measured the same way as the default
# training step: W warm-up steps, K timed steps between events on the launching stream (plus
# the library's events around the row's main kernel), clocks sampled meanwhile, an end-to-end
# leg with the step's inputs copied in from pinned host memory and its result copied out, and
# the oracle timed beside it on a bounded sample.
import dataclasses  # noqa: E402
from typing import Callable  # noqa: E402


@dataclasses.dataclass
class Row:
    config: dict                 # workload description for the JSON line
    metric: str
    unit: str                    # "TFLOP/s" or "GB/s"
    dtype: str
    amount: float                # algorithmic FLOPs or bytes per step (whole step)
    kernel: str                  # the main kernel the library brackets with events
    kernel_amount: float         # algorithmic FLOPs or bytes of that kernel per step
    bound: str                   # "tensor" or "hbm"
    peak: float
    peak_source: str
    step: Callable               # step(mark): one step; mark() right before the main kernel's call
    h2d: list                    # (device tensor, pinned host tensor) copied in per e2e step
    d2h: list                    # (device tensor, pinned host tensor) copied out per e2e step
    launches: int                # our kernels per step
    cpu: Callable[[], dict]      # the oracle on a bounded sample: {"amount", "seconds", "sample"}
    traffic_key: str | None = None
    peak_scale: float = 1.0      # tensor rows: multiple of the bf16 peaks (2 for e4m3)


def _pinned_pair(t: torch.Tensor):
    return t, torch.empty(t.shape, dtype=t.dtype).pin_memory()


def _peaks():
    peaks, src = load_peaks()
    bf16 = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return bf16, hbm, src


def row_fwd_d256(rank: int, dev) -> Row:
    import io_aware_exact_16_b200 as fa
    import oracle
    w = workloads.Workload("d256 fwd non-causal B2 H16 N4096 d256", 2, 16, 4096, 256, False,
                           1050 + 7919 * rank)
    inp = workloads.make_inputs(w, with_grad=False)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    flops = 4.0 * w.B * w.H * w.N * w.N * w.d
    bf16, _, src = _peaks()

    def cpu():
        heads = workloads.seeded_sample(w.seed + 5, w.B * w.H, 2)
        t0 = time.perf_counter()
        for flat in heads:
            b, h = divmod(flat, w.H)
            oracle.head_fwd(inp.q[b, h], inp.k[b, h], inp.v[b, h], w.scale, False)
        return {"amount": flops / (w.B * w.H) * len(heads), "seconds": time.perf_counter() - t0,
                "sample": f"fp64 C oracle forward on {len(heads)} of {w.B * w.H} heads"}

    return Row(config={"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "causal": False, "l2": "Q,K,V,O are 67 MB each"},
               metric="bf16 attention forward TFLOP/s at head dim 256", unit="TFLOP/s",
               dtype="bf16", amount=flops, kernel="fa_fwd_d256_kernel", kernel_amount=flops,
               bound="tensor", peak=bf16, peak_source=f"{src} bf16 sustained",
               step=lambda mark: (mark(), fa.forward(q, k, v, scale=w.scale, out=o, lse=lse)),
               h2d=[(q, inp.q.pin_memory()), (k, inp.k.pin_memory()), (v, inp.v.pin_memory())],
               d2h=[_pinned_pair(o)], launches=1, cpu=cpu, traffic_key="fa_fwd_d256_kernel")


def row_bwd_d256(rank: int, dev) -> Row:
    import io_aware_exact_16_b200 as fa
    import oracle
    w = workloads.Workload("d256 bwd non-causal B2 H16 N4096 d256", 2, 16, 4096, 256, False,
                           1080 + 7919 * rank)
    inp = workloads.make_inputs(w)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    o, lse = fa.forward(q, k, v, scale=w.scale)
    dq, dk, dv = (torch.empty_like(t) for t in (q, k, v))
    ws = torch.empty(fa.bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
    flops = 2.5 * 4.0 * w.B * w.H * w.N * w.N * w.d  # five GEMMs; the recompute is not counted
    bf16, _, src = _peaks()

    def cpu():
        heads = workloads.seeded_sample(w.seed + 5, w.B * w.H, 1)
        t0 = time.perf_counter()
        for flat in heads:
            b, h = divmod(flat, w.H)
            oracle.head_bwd(inp.q[b, h], inp.k[b, h], inp.v[b, h], inp.do[b, h], w.scale, False)
        return {"amount": flops / (w.B * w.H) * len(heads), "seconds": time.perf_counter() - t0,
                "sample": f"fp64 C oracle backward on {len(heads)} of {w.B * w.H} heads"}

    o_h, lse_h = o.cpu().pin_memory(), lse.cpu().pin_memory()
    return Row(config={"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "causal": False, "l2": "Q,K,V,O,dO,dQ,dK,dV are 67 MB each"},
               metric="bf16 attention backward TFLOP/s at head dim 256", unit="TFLOP/s",
               dtype="bf16", amount=flops, kernel="fa_bwd_d256_kernel", kernel_amount=flops,
               bound="tensor", peak=bf16, peak_source=f"{src} bf16 sustained",
               step=lambda mark: (mark(), fa.backward(q, k, v, o, do, lse, scale=w.scale, dq=dq,
                                                      dk=dk, dv=dv, workspace=ws)),
               h2d=[(q, inp.q.pin_memory()), (k, inp.k.pin_memory()), (v, inp.v.pin_memory()),
                    (do, inp.do.pin_memory()), (o, o_h), (lse, lse_h)],
               d2h=[_pinned_pair(dq), _pinned_pair(dk), _pinned_pair(dv)], launches=3, cpu=cpu,
               traffic_key="fa_bwd_d256_kernel")


def row_fwd_fp8(rank: int, dev) -> Row:
    import io_aware_exact_16_b200 as fa
    import oracle
    w = workloads.Workload("fp8 fwd non-causal B4 H16 N4096 d128", 4, 16, 4096, 128, False,
                           1060 + 7919 * rank)
    f = workloads.make_fp8_inputs(w)
    q, k, v = (t.to(dev) for t in (f.q, f.k, f.v))
    qd, kd, vd = (t.to(dev) for t in (f.q_descale, f.k_descale, f.v_descale))
    o = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    flops = 4.0 * w.B * w.H * w.N * w.N * w.d
    bf16, _, src = _peaks()

    def cpu():
        heads = workloads.seeded_sample(w.seed + 5, w.B * w.H, 2)
        t0 = time.perf_counter()
        for flat in heads:
            b, h = divmod(flat, w.H)
            oracle.attention_fwd_fp8(f.q[b:b + 1, h:h + 1], f.k[b:b + 1, h:h + 1],
                                     f.v[b:b + 1, h:h + 1], f.q_descale[b:b + 1, h:h + 1],
                                     f.k_descale[b:b + 1, h:h + 1],
                                     f.v_descale[b:b + 1, h:h + 1], w.scale, False)
        return {"amount": flops / (w.B * w.H) * len(heads), "seconds": time.perf_counter() - t0,
                "sample": f"fp64 oracle on the dequantised inputs, {len(heads)} of "
                          f"{w.B * w.H} heads"}

    # e4m3 tensor peak = measured bf16 peak x the nominal fp8 / bf16 ratio (4.5 / 2.25)
    return Row(config={"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "causal": False, "l2": "Q,K,V 34 MB each (e4m3) + O 67 MB"},
               metric="fp8 (e4m3) attention forward TFLOP/s", unit="TFLOP/s", dtype="e4m3",
               amount=flops, kernel="fa_fwd_fp8_kernel", kernel_amount=flops, bound="tensor",
               peak=2.0 * bf16, peak_source=f"{src} bf16 sustained x 2 (nominal e4m3/bf16 ratio)",
               step=lambda mark: (mark(), fa.forward_fp8(q, k, v, qd, kd, vd, scale=w.scale,
                                                         out=o, lse=lse)),
               h2d=[(q, f.q.pin_memory()), (k, f.k.pin_memory()), (v, f.v.pin_memory())],
               d2h=[_pinned_pair(o)], launches=1, cpu=cpu, traffic_key="fa_fwd_fp8_kernel",
               peak_scale=2.0)


def row_decode(rank: int, dev) -> Row:
    import io_aware_exact_16_b200 as fa
    import oracle
    B, H, H_kv, Nq, N, d = 8, 32, 8, 1, 8192, 128
    g = torch.Generator().manual_seed(1070 + 7919 * rank)
    q_h = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16)
    k_h = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16)
    v_h = torch.randn((B, H_kv, N, d), generator=g).to(torch.bfloat16)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    splits = fa.decode_num_splits(B, H, H_kv, Nq, N, d)
    ws = torch.empty(max(1, int(fa.decode_workspace_size(B, H, Nq, d, splits))),
                     dtype=torch.uint8, device=dev)
    cache_bytes = 2.0 * B * H_kv * N * d * 2
    step_bytes = cache_bytes + 2.0 * B * H * Nq * d * 2 + 4.0 * B * H * Nq
    _, hbm, src = _peaks()

    def cpu():
        t0 = time.perf_counter()
        oracle.attention_decode(q_h[:1], k_h[:1], v_h[:1], d ** -0.5, False)
        return {"amount": step_bytes / B, "seconds": time.perf_counter() - t0,
                "sample": f"fp64 oracle decode of 1 of {B} sequences (all heads)"}

    return Row(config={"workload": f"decode B{B} H{H} Hkv{H_kv} Nq{Nq} N{N} d{d}", "B": B,
                       "H": H, "H_kv": H_kv, "Nq": Nq, "N": N, "d": d, "splits": splits,
                       "l2": "KV cache 268 MB > L2"},
               metric="decode attention HBM GB/s (KV-cache read)", unit="GB/s", dtype="bf16",
               amount=step_bytes, kernel="fa_decode_kernel", kernel_amount=cache_bytes,
               bound="hbm", peak=hbm, peak_source=f"{src} copy bandwidth",
               step=lambda mark: (mark(), fa.decode(q, k, v, splits=splits, out=o, lse=lse,
                                                    workspace=ws)),
               h2d=[(q, q_h.pin_memory())], d2h=[_pinned_pair(o)],
               launches=2 if splits > 1 else 1, cpu=cpu, traffic_key="fa_decode_kernel")


def row_varlen(rank: int, dev) -> Row:
    import io_aware_exact_16_b200 as fa
    import oracle
    w = workloads.PackedWorkload("varlen causal train B8 H16 d128 lengths U[512, 8192]", 8, 16,
                                 16, 128, True, 1080 + 7919 * rank, len_range=(512, 8192))
    inp = workloads.make_packed_inputs(w)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    cu = inp.cu_seqlens.to(dev)
    lens = [int(inp.cu_seqlens[i + 1] - inp.cu_seqlens[i]) for i in range(w.B)]
    o = torch.empty_like(q)
    lse = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.bwd_workspace_size(w.B, w.H, inp.max_seqlen, w.d), dtype=torch.uint8,
                     device=dev)
    fwd = sum(4.0 * w.H * L * L * w.d / 2.0 for L in lens)
    bf16, _, src = _peaks()

    def step(mark):
        fa.forward_varlen(q, k, v, cu, inp.max_seqlen, causal=True, scale=w.scale, out=o, lse=lse)
        mark()
        fa.backward_varlen(q, k, v, o, do, lse, cu, inp.max_seqlen, causal=True, scale=w.scale,
                           dq=dq, dk=dk, dv=dv, workspace=ws)

    def cpu():
        b = min(range(w.B), key=lambda i: lens[i])  # the shortest sequence, one head
        t0, t1 = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        c0 = time.perf_counter()
        oracle.head_bwd(inp.q[t0:t1, 0], inp.k[t0:t1, 0], inp.v[t0:t1, 0], inp.do[t0:t1, 0],
                        w.scale, True)
        L = t1 - t0
        return {"amount": 3.5 * 4.0 * L * L * w.d / 2.0, "seconds": time.perf_counter() - c0,
                "sample": f"fp64 C oracle fwd+bwd of one head of the shortest sequence (L={L})"}

    return Row(config={"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "causal": True,
                       "total_tokens": int(q.shape[0]), "max_seqlen": inp.max_seqlen,
                       "l2": "Q,K,V,O,dO,dQ,dK,dV about %.0f MB each" % (q.numel() * 2 / 1e6)},
               metric="bf16 packed variable-length attention fwd/bwd TFLOP/s", unit="TFLOP/s",
               dtype="bf16", amount=3.5 * fwd, kernel="fa_bwd_kernel (packed)",
               kernel_amount=2.5 * fwd, bound="tensor", peak=bf16,
               peak_source=f"{src} bf16 sustained", step=step,
               h2d=[(q, inp.q.pin_memory()), (k, inp.k.pin_memory()), (v, inp.v.pin_memory()),
                    (do, inp.do.pin_memory())],
               d2h=[_pinned_pair(t) for t in (o, dq, dk, dv)], launches=4, cpu=cpu)


ROWS = {"fwd-d256": row_fwd_d256, "bwd-d256": row_bwd_d256, "fwd-fp8": row_fwd_fp8, "decode": row_decode,
        "varlen": row_varlen}


def run_row(args, rank: int, world: int, local_rank: int) -> dict | None:
    import io_aware_exact_16_b200 as fa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    row = ROWS[args.row](rank, dev)
    stream = torch.cuda.current_stream(dev)
    no_mark = lambda: None  # noqa: E731
    for _ in range(args.warmup):
        row.step(no_mark)
    torch.cuda.synchronize(dev)
    if fa.check_device_error(dev) != 0:
        raise RuntimeError("device error flag set during warm-up")

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for e in (x for pair in kev for x in pair):
        e.record(stream)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s_ in range(args.steps):
            row.step(lambda: fa.time_next_kernel(kev[s_][0], kev[s_][1]))
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    elapsed_ms = start.elapsed_time(end)
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    if fa.check_device_error(dev) != 0:
        raise RuntimeError("device error flag set in the timed region")

    e2e_steps = max(1, min(args.steps, 10))
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for dst, src in row.h2d:
            dst.copy_(src, non_blocking=True)
        row.step(no_mark)
        for src, dst in row.d2h:
            dst.copy_(src, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    elapsed_ms, kernel_ms, e2e_ms = reduce_max([elapsed_ms, kernel_ms, e2e_ms], world, dev)
    if rank != 0:
        return None

    scale_unit = 1e12 if row.unit == "TFLOP/s" else 1e9
    clock_summary = clocks.summary()
    value = row.amount * args.steps * world / (elapsed_ms * 1e-3) / scale_unit
    achieved = row.kernel_amount / (kernel_ms * 1e-3) / scale_unit
    traffic = dram_traffic(row.traffic_key, row.config["workload"]) if row.traffic_key else None
    line = {
        "metric": row.metric, "value": round(value, 2), "unit": row.unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": row.dtype,
        "data": "synthetic (seeded N(0,1) draws)", "row": args.row,
        "config": dict(row.config, parallelism=f"independent batches x{world}"),
        "roofline": ({"kernel": row.kernel, "bound": row.bound, "achieved": round(achieved, 2),
                      "peak": row.peak, "unit": row.unit, "frac": round(achieved / row.peak, 4),
                      "peak_source": row.peak_source, "kernel_ms": round(kernel_ms, 4),
                      "traffic": traffic} if row.bound != "tensor" else
                     roofline_tensor(row.kernel, achieved, kernel_ms, *load_peaks(),
                                     elapsed_ms * 1e-3, clock_summary, traffic,
                                     scale=row.peak_scale)),
        "e2e": {"value": round(row.amount * e2e_steps * world / (e2e_ms * 1e-3) / scale_unit, 2),
                "unit": row.unit,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t, _ in row.h2d),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t, _ in row.d2h),
                "steps": e2e_steps},
        "gpu_launches": row.launches * args.steps,
        "clocks": clock_summary,
    }
    if not args.no_cpu_baseline:
        import oracle
        oracle.build()
        c = row.cpu()
        line["cpu_baseline"] = {"value": round(c["amount"] / c["seconds"] / scale_unit, 6),
                                "unit": row.unit, "cores": oracle.get_threads(),
                                "kind": "oracle", "sample": f"{c['sample']} ({c['seconds']:.1f} s)"}
    return line


def run_row_reference(args, rank: int, world: int) -> dict | None:
    """The oracle on the row's workload: its bounded sample (Row.cpu) once per step."""
    if rank != 0:
        return None
    import oracle
    oracle.build()
    row = ROWS[args.row](0, torch.device("cuda", 0))
    for _ in range(args.warmup):
        row.cpu()
    amount = seconds = 0.0
    sample = ""
    for _ in range(args.steps):
        c = row.cpu()
        amount += c["amount"]
        seconds += c["seconds"]
        sample = c["sample"]
    scale_unit = 1e12 if row.unit == "TFLOP/s" else 1e9
    value = amount / seconds / scale_unit
    return {
        "impl": "reference", "metric": row.metric, "value": round(value, 6), "unit": row.unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(seconds * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "row": args.row, "config": row.config,
        "cpu_baseline": {"value": round(value, 6), "unit": row.unit,
                         "cores": oracle.get_threads(), "kind": "oracle",
                         "sample": f"{sample}, once per step"},
        "e2e": {"value": round(value, 6), "unit": row.unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def relaunch(n: int, argv: list[str], timeout_s: int) -> int:
    """`--gpus N` without a launcher: start N ranks of this script with torch.distributed.run
    (one process per GPU, rendezvous on 127.0.0.1) and pass rank 0's JSON line through.  Every
    rank's timing is reduced to the maximum over ranks inside the job."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = ["timeout", "-k", "60", str(timeout_s), sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", f"--nproc-per-node={n}", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__)] + argv
    return subprocess.call(cmd)


def run_selftest_ranks(args, rank: int, world: int) -> dict | None:
    """Host-side check of the multi-rank path without a GPU (gloo): each rank reports a
    different fake time; rank 0 returns the line the real run would print, with the maximum."""
    fake_ms = [10.0 + rank, 100.0 - rank]
    elapsed_ms, other = reduce_max(fake_ms, world)
    if rank != 0:
        return None
    return {"metric": METRIC, "selftest": True, "n_gpus": world, "scaling": "weak",
            "ms_max_over_ranks": [elapsed_ms, other]}


def main(argv: list[str] | None = None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD,
                    help="workload of the default training row")
    ap.add_argument("--row", choices=["train"] + sorted(ROWS), default="train",
                    help="train: forward + backward step (default); others: the further "
                         "entry points, each on its own workload")
    ap.add_argument("--sweep", action="store_true",
                    help="one training line per throughput-sweep point (N 512..16384 x "
                         "(H16, d128), (H32, d64) x causal and not), without the end-to-end "
                         "leg and the oracle")
    ap.add_argument("--cpu-heads", type=int, default=12)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--selftest-ranks", action="store_true",
                    help="check the multi-rank launch and max-over-ranks logic on CPU (gloo)")
    ap.add_argument("--launch-timeout", type=int, default=1800,
                    help="seconds before a self-launched multi-rank job is stopped")
    raw = sys.argv[1:] if argv is None else argv
    args = ap.parse_args(raw)
    if args.warmup < 3 and args.impl == "ours" and not args.selftest_ranks:
        ap.error("--warmup must be >= 3")

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return relaunch(args.gpus, raw, args.launch_timeout)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"error: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
        return 2
    distributed = world > 1 and (args.impl == "ours" or args.selftest_ranks)
    if distributed:
        import datetime
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if args.selftest_ranks:
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        else:
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.selftest_ranks:
            lines = [run_selftest_ranks(args, rank, world)]
        elif args.row != "train":
            lines = [run_row_reference(args, rank, world) if args.impl == "reference"
                     else run_row(args, rank, world, local_rank)]
        elif args.impl == "reference":
            lines = [run_reference(args, rank, world)]
        elif args.sweep:
            lines = []
            for name in SWEEP_NAMES:
                pa = argparse.Namespace(**vars(args))
                pa.workload, pa.skip_e2e, pa.no_cpu_baseline = name, True, True
                line = run_ours(pa, rank, world, local_rank)
                if line is not None:
                    line["row"] = "sweep"
                    print(json.dumps(line), flush=True)
        else:
            lines = [run_ours(args, rank, world, local_rank)]
        for line in lines:
            if line is not None:
                print(json.dumps(line), flush=True)
    finally:
        if distributed:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
