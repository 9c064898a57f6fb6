"""Throughput of exact attention (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long_ctx] [--seq N] [--no-cpu-baseline] [--e2e-steps E]
                    [--deterministic] [--varlen] [--fp8] [--e2e-serial] [--e2e-chunks C]

One step is one pass of the whole hot path over one batch of synthetic input:
the forward kernel, then the three backward kernels (D preprocess, main,
dQ convert), all through the library's C ABI.  The default workload is the
long-context causal bf16 attention layer B=1, H=16, N=16384, d=128 (Q, K, V
scaled by 0.5), the configuration the headline tensor-roofline target is
quoted on.  Flops are algorithmic: forward 4*B*H*N*N*d, halved for causal;
backward 2.5x that.

Rank 0 prints ONE JSON line.  For N > 1 (torchrun, one process per GPU) every
rank runs an independent replica of the workload: the path has no exchange
step, so there is no collective on the data path; the timing is the max over
ranks (an all-reduce of the elapsed time only).

--varlen times a packed variable-length batch instead (attn_fwd_varlen and
attn_bwd_varlen on a seeded length mix; see workloads.VARLEN_MIX).

--fp8 times the FP8 forward instead (attn_fwd_fp8 on E4M3 Q, K, V with
per-tensor descales; see workloads.FWD_FP8), against an 8-bit peak of twice
the measured bf16 peak (the nominal dense ratio).

The e2e leg runs the step end to end through the library's public call for
host-resident tensors, attn_host_step: every step it copies the inputs from
pinned host memory to the device, runs the forward and backward kernels and
copies every result back, with the copies of one chunk of (batch, head)
slices overlapping the kernels of another.  --e2e-serial instead copies the
inputs, calls attn_fwd / attn_bwd and copies the results back in order on
one stream.  Forward-only workloads always take the serial form.

--impl reference times the fp64 CPU oracle (the correctness reference) on a
bounded sample of the same workload on the host cores, and prints the same
line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s on 1 B200 and fraction of dense BF16/FP16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of a kernel,
# measured by ncu on this bench's command, keyed by (workload name, N) and
# kernel.  Only valid for the kernel version it was taken on: remove an entry
# when its kernel changes.  long_ctx: the full-set capture of the first timed
# step of `bench.py --steps 2 --warmup 1 --e2e-steps 0 --no-cpu-baseline`.
KERNEL_TRAFFIC: dict = {
    ("long_ctx", 16384): {"bwd_main_kernel": 405_487_872 + 224_790_016, "fwd_kernel": 236_569_600 + 52_866_816},
}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="long_ctx")
    p.add_argument("--seq", type=int, default=None, help="override the sequence length (profiling runs)")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--varlen", action="store_true", help="time a packed variable-length batch")
    p.add_argument("--fp8", action="store_true", help="time the FP8 (E4M3) forward")
    p.add_argument("--e2e-serial", action="store_true",
                   help="run the e2e leg as copies, attn_fwd, attn_bwd, copies in order on one stream instead of "
                        "through attn_host_step")
    p.add_argument("--e2e-chunks", type=int, default=8, help="chunks of (batch, head) slices of attn_host_step")
    p.add_argument("--deterministic", action="store_true",
                   help="time the bit-reproducible backward (attn_bwd_deterministic) instead of attn_bwd")
    return p.parse_args(argv)


# ---------------------------------------------------------------- helpers

def add_spread(kernels: dict, evs, spans: dict) -> None:
    """Adds the median and the minimum of each kernel's per-step event times
    (events a -> b of every step) beside its mean."""
    for name, (a, b) in spans.items():
        if name not in kernels or not evs:
            continue
        t = [e[a].elapsed_time(e[b]) for e in evs]
        kernels[name]["ms_median"] = statistics.median(t)
        kernels[name]["ms_min"] = min(t)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# The sustained peak in MEASURED_PEAKS.json is a cuBLAS loop run back to back
# for this long under the power cap; a timed region shorter than that is a
# burst and is held to the burst peak.
SUSTAINED_WINDOW_S = 4.0


def choose_peak(peaks: dict, peak_src: str, timed_s: float, clocks: dict, scale: float = 1.0):
    """The bf16 tensor peak (times `scale`, e.g. 2 for the 8-bit path) that
    a kernel timed over `timed_s` seconds is held to: the burst figure when
    the timed region is shorter than the sustained measurement, else the
    sustained one.  Also returns the burst peak scaled by the median sampled
    SM clock over its maximum, the roofline at the clock the run actually
    saw."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    if timed_s < SUSTAINED_WINDOW_S:
        peak, which = burst, "bf16_tflops (burst: the timed region, %.2f s, is shorter than the %g s sustained " \
                             "measurement)" % (timed_s, SUSTAINED_WINDOW_S)
    else:
        peak, which = sustained, "bf16_tflops_sustained (the timed region, %.2f s, is a sustained load)" % timed_s
    at_clock = None
    mhz, max_mhz = clocks.get("sm_mhz"), clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz")
    if mhz and max_mhz:
        at_clock = scale * burst * min(1.0, float(mhz) / float(max_mhz))
    src = f"{peak_src} {which}" + (f" x {scale:g}" if scale != 1.0 else "")
    return scale * peak, src, at_clock


def roofline_entry(kernel: str, achieved: float, peak: float, src: str, at_clock, traffic):
    r = {"kernel": kernel, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
         "frac": achieved / peak, "traffic": traffic, "peak_source": src}
    if at_clock:
        r["peak_at_sampled_clock"] = at_clock
        r["frac_at_sampled_clock"] = achieved / at_clock
    return r


def get_workload(name, seq):
    import dataclasses
    from exact_attention_150_b200 import workloads
    w = workloads.by_name(name)
    if seq is not None:
        w = dataclasses.replace(w, N=seq, name=f"{w.name}_N{seq}")
    return w


def dist_info():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank processes `steps` steps of its replica."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def call_overhead(call, stream, c_call=None, n_host=200, n_graph=50, replays=10) -> dict:
    """Where the time of a short call goes: the host's cost to enqueue one
    call through the Python binding (wall clock over n_host calls, the device
    idle or ahead) and through the bare C ABI with integer pointers
    (c_call: validation, tensor-map encoding and the launch), and the device
    time of one call with no host gaps (a CUDA graph of n_graph calls,
    replayed)."""
    import torch
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(n_host):
        call()
    t1 = time.perf_counter()
    torch.cuda.synchronize()
    c_us = None
    if c_call is not None:
        c0 = time.perf_counter()
        for _ in range(n_host):
            c_call()
        c_us = 1e6 * (time.perf_counter() - c0) / n_host
        torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for _ in range(n_graph):
                call()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    out = {"host_us_per_call": 1e6 * (t1 - t0) / n_host,
           "graph_us_per_call": 1e3 * a.elapsed_time(b) / (replays * n_graph)}
    if c_us is not None:
        out["c_abi_us_per_call"] = c_us
    return out


def sample_flops(w, rows) -> float:
    """Algorithmic fwd+bwd flops of query rows `rows` (absolute indices) of one head."""
    keys = sum((r + 1) if w.causal else w.N for r in rows)
    return 4.0 * w.d * keys * 3.5  # forward (4 d per visible key) plus backward at 2.5x


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        else:
            self.lines = []

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle

def oracle_sample_run(w, q, k, v, do, rows_count: int):
    """One fp64 oracle forward + backward on the last `rows_count` query rows
    of head (0, 0) against all keys.  Returns (seconds, flops, description,
    (r0, O, LSE, dQ)): the oracle's outputs for those rows, which depend on
    no other query row."""
    import oracle
    import torch
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    n = w.N
    r0 = n - rows_count
    qs, dos = f64(q[0, 0, r0:]), f64(do[0, 0, r0:])
    ks, vs = f64(k[0, 0]), f64(v[0, 0])
    t0 = time.perf_counter()
    o, lse, _ = oracle.forward(qs, ks, vs, w.scale, w.causal, q_offset=r0)
    dq, _, _ = oracle.backward(qs, ks, vs, dos, w.scale, w.causal, q_offset=r0)
    dt = time.perf_counter() - t0
    desc = (f"fp64 oracle forward+backward of query rows [{r0},{n}) of head (0,0) against all {n} keys "
            f"({rows_count} of {w.B * w.H * n} rows of the workload)")
    return dt, sample_flops(w, range(r0, n)), desc, (r0, o, lse, dq)


# Parity bars: max-abs O (by dtype), max-abs LSE, relative Frobenius dQ.
PARITY_TOL = {"o": {"bf16": 1e-2, "fp16": 2e-3}, "lse": 1e-3, "dq": 2e-2}


def sample_parity(w, ref, o, lse, dq):
    """Errors of the timed run's outputs (device tensors [B,H,N,...]) against
    the oracle's outputs `ref` from oracle_sample_run; dq None when the
    workload has no backward."""
    import numpy as np
    import torch
    r0, o_ref, lse_ref, dq_ref = ref
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    got_o, got_l = f64(o[0, 0, r0:]), f64(lse[0, 0, r0:])
    fin = np.isfinite(lse_ref)
    out = {"rows": f"query rows [{r0},{r0 + len(lse_ref)}) of head (0,0)",
           "o_max_abs_err": float(np.max(np.abs(got_o - o_ref), initial=0.0)),
           "lse_max_abs_err": float(np.max(np.abs(got_l[fin] - lse_ref[fin]), initial=0.0)),
           "tol": {"o": PARITY_TOL["o"][w.dtype], "lse": PARITY_TOL["lse"]}}
    ok = out["o_max_abs_err"] <= out["tol"]["o"] and out["lse_max_abs_err"] <= out["tol"]["lse"]
    if dq is not None:
        den = float(np.linalg.norm(dq_ref))
        out["dq_rel_fro_err"] = float(np.linalg.norm(f64(dq[0, 0, r0:]) - dq_ref)) / (den if den > 0 else 1.0)
        out["tol"]["dq"] = PARITY_TOL["dq"]
        ok = ok and out["dq_rel_fro_err"] <= PARITY_TOL["dq"]
    out["within_tol"] = bool(ok)
    for key in ("o_max_abs_err", "lse_max_abs_err", "dq_rel_fro_err"):  # keep the line strict JSON
        if key in out and not math.isfinite(out[key]):
            out[key] = "non-finite"
            out["within_tol"] = False
    return out


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = [x for x in threadpool_info() if x.get("user_api") == "blas"]
        if info:
            return int(max(x.get("num_threads", 1) for x in info))
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------- arms

L2_BYTES = 126 * 2**20
FLUSH_BYTES = 256 * 2**20


def step_input_bytes(w):
    """Bytes of the 16-bit inputs one step reads: Q, K, V (and dO)."""
    return (4 if w.backward else 3) * w.B * w.H * w.N * w.d * 2


def needs_flush(w):
    return step_input_bytes(w) <= L2_BYTES


def config_of(w, world):
    mb = w.B * w.H * w.N * w.d * 2 / 2**20
    if needs_flush(w):
        l2 = ("flush: a %d MB buffer is written before every timed step, outside the step's events; the step "
              "time is the sum of the steps' own spans (inputs of %.2f MB each fit the 126 MB L2)"
              % (FLUSH_BYTES // 2**20, mb))
    else:
        l2 = "no flush: inputs larger than the 126 MB L2 (Q, K, V%s of %d MB each)" % (
            ", dO" if w.backward else "", round(mb))
    return {"workload": w.label(), "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "passes": "fwd+bwd" if w.backward else "fwd", "input_scale": w.input_scale, "l2": l2,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def run_reference(args):
    rank, world, _ = dist_info()
    if rank != 0:
        return 0
    from exact_attention_150_b200 import workloads
    w = get_workload(args.workload, args.seq)
    q, k, v, do = workloads.make_inputs(w, with_grad=True)
    rows = 512
    times, flops = [], 0.0
    desc = ""
    for i in range(args.warmup + args.steps):
        dt, fl, desc, _ = oracle_sample_run(w, q, k, v, do, rows)
        if i >= args.warmup:
            times.append(dt)
            flops = fl
    total = sum(times)
    value = flops * len(times) / total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": "each step: " + desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    rank, world, local_rank = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(device)

    from exact_attention_150_b200 import native, workloads
    native.load()
    w = get_workload(args.workload, args.seq)
    q_h, k_h, v_h, do_h = workloads.make_inputs(w, with_grad=True)
    q, k, v, do = (t.to(device) for t in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(native.attn_bwd_workspace_bytes(w.B, w.H, w.N, w.N, w.d), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def fwd():
        native.forward(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)

    def bwd(phase):
        native.backward(q, k, v, o, lse, do, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv, workspace=ws,
                        phase=phase, deterministic=args.deterministic and phase == native.ATTN_BWD_ALL)

    # The reproducible backward, and every d = 256 backward, is one call of
    # three kernels (preprocess, dK/dV, dQ) timed as a whole.
    one_call = args.deterministic or w.d == 256

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fwd()
        if not w.backward:
            if ev is not None:
                ev[1].record(stream)
            return
        if ev is not None:
            ev[1].record(stream)
        if one_call:
            # One call: preprocess, dK/dV and dQ kernels.
            bwd(native.ATTN_BWD_ALL)
            if ev is not None:
                for e in ev[2:]:
                    e.record(stream)
            return
        bwd(native.ATTN_BWD_PREPROCESS)
        if ev is not None:
            ev[2].record(stream)
        bwd(native.ATTN_BWD_MAIN)
        if ev is not None:
            ev[3].record(stream)
        bwd(native.ATTN_BWD_CONVERT)
        if ev is not None:
            ev[4].record(stream)

    launches_per_step = 4 if w.backward else 1
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(device)
    native.device_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # Inputs that fit L2 would stay there from one step to the next: write a
    # buffer larger than L2 before every step and time the steps' own spans.
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device) if needs_flush(w) else None
    last_ev = 4 if w.backward else 1
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index) as clocks:
        start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            step(evs[i])
        end.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    native.device_status()
    if flush is not None:
        elapsed = sum(e[0].elapsed_time(e[last_ev]) for e in evs)
    else:
        elapsed = start.elapsed_time(end)
    max_ms = max_over_ranks(elapsed, world, device)

    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    step_flops = w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)
    value = aggregate(step_flops, args.steps, world, max_ms)
    peaks, peak_src = load_peaks()
    clock_summary = clocks.summary()
    peak, peak_note, peak_clk = choose_peak(peaks, peak_src, max_ms * 1e-3, clock_summary)
    # Forward algorithmic bytes: read Q, K, V, write O (16-bit) and LSE (fp32).
    fwd_bytes = w.B * w.H * (2 * (2 * w.N + 2 * w.N) * w.d + 4 * w.N)
    kernels = {"fwd_kernel": {"ms": fwd_ms, "tflops": w.fwd_flops() / fwd_ms / 1e9, "gbs": fwd_bytes / fwd_ms / 1e6}}
    one_name = ("bwd_deterministic (preprocess, dK/dV and dQ kernels)" if w.d != 256
                else "bwd, d = 256 (preprocess, 64-key dK/dV and dQ kernels)")
    if w.backward and one_call:
        det_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        kernels[one_name] = {"ms": det_ms, "tflops": w.bwd_flops() / det_ms / 1e9}
        dom_name, dom_ms, dom_flops = one_name.split(" (")[0], det_ms, w.bwd_flops()
    elif w.backward:
        pre_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        main_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
        post_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in evs)
        rows = w.B * w.H * w.N
        kernels["bwd_pre_kernel"] = {"ms": pre_ms, "gbs": rows * (2 * w.d * 2 + 4 + 8 + 4 * w.d) / pre_ms / 1e6}
        kernels["bwd_main_kernel"] = {"ms": main_ms, "tflops": w.bwd_flops() / main_ms / 1e9}
        kernels["bwd_post_kernel"] = {"ms": post_ms, "gbs": rows * w.d * (4 + 2) / post_ms / 1e6}
        dom_name, dom_ms, dom_flops = "bwd_main_kernel", main_ms, w.bwd_flops()
    else:
        dom_name, dom_ms, dom_flops = "fwd_kernel", fwd_ms, w.fwd_flops()
    spans = {"fwd_kernel": (0, 1), one_name: (1, 2),
             "bwd_pre_kernel": (1, 2), "bwd_main_kernel": (2, 3), "bwd_post_kernel": (3, 4)}
    add_spread(kernels, evs, spans)
    for name, kinfo in kernels.items():
        if "tflops" in kinfo:
            kinfo["frac"] = kinfo["tflops"] / peak
    achieved = dom_flops / dom_ms / 1e9
    traffic = None if one_call else KERNEL_TRAFFIC.get((w.name, w.N), {}).get(dom_name)
    if fwd_ms < 0.1:
        ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr())
        code = native.ATTN_BF16 if w.dtype == "bf16" else native.ATTN_FP16
        ccode, sptr = native.causal_code(w.causal), stream.cuda_stream

        def fwd_c():
            native.attn_fwd(*ptrs, w.B, w.H, w.N, w.N, w.d, w.scale, ccode, code, sptr)

        kernels["fwd_kernel"].update(call_overhead(fwd, stream, c_call=fwd_c))

    # End to end through the public API: pinned host inputs -> device, the
    # forward and backward calls, results -> pinned host, every step.
    e2e = None
    if args.e2e_steps > 0:
        pin = lambda t: t.pin_memory()
        hq, hk, hv, hdo = (pin(t) for t in (q_h, k_h, v_h, do_h))
        outs_h = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse, dq, dk, dv)]
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
        d2h = sum(t.numel() * t.element_size() for t in outs_h)

        def e2e_step():
            for dst, src in ((q, hq), (k, hk), (v, hv), (do, hdo)):
                dst.copy_(src, non_blocking=True)
            fwd()
            if w.backward:
                bwd(native.ATTN_BWD_ALL)  # deterministic when --deterministic
            for dst, src in zip(outs_h, (o, lse, dq, dk, dv)):
                dst.copy_(src, non_blocking=True)

        pipelined = w.backward and not args.e2e_serial
        if pipelined:
            # The same step through attn_host_step: the library copies every
            # chunk in, runs its kernels and copies its results out, with the
            # copies of one chunk overlapping the kernels of another.
            dev_buf = torch.empty(native.attn_host_step_device_bytes(w.B, w.H, w.N, w.N, w.d, args.e2e_chunks),
                                  dtype=torch.uint8, device=device)

            def e2e_step():  # noqa: F811
                native.host_step(hq, hk, hv, hdo, causal=w.causal, scale=w.scale, chunks=args.e2e_chunks,
                                 deterministic=args.deterministic, outs=outs_h, device_buffer=dev_buf,
                                 device=device, stream=stream.cuda_stream)

        e2e_step()
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e2.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        native.device_status()
        e2e_ms = max_over_ranks(s2.elapsed_time(e2), world, device)
        e2e = {"value": aggregate(step_flops, args.e2e_steps, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "path": (f"attn_host_step, {args.e2e_chunks} chunks" if pipelined
                        else "copies, attn_fwd%s, copies on one stream" % (", attn_bwd" if w.backward else ""))}

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, fl, desc, ref = oracle_sample_run(w, q_h, k_h, v_h, do_h, min(4096, w.N))
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": desc}
        # The same oracle rows against this run's outputs.
        parity = sample_parity(w, ref, o, lse, dq if w.backward else None)

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp16",
        "data": "synthetic: seeded i.i.d. N(0,1) Q, K, V, dO (x%g)" % w.input_scale,
        "config": {**config_of(w, world), **({"backward": "deterministic"} if args.deterministic else {})},
        "fwd_tflops": w.fwd_flops() / fwd_ms / 1e9,
        "bwd_tflops": (w.bwd_flops() / (max_ms / args.steps - fwd_ms) / 1e9) if w.backward else None,
        "kernels": kernels,
        "roofline": roofline_entry(dom_name, achieved, peak, peak_note, peak_clk, traffic),
        "clocks": clock_summary,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "cpu_baseline": cpu,
        "parity": parity,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_varlen(args):
    """The packed variable-length batch: forward then backward per step."""
    import torch
    rank, world, local_rank = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(device)
    from exact_attention_150_b200 import native, workloads
    native.load()
    m = workloads.VARLEN_MIX
    lens = workloads.varlen_lengths(m["seed"], m["total"], m["lo"], m["hi"])
    H, d = m["H"], m["d"]
    dtype = torch.bfloat16 if m["dtype"] == "bf16" else torch.float16
    q, k, v, do, cu = (t.to(device) for t in workloads.make_varlen_inputs(lens, H, d, dtype, m["seed"],
                                                                           m["input_scale"]))
    mx = max(lens)
    scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty(H, q.shape[1], dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(native.attn_bwd_varlen_workspace_bytes(len(lens), H, q.shape[1], mx, d), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)
    fwd_flops = sum(4.0 * H * n * n * d / (2 if m["causal"] else 1) for n in lens)
    bwd_flops = 2.5 * fwd_flops

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        native.forward_varlen(q, k, v, cu, cu, mx, mx, causal=m["causal"], scale=scale, out=o, lse=lse)
        if ev is not None:
            ev[1].record(stream)
        native.backward_varlen(q, k, v, o, lse, do, cu, cu, mx, mx, causal=m["causal"], scale=scale, dq=dq, dk=dk,
                               dv=dv, workspace=ws, deterministic=args.deterministic)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(device)
    native.device_status()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index) as clocks:
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        end.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    native.device_status()
    max_ms = max_over_ranks(start.elapsed_time(end), world, device)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    peaks, peak_src = load_peaks()
    clock_summary = clocks.summary()
    peak, peak_note, peak_clk = choose_peak(peaks, peak_src, max_ms * 1e-3, clock_summary)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    bwd_tf = bwd_flops / bwd_ms / 1e9
    line = {
        "metric": METRIC, "value": aggregate(fwd_flops + bwd_flops, args.steps, world, max_ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": m["dtype"],
        "data": "synthetic: seeded i.i.d. N(0,1) packed Q, K, V, dO (x%g)" % m["input_scale"],
        "config": {"workload": f"{m['name']}: packed causal {m['dtype']} H{H} d{d}, {len(lens)} sequences, "
                               f"{sum(lens)} tokens, lengths {min(lens)}..{max(lens)}",
                   "lengths": lens, "backward": "deterministic" if args.deterministic else "atomic dQ",
                   "l2": "no flush: packed Q, K, V, dO of %d MB each" % (H * sum(lens) * d * 2 // 2**20),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "fwd_tflops": fwd_flops / fwd_ms / 1e9, "bwd_tflops": bwd_tf,
        "kernels": {"fwd_kernel (varlen)": {"ms": fwd_ms, "tflops": fwd_flops / fwd_ms / 1e9},
                    "bwd (varlen, all kernels)": {"ms": bwd_ms, "tflops": bwd_tf}},
        "roofline": roofline_entry("bwd (varlen, all kernels)", bwd_tf, peak, peak_note, peak_clk, None),
        "clocks": clock_summary, "e2e": None, "gpu_launches": 4 * args.steps,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_fp8(args):
    """The FP8 (E4M3) forward on workloads.FWD_FP8, one forward per step."""
    import torch
    rank, world, local_rank = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(device)
    from exact_attention_150_b200 import native, workloads
    native.load()
    w = workloads.FWD_FP8
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    q8, k8, v8, dq, dk, dv = workloads.draw_fp8(B, H, N, N, d, w["seed"], device=device)
    scale = 1.0 / math.sqrt(d)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    flops = 4.0 * B * H * N * N * d / (2 if w["causal"] else 1)
    # Algorithmic bytes: read Q, K, V (1 byte each), write O (bf16) and LSE.
    nbytes = B * H * N * (3 * d + 2 * d + 4)

    def step():
        native.forward_fp8(q8, k8, v8, dq, dk, dv, causal=w["causal"], scale=scale, out=o, lse=lse)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(device)
    native.device_status()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index) as clocks:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    native.device_status()
    max_ms = max_over_ranks(start.elapsed_time(end), world, device)
    peaks, peak_src = load_peaks()
    clock_summary = clocks.summary()
    # The 8-bit peak: the measured bf16 peak times the nominal 8-bit : 16-bit
    # ratio of 2 (4.5 / 2.25 PFLOP/s dense).
    peak8, peak_note, peak_clk = choose_peak(peaks, peak_src, max_ms * 1e-3, clock_summary, scale=2.0)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    fwd_ms = max_ms / args.steps
    tf = flops / fwd_ms / 1e9
    line = {
        "metric": METRIC, "value": aggregate(flops, args.steps, world, max_ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": fwd_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic: seeded i.i.d. N(0,1) Q, K, V quantised to E4M3 with per-tensor descales (max|x|/448)",
        "config": {"workload": f"{w['name']}: fwd causal e4m3 B{B} H{H} N{N} d{d}, bf16 O",
                   "l2": "no flush: E4M3 Q, K, V of %d MB each" % (B * H * N * d // 2**20),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "fwd_tflops": tf,
        "kernels": {"fwd_kernel (e4m3)": {"ms": fwd_ms, "tflops": tf, "gbs": nbytes / fwd_ms / 1e6,
                                          "frac": tf / peak8}},
        "roofline": roofline_entry("fwd_kernel (e4m3)", tf, peak8, peak_note + " (nominal e4m3 : bf16 ratio)",
                                   peak_clk, None),
        "clocks": clock_summary, "e2e": None, "gpu_launches": args.steps,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.varlen:
        return run_varlen(args)
    if args.fp8:
        return run_fp8(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
