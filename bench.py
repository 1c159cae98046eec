"""Decode benchmark of the DF-SSM decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the 48-layer Mamba-2-1.3B-shaped DF-SSM model (d_model 2048, d_inner
4096, 64 heads x 64, d_state 128, LoRA rank 32, vocab 50280, fp16 tied LM head),
random-init from a seed, batch 1, greedy decode from a 1-token prompt.  One step =
one decode token for the batch (embedding, 48 layers, final norm, LM head, argmax),
replayed as one CUDA graph with the token fed back on the device.  Each step
streams ~598 MB, far more than the 126 MB L2, so no L2 flush is needed between steps.

Prints one JSON line (rank 0).  Under torchrun each rank decodes an independent
replica on its own GPU (replicas only: no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
from dataclasses import replace
import re
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_scaffold_quantized_b200 import synth as S  # noqa: E402
from bit_scaffold_quantized_b200 import replicas as RP  # noqa: E402
from bit_scaffold_quantized_b200 import roofline as R  # noqa: E402

WORKLOAD = "model_48x2048_v50280_b1_greedy512"
METRIC = "batch-1 decode tokens/s and achieved HBM GB/s (fraction of B200 roofline)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}

THROTTLE_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def profiled_traffic():
    """DRAM bytes per launch of the decode kernel from the committed ncu summary, or
    None with the reason.  Returns None when the kernel source has changed since those
    counters were taken, or when the summary records that the kernel could not be
    captured."""
    path = os.path.join(ROOT, "profiles", "k_decode_persistent_model_48x2048_b1.md")
    src = os.path.join(ROOT, "bit_scaffold_quantized_b200", "csrc", "persistent.cuh")
    try:
        with open(path) as f:
            text = f.read()
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    t = re.search(r"^traffic_bytes_per_launch: (\d+)$", text, re.M)
    h = re.search(r"^kernel_source_sha256: ([0-9a-f]{64})$", text, re.M)
    if not t or not h or h.group(1) != sha:
        return None
    return int(t.group(1))


def traffic_note(traffic):
    if traffic is not None:
        return "dram__bytes_read.sum + dram__bytes_write.sum per launch, profiles/k_decode_persistent_model_48x2048_b1.md"
    return ("not measured: ncu cannot launch the cooperative cluster token kernel (LaunchFailed under the "
            "profiler, even for the one-pass launch list); see profiles/k_decode_persistent_model_48x2048_b1.md")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None
        self.window = None

    def wait_first(self, limit_s: float):
        """Let nvidia-smi start up before the region it has to cover (bounded)."""
        t_end = time.monotonic() + limit_s
        while self.proc is not None and not self.rows and time.monotonic() < t_end:
            time.sleep(0.02)

    def mark(self, t0: float, t1: float):
        """Restrict the summary to samples taken between two monotonic times."""
        self.window = (t0, t1)

    def __enter__(self):
        cmd = ["nvidia-smi", "-i", str(self.gpu),
               "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", "100"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self

        def reader():
            for line in self.proc.stdout:
                self.rows.append((time.monotonic(), line.strip()))
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], [], set()
        rows = self.rows
        if self.window is not None:
            inside = [r for r in rows if self.window[0] <= r[0] <= self.window[1]]
            rows = inside or rows[-1:]
        for _, r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 3:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                bits = int(parts[2], 16)
            except ValueError:
                continue
            for b, name in THROTTLE_BITS.items():
                if bits & b:
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle legs

def oracle_slice(m, tok, n_layers: int, vocab_rows: int):
    """A bounded slice of one decode token through the oracle: embedding, the first
    n_layers layers, final norm and vocab_rows rows of the LM head."""
    from oracle import dfssm_oracle as O
    d = m.dims
    res = m.embed[tok.astype(np.int64)].astype(np.float32)
    for lw in m.layers[:n_layers]:
        st = S.zero_state(d)
        res = O.layer_step(res, lw, O.State(st.conv, st.ssm), d).res
    xf = O.rmsnorm(res, m.normf_w)
    logits = xf @ m.embed[:vocab_rows].astype(np.float64).T
    return int(np.argmax(logits[0]))


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class _OneThread:
    """The oracle runs single-threaded on one host core: BLAS limited to one thread
    (numpy's own loops are single-threaded) and the process pinned to one core for the
    duration.  Reports the threads the BLAS pools actually had inside the region."""

    def __enter__(self):
        from threadpoolctl import threadpool_limits, threadpool_info
        self._lim = threadpool_limits(limits=1)
        self._aff = None
        if hasattr(os, "sched_getaffinity"):
            self._aff = os.sched_getaffinity(0)
            os.sched_setaffinity(0, {min(self._aff)})
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        self.threads = max(n) if n else 1
        return self

    def __exit__(self, *exc):
        if self._aff is not None:
            os.sched_setaffinity(0, self._aff)
        self._lim.restore_original_limits()


def time_oracle(m, tok, n_layers: int, vocab_rows: int, reps: int):
    """(seconds per repetition of the slice, threads used); one thread, one core."""
    with _OneThread() as one:
        oracle_slice(m, tok, 1, 16)      # import + first-touch outside the timing
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle_slice(m, tok, n_layers, vocab_rows)
        return (time.perf_counter() - t0) / reps, one.threads


def slice_fraction(m, n_layers: int, vocab_rows: int) -> float:
    """Fraction of one token's algorithmic bytes that the slice covers."""
    d = m.dims
    full = R.model_token_bytes(d, len(m.layers), m.vocab)
    part = n_layers * (R.layer_weight_bytes(d) + R.layer_state_bytes(d)) + 2 * vocab_rows * d.d_model
    return part / full


# ------------------------------------------------------------------ GPU arm

def run_ours(args, rank, world, local_rank):
    import torch
    from bit_scaffold_quantized_b200 import dfssm as F

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    F.lib()
    m, tok0 = S.model_workload(args.workload)
    if args.state == "fp16":
        m.dims = replace(m.dims, ssm_state_dtype=1)
    d = m.dims
    dm = F.DeviceModel.from_host(m, device=dev, head=args.head)
    states = [F.DeviceState.zeros(d, device=dev) for _ in m.layers]
    call = F.ModelCall(dm, states)
    ws = F.workspace(d, len(m.layers), m.vocab, device=dev)
    tok = torch.from_numpy(tok0).to(dev)          # tok_in and tok_out alias: greedy feedback on device
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    # eager warm-up (also verifies the call succeeds), then capture one decode step
    with torch.cuda.stream(stream):
        call(tok, tok, ws, None, stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call(tok, tok, ws, None, stream)
    launches_per_step = F.launches_per_decode_step(d, len(m.layers), m.vocab)

    with ClockSampler(local_rank) as clk:
        clk.wait_first(3.0)
        for _ in range(args.warmup):
            with torch.cuda.stream(stream):
                graph.replay()
        stream.synchronize()

        RP.barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t_begin = time.monotonic()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        stream.synchronize()
        clk.mark(t_begin, time.monotonic())
    torch.cuda.synchronize()
    RP.barrier(world)
    ms = e0.elapsed_time(e1)

    # end-to-end: host token in (pinned) -> decode step -> host token out, every step
    h_in = torch.from_numpy(tok0.copy()).pin_memory()
    h_out = torch.empty_like(h_in).pin_memory()
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for _ in range(args.steps):
            tok.copy_(h_in, non_blocking=True)
            graph.replay()
            h_out.copy_(tok, non_blocking=True)
            stream.synchronize()
            h_in.copy_(h_out)
        f1.record(stream)
    stream.synchronize()
    ms_e2e = f0.elapsed_time(f1)

    ms, ms_e2e = RP.max_over_ranks([ms, ms_e2e], world, device=dev)
    del graph

    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    tokens = args.steps * d.batch * world
    tok_s = RP.job_tokens_per_s(args.steps, d.batch, world, ms)
    bytes_tok = R.model_token_bytes(d, len(m.layers), m.vocab, head=args.head)
    step_s = ms / 1e3 / args.steps
    achieved = bytes_tok / step_s / 1e9        # GB/s; one step = one token for every batch row
    peak = float(peaks["hbm_gbs"])
    line = {
        "metric": METRIC,
        "value": round(tok_s, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"1-bit scaffold x fp16 act (fp32 acc), int8 LoRA (int32 acc), {args.state} SSM state",
        "data": "synthetic (seeded random-init weights, random 1-token prompt)",
        "config": {"workload": args.workload, "head": args.head, "ssm_state": args.state,
                   "n_layer": len(m.layers), "d_model": d.d_model,
                   "d_inner": d.d_inner, "nheads": d.nheads, "headdim": d.headdim, "d_state": d.d_state,
                   "rank": d.rank, "vocab": m.vocab, "batch": d.batch, "parallelism": f"replicas x{world}",
                   "cuda_graph": True,
                   "l2": f"no flush: each step streams {bytes_tok / 1e6:.1f} MB > 126 MB L2"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": profiled_traffic(),
                     "traffic_source": traffic_note(profiled_traffic()),
                     "kernel": "whole decode step (graph replay)",
                     "algorithmic_bytes_per_step": bytes_tok, "peak_source": peak_kind},
        "roofline_tokens_per_s": round(peak * 1e9 / bytes_tok * d.batch, 1),   # one step = batch tokens
        "e2e": {"value": round(RP.job_tokens_per_s(args.steps, d.batch, world, ms_e2e), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": 4 * d.batch, "d2h_bytes_per_step": 4 * d.batch},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        nl, vr = 1, m.vocab // 48
        reps = 3
        sec, threads = time_oracle(m, tok0, nl, vr, reps)
        frac = slice_fraction(m, nl, vr)
        line["cpu_baseline"] = {"value": round(frac / sec * d.batch, 5), "unit": "tokens/s",
                                "cores": threads, "kind": "oracle", "cpu_model": _cpu_model(),
                                "host_cpus": os.cpu_count(),
                                "sample": f"{reps} x (1 of 48 layers + {vr} of {m.vocab} LM-head rows), "
                                          f"= {frac:.4f} token each by algorithmic bytes; single thread "
                                          f"on one core, extrapolated to a token"}
    return line


def run_sweep(args):
    """The isolated scaffold + int8-LoRA projection sweep: one JSON line per point.

    Each point cycles through enough copies of the packed sign words to exceed 4x L2,
    as a CUDA graph of one call per copy, and times 1000+ calls with CUDA events."""
    import torch
    from bit_scaffold_quantized_b200 import dfssm as F
    dev = torch.device("cuda", 0)
    F.lib()
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    int8_tops = 2.0 * float(peaks["bf16_tflops"])      # int8 dense = 2x the measured bf16 rate (nominal ratio)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)
    for d_in, d_out in S.PROJ_SWEEP_SHAPES:
        for r in S.PROJ_SWEEP_RANKS:
            for b in S.PROJ_SWEEP_BATCHES:
                pw, x_h = S.proj_workload(d_in, d_out, r, b)
                p = F.DeviceProj.from_host(pw, device=dev)
                wbytes = R.proj_weight_bytes(d_out, d_in, r)
                ncopy = max(1, min(128, -(-4 * l2 // wbytes)))
                copies = [p.bits.clone() for _ in range(ncopy)]
                x = torch.from_numpy(x_h).to(dev)
                y = torch.empty((b, d_out), dtype=torch.float32, device=dev)
                ws = F.proj_workspace(d_out, d_in, r, b, device=dev)
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=stream):
                    for c in copies:
                        p.bits = c
                        F.proj_forward(p, r, x, y, ws, stream)
                reps = max(1, -(-1000 // ncopy))
                for _ in range(2):
                    graph.replay()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    for _ in range(reps):
                        graph.replay()
                    e1.record(stream)
                stream.synchronize()
                us = e0.elapsed_time(e1) * 1e3 / (reps * ncopy)
                gbs = R.proj_bytes(d_out, d_in, r, b) / (us * 1e-6) / 1e9
                tops = R.proj_flops(d_out, d_in, r, b) / (us * 1e-6) / 1e12
                print(json.dumps({
                    "metric": "fused scaffold + int8-LoRA projection", "value": round(us, 3), "unit": "us/call",
                    "higher_is_better": False, "config": {"d_in": d_in, "d_out": d_out, "rank": r, "batch": b,
                                                          "weight_copies": ncopy, "calls": reps * ncopy},
                    "hbm": {"achieved_gbs": round(gbs, 1), "peak": hbm, "frac": round(gbs / hbm, 4)},
                    "tensor": {"achieved_tops": round(tops, 2), "peak_int8_tops": int8_tops,
                               "frac": round(tops / int8_tops, 5)},
                    "peak_source": peak_kind}), flush=True)
                del graph, copies


def run_proj_point(args):
    """One projection sweep point, called a few times (a short target for profilers)."""
    import torch
    from bit_scaffold_quantized_b200 import dfssm as F
    d_in, d_out, r, b = args.proj
    F.lib()
    pw, x_h = S.proj_workload(d_in, d_out, r, b)
    p = F.DeviceProj.from_host(pw)
    x = torch.from_numpy(x_h).cuda()
    y = torch.empty((b, d_out), dtype=torch.float32, device="cuda")
    ws = F.proj_workspace(d_out, d_in, r, b)
    for _ in range(3):
        F.proj_forward(p, r, x, y, ws)
    torch.cuda.synchronize()
    print(json.dumps({"proj": [d_in, d_out, r, b], "calls": 3, "ok": True}))


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle as it stands, on this machine's host cores."""
    if rank != 0:
        return None
    m, tok0 = S.model_workload(args.workload)
    nl, vr = 1, m.vocab // 48
    frac = slice_fraction(m, nl, vr)
    with _OneThread() as one:
        for _ in range(args.warmup):
            oracle_slice(m, tok0, nl, vr)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_slice(m, tok0, nl, vr)
        sec = time.perf_counter() - t0
        threads = one.threads
    d = m.dims
    value = args.steps * frac * d.batch / sec
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 5), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded random-init weights, random 1-token prompt)",
        "config": {"workload": args.workload, "batch": d.batch, "n_layer": len(m.layers), "vocab": m.vocab},
        "cpu_baseline": {"value": round(value, 5), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "cpu_model": _cpu_model(), "host_cpus": os.cpu_count(),
                         "sample": f"each step = 1 of 48 layers + {vr} LM-head rows = {frac:.4f} token, "
                                   f"single thread on one core"},
        "e2e": {"value": round(value, 5), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[k for k in S.WORKLOADS if k.startswith("model_")],
                    help="model decode workload (default: the batch-1 greedy decode)")
    ap.add_argument("--head", choices=["fp16", "int8"], default="fp16",
                    help="tied embedding / LM head precision (int8: per-row codes + fp32 scales)")
    ap.add_argument("--state", choices=["fp32", "fp16"], default="fp32",
                    help="SSM state storage (fp16: multi-launch path at every batch size)")
    ap.add_argument("--sweep", action="store_true", help="time the isolated projection sweep instead")
    ap.add_argument("--proj", type=int, nargs=4, metavar=("D_IN", "D_OUT", "RANK", "BATCH"),
                    help="call one projection sweep point three times (a target for profilers)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.sweep:
        run_sweep(args)
        return
    if args.proj:
        run_proj_point(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1 and args.impl == "ours":
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
