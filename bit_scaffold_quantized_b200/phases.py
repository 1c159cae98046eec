"""Per-phase time breakdown of the batch-1 token kernel on the GPU.

    python -m bit_scaffold_quantized_b200.phases [--tokens 64] [--warmup 8] [--head fp16|int8]

Decodes the 48-layer, d_model 2048 benchmark model (batch 1, greedy, CUDA graph per
token) with the phase-timer build of the library (libdfssm_phases.so, built here
with -DDFSSM_PHASE_TIMERS on first use), then prints, per phase, the microseconds
per layer that thread 0 of each CTA spent there (mean and max over CTAs; SM clock
taken from the device's maximum), plus the event-timed token time of the timer
build.  The timers add a few clock reads per phase; the product build has none.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

PHASES = ["gather residual", "wait AB copies", "prep x (whole vector)", "codes + LoRA partials (send)",
          "MMA shared tiles", "wait LoRA partials", "shared rows (send)", "MMA z/x tiles", "z/x epilogue",
          "wait shared rows", "SSM + publish g", "gather g", "wait CD copies", "prep xo (whole vector)",
          "codes + LoRA partials (send)", "MMA out tiles", "wait LoRA partials", "residual rows + publish",
          "LM head: gather + final norm", "LM head: stream rows (thread 0's warp)",
          "LM head: argmax exchange"]
N_LAYER_PHASES = 18      # the per-layer phases; the LM-head phases after them are per token
SLOTS = 32


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--head", choices=["fp16", "int8"], default="fp16", help="LM-head format")
    ap.add_argument("--json", action="store_true")
    args = ap.parse_args()
    os.environ["DFSSM_VARIANT"] = "phases"
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import ctypes as C
    import numpy as np
    import torch
    from bit_scaffold_quantized_b200 import build
    if not os.environ.get("DFSSM_LIBRARY"):
        build.build(variant="phases")
    from bit_scaffold_quantized_b200 import dfssm as F
    from bit_scaffold_quantized_b200 import synth as S
    L = F.lib()
    m, tok0 = S.model_workload("model_48x2048_v50280_b1_greedy512")
    d = m.dims
    dm = F.DeviceModel.from_host(m, head=args.head)
    states = [F.DeviceState.zeros(d) for _ in m.layers]
    call = F.ModelCall(dm, states)
    ws = F.workspace(d, len(m.layers), m.vocab)
    tok = torch.from_numpy(tok0).cuda()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        call(tok, tok, ws, None, stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call(tok, tok, ws, None, stream)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    buf = (C.c_uint64 * (256 * SLOTS))()
    n = L.dfssm_phase_timers(buf, 0, 1)           # reset
    if n < 0:
        raise SystemExit(F.last_error())
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.tokens):
            graph.replay()
        e1.record(stream)
    stream.synchronize()
    us_tok = e0.elapsed_time(e1) * 1e3 / args.tokens
    L.dfssm_phase_timers(buf, 256 * SLOTS, 0)
    a = np.frombuffer(buf, dtype=np.uint64).reshape(256, SLOTS).astype(np.float64)
    ctas = np.nonzero(a[:, SLOTS - 1])[0]
    calls = a[ctas, SLOTS - 1]
    mhz = torch.cuda.get_device_properties(0).clock_rate / 1e3 if hasattr(torch.cuda.get_device_properties(0), "clock_rate") else 1965.0
    cyc = a[ctas, :len(PHASES)] / calls[:, None]             # cycles per token per CTA
    per = cyc.copy()
    per[:, :N_LAYER_PHASES] /= len(m.layers)                  # per layer, except the LM head
    us = per / mhz
    rows = []
    for i, name in enumerate(PHASES):
        rows.append({"phase": name, "us_mean": round(float(us[:, i].mean()), 3), "us_max": round(float(us[:, i].max()), 3)})
    layer_us = float(us[:, :N_LAYER_PHASES].sum(axis=1).mean())
    out = {"tokens": args.tokens, "head": args.head, "ctas": int(len(ctas)), "sm_mhz_assumed": mhz, "us_per_token_event": round(us_tok, 2),
           "us_per_layer_phase_sum": round(layer_us, 3), "phases": rows}
    if args.json:
        print(json.dumps(out))
        return
    print(f"token (event-timed, timer build): {us_tok:.1f} us over {args.tokens} tokens; {len(ctas)} CTAs; "
          f"clock {mhz:.0f} MHz assumed")
    print(f"{'phase':40s} {'us/layer mean':>14s} {'max over CTAs':>14s}")
    for r in rows:
        print(f"{r['phase']:40s} {r['us_mean']:14.3f} {r['us_max']:14.3f}")
    print(f"{'sum of layer phases':40s} {layer_us:14.3f}")
    print("(the LM-head rows are microseconds per token, not per layer)")


if __name__ == "__main__":
    main()
