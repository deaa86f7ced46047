"""Per-unit timeline of the engine (profiling build).

Compiles the engine with the timeline hooks of marks.cuh into libfmoe_trace.so beside this
file, runs 64 tokens of a single-layer benchmark workload's launch (default full_q4, with 16
round-robin copies of router / shared expert as bench.py runs it) and prints, for CTAs 0 and
77, the median over units 8..62 of each event's time after the unit's previous-unit-done
event, in microseconds, with its range. The marks themselves cost a few per cent of a unit.

With --all-ctas (libfmoe_trace_all.so, every CTA recorded) it prints instead, per CTA, how
far its unit start lags the median CTA's, the median durations of its phases, and when the
unit's last router logits were stored relative to the median CTA's start of the top-K.

    python -m bit_dequant_expert_gemv_b200.timeline.timeline [workload] [--all-ctas]
"""
from __future__ import annotations

import ctypes as C
import os
import statistics
import subprocess
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
SO = os.path.join(HERE, "libfmoe_trace.so")
SO_ALL = os.path.join(HERE, "libfmoe_trace_all.so")
UNITS, EVENTS, ALL_CTAS = 64, 88, 148   # as in marks.cuh
TOKENS = 64

# event ids of engine.cu's MarkEv, as printed
NAMES = {0: "C unit start", 1: "C prev unit done", 2: "C x in smem", 3: "K top-K start",
         4: "K top-K done", 5: "C xfree", 6: "C shared signal", 7: "C h_s in smem",
         24: "K x ready", 25: "K router done", 26: "K x digits", 27: "K shared g/u done",
         28: "K h_s ready", 29: "K shared down done", 62: "K out written",
         63: "B routing seen", 64: "B last issue", 65: "A first issue", 66: "A last issue",
         67: "R dot done (w0)", 68: "R reduce done (w0)", 69: "R chunk_last (w0)",
         70: "R logits stored (last warp)", 71: "R dot done (w7)", 72: "R reduce done (w7)",
         73: "R chunk_last (w7)", 74: "G0 dot done (w0)", 75: "G0 reduce done (w0)",
         76: "G0 chunk_last (w0)", 77: "G0 h stored (last warp)", 78: "G0 dot done (w7)",
         79: "G0 reduce done (w7)", 80: "G0 chunk_last (w7)", 81: "J1 top (w0)",
         82: "J1 first chunk landed (w0)", 83: "B issued chunk 2", 84: "B issued chunk 3",
         85: "G0 epilogue end"}
for k in range(8):
    NAMES[8 + k] = f"C S2_{k} signal"
    NAMES[16 + k] = f"C h_{k} in smem"
    NAMES[30 + k] = f"K P2_{k} first data"
    NAMES[38 + k] = f"K P2_{k} done"
    NAMES[46 + k] = f"K h_{k} ready"
    NAMES[54 + k] = f"K D_{k} done"


def build_traced(_build, all_ctas: bool = False) -> str:
    """The engine with the marks force-included; the other sources as in the library."""
    so = SO_ALL if all_ctas else SO
    srcs = [os.path.join(_build.CSRC, f) for f in _build.SOURCES + _build.HEADERS]
    srcs.append(os.path.join(HERE, "marks.cuh"))
    if os.path.exists(so) and os.path.getmtime(so) >= max(os.path.getmtime(f) for f in srcs):
        return so
    objs = []
    for src in _build.SOURCES:
        o = os.path.join(HERE, src + (".all" if all_ctas else "") + ".o")
        cmd = ["nvcc", "-O3", "-std=c++17", *_build.ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
               "-I", _build.INCLUDE, "-I", _build.CSRC]
        if all_ctas:
            cmd.append("-DFMOE_TRACE_ALL_CTAS")
        if src == "engine.cu":
            cmd += ["-include", os.path.join(HERE, "marks.cuh")]
        subprocess.run(cmd + ["-c", os.path.join(_build.CSRC, src), "-o", o], check=True)
        objs.append(o)
    subprocess.run(["nvcc", *_build.ARCH, "-shared", *objs, "-o", so, "-lcudart"], check=True)
    return so


# phases of a unit for the per-CTA view: (name, from event, to event; None = next unit's x)
PHASES = [("router", 24, 25), ("x digits", 25, 26), ("shared g/u", 26, 27), ("top-K", 3, 4),
          ("routed g/u 0", 30, 38), ("routed g/u 3", 33, 41), ("shared down", 28, 29),
          ("down 3", 56, 57), ("outputs", 57, 62), ("unit period", 24, None)]


def report_all_ctas(buf, nctas: int) -> None:
    """Per-CTA phase shifts and durations (medians over units 8..62), in microseconds."""
    us = lambda a, b: (int(a) - int(b)) / 1000.0  # noqa: E731
    units = range(8, 62)
    lag = {c: [] for c in range(nctas)}
    for u in units:
        starts = [int(buf[c, u, 24]) for c in range(nctas) if buf[c, u, 24]]
        med = statistics.median(starts)
        for c in range(nctas):
            if buf[c, u, 24]:
                lag[c].append((int(buf[c, u, 24]) - med) / 1000.0)
    mean_lag = {c: statistics.mean(v) for c, v in lag.items() if v}
    order = sorted(mean_lag, key=lambda c: -mean_lag[c])
    print("unit start after the median CTA's (mean over units 8..61, us):")
    print("  latest:  " + "  ".join(f"CTA {c} {mean_lag[c]:+.2f}" for c in order[:6]))
    print("  earliest: " + "  ".join(f"CTA {c} {mean_lag[c]:+.2f}" for c in order[-3:]))
    print("phase durations (median over units, us): min / median / max over CTAs")
    for name, a, b in PHASES:
        per = []
        for c in range(nctas):
            v = [us(buf[c, u + 1, 24] if b is None else buf[c, u, b], buf[c, u, a]) for u in units
                 if buf[c, u, a] and (buf[c, u + 1, 24] if b is None else buf[c, u, b])]
            if v:
                per.append(statistics.median(v))
        if per:
            print(f"  {name:14s} {min(per):6.2f} {statistics.median(per):6.2f} {max(per):6.2f}")
    gaps = []
    for u in units:
        last_logit = max(int(buf[c, u, 70]) for c in range(nctas))
        topk_starts = [int(buf[c, u, 3]) for c in range(nctas) if buf[c, u, 3]]
        if last_logit and topk_starts:
            gaps.append((last_logit - statistics.median(topk_starts)) / 1000.0)
    if gaps:
        print(f"last logits stored, after the median CTA's top-K start: median {statistics.median(gaps):+.2f} us")


def main(wl_name: str = "full_q4", all_ctas: bool = False) -> None:
    sys.path.insert(0, ROOT)
    import torch
    import synth
    import bit_dequant_expert_gemv_b200 as fmoe
    from bit_dequant_expert_gemv_b200 import _build
    from bit_dequant_expert_gemv_b200.workload import build_layer, token_inputs_dev

    fmoe.LIB = build_traced(_build, all_ctas)
    lib = fmoe.lib()
    lib.fmoe_trace_read.argtypes = [C.c_void_p, C.c_size_t]
    wl = synth.WORKLOADS[wl_name]
    assert wl.layers == 1, "single-layer workloads only"
    dl = build_layer(wl, 0)
    descs, keep = [dl.desc], []
    for _ in range(1, 16):  # the bench's round-robin copies of the data-independent tensors
        router = dl.router.clone()
        gate = None if dl.gate is None else dl.gate.clone()
        shared = None if dl.shared is None else dl.shared.clone()
        keep.append((router, gate, shared))
        descs.append(fmoe.LayerDesc(wl.H, wl.I, wl.E, wl.K, wl.bits, dl.experts, dl.stride,
                                    shared, router, gate))
    x = token_inputs_dev(wl, 0, TOKENS)
    res = token_inputs_dev(wl, 0, TOKENS, kind=synth.KIND_RES)
    bias_np = synth.logit_bias(wl, tokens=TOKENS)
    bias = None if bias_np is None else torch.from_numpy(np.ascontiguousarray(bias_np[:, 0])).cuda()
    out = torch.empty_like(x)
    for _ in range(3):
        fmoe.moe_layer_seq(descs, x, res, bias, out=out)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    fmoe.moe_layer_seq(descs, x, res, bias, out=out)
    b.record()
    torch.cuda.synchronize()
    print(f"{wl_name}: {a.elapsed_time(b) * 1000 / TOKENS:.2f} us per unit (profiling build)")
    assert fmoe.sync_status() == 0
    nctas = ALL_CTAS if all_ctas else 2
    buf = np.zeros((nctas, UNITS, EVENTS), dtype=np.uint64)
    assert lib.fmoe_trace_read(buf.ctypes.data, buf.nbytes) == 0
    if all_ctas:
        report_all_ctas(buf, min(nctas, int(torch.cuda.get_device_properties(0).multi_processor_count)))
        return
    for cta in range(2):
        print(f"--- CTA {0 if cta == 0 else 77}: median over units 8..62 of "
              f"(event - 'C prev unit done'), us [min max]")
        rows = []
        for ev in range(EVENTS):
            vals = [(int(buf[cta, u, ev]) - int(buf[cta, u, 1])) / 1000.0
                    for u in range(8, 63) if buf[cta, u, ev] and buf[cta, u, 1]]
            if vals:
                rows.append((statistics.median(vals), ev, min(vals), max(vals)))
        for med, ev, lo, hi in sorted(rows):
            print(f"  {med:8.2f}  [{lo:7.2f} {hi:7.2f}]  {NAMES.get(ev, ev)}")
        per = [(int(buf[cta, u + 1, 1]) - int(buf[cta, u, 1])) / 1000.0 for u in range(8, 62)]
        print(f"  unit period median {statistics.median(per):.2f} us")


if __name__ == "__main__":
    args = [a for a in sys.argv[1:] if not a.startswith("--")]
    main(*args[:1], all_ctas="--all-ctas" in sys.argv[1:])
