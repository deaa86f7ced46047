"""Benchmark of the batch-1 MoE layer on B200: decode tokens/s and µs per MoE layer.

Default workload (one step): 1000 sequential decode tokens through one full-shape MoE layer
(hidden 4096, 512 experts, top-4 routed + 1 shared, intermediate 1024, 4-bit experts, fp32
activations), router logits forced so that expert selection is uniform over the 512 experts.
All tokens run in ONE launch of the engine kernel, strictly one after another (token t+1
computes only after token t's output is written). The data-independent tensors of the layer
(router, shared expert, shared gate) exist in 16 copies used round-robin by consecutive
tokens, so that neither they nor the routed experts are re-read out of the 126 MB L2: each
token's working set was last touched at least 15 tokens (>600 MB of traffic) earlier, as in a
real model where every layer's tensors are read once per token.

Prints ONE JSON line (rank 0). Multi-GPU (torchrun): replicas only -- every rank runs its own
token stream on its own GPU with no collective on the data path; the time is the max over
ranks and `value` counts the tokens of all ranks.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s & µs/layer (batch 1); achieved HBM GB/s vs peak"
REPLICAS = 16
# The arithmetic of the expert GEMVs: codes (u4 / u2) times x re-encoded per 32-column slice
# as three signed 8-bit digit planes, integer dp4a products, fp32 combine and accumulation;
# router dot products are fp32 x fp32 accumulated in binary64.
DTYPE = "u4/u2 x s8x3-digit dp4a -> fp32 (router f32->f64)"
# the arithmetic of each selectable dot-product form (fmoe_set_dot_form)
FORMS = {"digits": (0, DTYPE),
         "fma": (1, "u4/u2 -> f32, fma(q, s*x, z*x) per weight -> fp32 (router f32->f64)"),
         "naive": (2, "u4/u2 -> f32, (q*s + z)*x per weight -> fp32 (router f32->f64)")}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="full_q4",
                    choices=["full_q4", "full_q4_natural", "full_q2", "tiny", "stack_q4_uniform",
                             "stack_q4_skewed", "stack_q2"])
    ap.add_argument("--tokens", type=int, default=0, help="tokens per step (0 = workload's)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the number of routed experts (small cases for profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--form", default="digits", choices=sorted(FORMS),
                    help="dot-product form of the expert GEMVs (the pages' FMA comparison)")
    return ap.parse_args()


def dist_info():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(value: float, device, world: int) -> float:
    """The maximum of `value` over all ranks (one all-reduce; identity on one rank)."""
    if world <= 1:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def arm_config(wl, T: int, world: int, form: str = "digits") -> dict:
    """The `config` object of the JSON line; both arms report the same one."""
    stack = wl.layers > 1
    return {"workload": wl.name, "hidden": wl.H, "experts": wl.E, "top_k": wl.K,
            "shared_experts": 1, "inter": wl.I, "bits": wl.bits, "group": 64,
            "layers": wl.layers, "tokens_per_step": T, "routing": wl.routing,
            "launches_per_step": 1,
            "l2": ("inputs larger than L2: 16 round-robin copies of router/shared expert, "
                   "512 routed experts (3.6 GB)") if not stack else
                  "inputs larger than L2: every layer's tensors once per token",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "dot_form": form}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "bit_dequant_expert_gemv_b200", "csrc")
    for n in sorted(os.listdir(d)):
        with open(os.path.join(d, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """Per-token DRAM bytes of the engine kernel from the committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", f"engine_{workload}_dram.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_sources_sha256_16") != kernel_hash():
        return None
    try:
        return float(kv["dram_bytes_per_token"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
        else:
            self.lines = []

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
def _oracle_tokens(wl_name: str, experts: int, seconds: float, worker: int):
    """One oracle process: route + layer for fresh tokens of the workload (token 0's routed
    experts, so that only K + 1 experts are materialised) until `seconds` of wall time are
    spent. Returns (tokens, seconds). Runs in a spawned process for the all-cores figure."""
    import dataclasses

    import numpy as np

    import oracle
    import synth
    from oracle.workload import HostLayer
    wl = synth.WORKLOADS[wl_name]
    if experts:
        wl = dataclasses.replace(wl, E=experts)
    o = oracle.load()
    hl = HostLayer(o, wl, 0)
    bias = synth.logit_bias(wl, tokens=1)
    b0 = None if bias is None else bias[0, 0]
    x0 = synth.token_inputs(wl, 0, 1)[0].astype(np.float64)
    idx, w, _, _ = o.route(x0, hl.router, b0, wl.K)
    layer = hl.as_dict(idx)
    t_first = 1 + 64 * worker
    xs = synth.token_inputs(wl, t_first, 64)
    rs = synth.token_inputs(wl, t_first, 64, kind=synth.KIND_RES)
    n, t0 = 0, time.perf_counter()
    while n < 64:
        x = xs[n].astype(np.float64)
        o.route(x, hl.router, b0, wl.K)
        o.layer_forced(layer, x, rs[n].astype(np.float64), idx, w)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    return n, time.perf_counter() - t0


def cpu_baseline(wl, seconds: float, procs: int = 0, base: str | None = None):
    """The oracle (plain C, binary64) on this host: the same layer shape, a bounded sample of
    tokens (fresh x each) through the router and the routed experts of token 0 plus the shared
    expert, for about `seconds` of wall time. procs = 0 uses every core: that many independent
    oracle processes (spawned) on disjoint tokens, throughput summed; the single-thread figure
    is reported beside it."""
    import multiprocessing as mp
    ncpu = os.cpu_count() or 1
    name = base or wl.name
    ex = wl.E if wl.E != 512 else 0
    n1, dt1 = _oracle_tokens(name, ex, seconds / 2, 0)
    single = n1 / dt1
    P = procs or ncpu
    tot, dmax = n1, dt1
    if P > 1:
        with mp.get_context("spawn").Pool(P) as pool:
            res = pool.starmap(_oracle_tokens, [(name, ex, seconds / 2, i) for i in range(P)])
        tot = sum(r[0] for r in res)
        dmax = max(r[1] for r in res)
    value = tot / dmax
    layers = wl.layers
    sample = (f"{tot} tokens of one {wl.name} layer shape (router + softmax/top-{wl.K} over "
              f"{wl.E} + {wl.K} routed experts + shared expert, binary64) in {P} independent "
              f"oracle processes, {dmax:.1f} s; single thread {single:.3f} tokens/s "
              f"({n1} tokens, {dt1:.1f} s); host has {ncpu} cores")
    if layers > 1:
        sample += f"; stack figure extrapolated as the per-layer rate / {layers} layers"
    return {"value": value / layers, "unit": "tokens/s", "cores": P, "kind": "oracle",
            "sample": sample, "seconds": dmax, "single_thread_value": single / layers}


def run_reference(args):
    """The oracle arm: the plain C oracle (binary64) on this host's cores (one process per
    core, disjoint tokens), timed on a bounded sample of the same workload each step. Under
    torchrun only rank 0 runs it."""
    rank, _, world = dist_info()
    if rank != 0:
        return
    import synth
    wl0 = synth.WORKLOADS[args.workload]
    per_step = max(2.0, min(args.cpu_seconds, 60.0) / max(1, args.steps))
    for _ in range(args.warmup):  # untimed, short: page in the oracle, its inputs and weights
        cpu_baseline(wl0, 0.5)
    vals, samples, secs, cores = [], [], [], 1
    for _ in range(args.steps):
        r = cpu_baseline(wl0, per_step)
        vals.append(r["value"])
        samples.append(r["sample"])
        secs.append(r["seconds"])
        cores = r["cores"]
        if len(vals) * per_step > 120:
            break
    v = statistics.median(vals)
    sample = f"{len(vals)} steps, each {samples[0]}"
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": len(vals), "warmup": args.warmup,
            "ms_per_step": 1000.0 * statistics.median(secs), "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(wl0, args.tokens or wl0.tokens, world, args.form),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
def run_ours(args):
    import numpy as np
    import torch

    rank, local_rank, world = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)

    import bit_dequant_expert_gemv_b200 as fmoe
    import synth
    from bit_dequant_expert_gemv_b200.workload import build_layer, token_inputs_dev
    fmoe.build()
    fmoe.set_dot_form(FORMS[args.form][0])

    wl = synth.WORKLOADS[args.workload]
    if args.experts:
        import dataclasses
        wl = dataclasses.replace(wl, E=args.experts, name=f"{wl.name}_E{args.experts}")
    stack = wl.layers > 1
    T = args.tokens or wl.tokens
    # rank r runs its own stream of tokens (different x), same weights
    t_base = rank * T
    torch.manual_seed(0)

    if stack:
        dls = [build_layer(wl, l, device=dev) for l in range(wl.layers)]
        descs = [d.desc for d in dls]
        bias_np = synth.logit_bias(wl, tokens=T)
        h_in = token_inputs_dev(wl, t_base, T, device=dev)
        h_out = torch.empty_like(h_in)
        bias = None if bias_np is None else torch.from_numpy(bias_np).to(dev)
        graph = fmoe.StackGraph(descs, h_in, h_out, bias=bias, eps=wl.eps, tokens_per_launch=0)
        layers_per_step = T * wl.layers
        bytes_per_layer = wl.K * fmoe.expert_bytes(wl.H, wl.I, wl.bits) + \
            fmoe.expert_bytes(wl.H, wl.I, wl.bits) + wl.E * wl.H * 4
        step = lambda: graph.launch()  # noqa: E731
    else:
        dl = build_layer(wl, 0, device=dev)
        descs = [dl.desc]
        keep = []
        for r in range(1, REPLICAS):
            router = dl.router.clone()
            g = None if dl.gate is None else dl.gate.clone()
            sh = None if dl.shared is None else dl.shared.clone()
            keep.append((router, g, sh))
            descs.append(fmoe.LayerDesc(wl.H, wl.I, wl.E, wl.K, wl.bits, dl.experts, dl.stride, sh,
                                        router, g))
        x = token_inputs_dev(wl, t_base, T, device=dev)
        res = token_inputs_dev(wl, t_base, T, kind=synth.KIND_RES, device=dev)
        bias_np = synth.logit_bias(wl, tokens=T)
        bias = None if bias_np is None else torch.from_numpy(np.ascontiguousarray(bias_np[:, 0])).to(dev)
        out = torch.empty_like(x)
        layers_per_step = T
        bytes_per_layer = (wl.K + 1) * fmoe.expert_bytes(wl.H, wl.I, wl.bits) + wl.E * wl.H * 4
        step = lambda: fmoe.moe_layer_seq(descs, x, res, bias, out=out)  # noqa: E731

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step()
    if fmoe.sync_status() != 0:
        raise RuntimeError("device status after warm-up: " + fmoe.last_error())

    # ---- timed region: K steps, per-launch events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    l0 = fmoe.launch_count()
    with ClockSampler(local_rank) as clk:
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("timed")
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
        torch.cuda.nvtx.range_pop()
    launches = fmoe.launch_count() - l0
    if fmoe.sync_status() != 0:
        raise RuntimeError("device status after timing: " + fmoe.last_error())
    total_ms = start.elapsed_time(stop)
    total_ms = max_over_ranks(total_ms, dev, world)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_per_step = total_ms / args.steps

    # ---- end to end through the host-buffer entry point (single-layer workloads)
    e2e = None
    if not args.no_e2e and not stack:
        xh = x.cpu().pin_memory()
        rh = res.cpu().pin_memory()
        bh = None if bias is None else bias.cpu().pin_memory()
        oh = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        for _ in range(2):
            fmoe.moe_layer_seq_host(descs, xh, rh, bh, oh)
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 30))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            fmoe.moe_layer_seq_host(descs, xh, rh, bh, oh)
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = a.elapsed_time(b) / n_e2e
        e2e_ms = max_over_ranks(e2e_ms, dev, world)
        h2d = xh.numel() * 4 + rh.numel() * 4 + (0 if bh is None else bh.numel() * 4)
        d2h = oh.numel() * 4
        e2e = {"value": world * T / (e2e_ms / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    # ---- CPU baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(wl, args.cpu_seconds, base=args.workload)

    if rank == 0:
        hbm, peak_kind = peaks()
        bytes_per_launch = bytes_per_layer * layers_per_step
        achieved = bytes_per_launch / (launch_ms / 1000.0) / 1e9
        traffic_tok = recorded_traffic(args.workload)
        value = world * T / (ms_per_step / 1000.0)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": FORMS[args.form][1], "data": "synthetic",
            "config": arm_config(wl, T, world, args.form),
            "us_per_layer": ms_per_step * 1000.0 / layers_per_step,
            "gbs_algorithmic": bytes_per_layer * layers_per_step / (ms_per_step / 1000.0) / 1e9,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "bytes_per_launch": bytes_per_launch,
                         "bytes_per_token_layer": bytes_per_layer,
                         "traffic": None if traffic_tok is None else traffic_tok * layers_per_step,
                         "kernel": "fmoe::engine_kernel", "launch_ms": launch_ms},
            "clocks": clk.summary(),
            "gpu_launches": int(launches),
        }
        if e2e:
            line["e2e"] = e2e
        if cpu:
            line["cpu_baseline"] = {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample",
                                                        "single_thread_value")}
        print(json.dumps(line), flush=True)
    if stack:
        graph.close()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
