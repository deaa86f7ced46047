"""Seeded synthetic inputs for the MoE layer (weights, activations, forced routing).

This package holds none of the method's arithmetic: it only draws numbers. The same values
are produced on the host (``synth_host.c``, for the oracle side) and on the device
(``synth_dev.cu``, for the CUDA side, so that 100+ GB of weights never pass through the
host); see ``philox.h`` for the recipe. Every tensor of a workload is addressed by a
64-bit stream id built from (kind, layer, expert, matrix).
"""
from __future__ import annotations

import ctypes as C
import math
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(HERE, "libsynth_host.so")
DEV_LIB = os.path.join(HERE, "libsynth_dev.so")

KIND_EXPERT, KIND_SHARED, KIND_ROUTER, KIND_GATEVEC, KIND_X, KIND_RES, KIND_ROUTE = 1, 2, 3, 4, 5, 6, 7
MAT_GATE, MAT_UP, MAT_DOWN = 0, 1, 2

_lock = threading.Lock()
_host = None
_dev = None


def _stale(out, *srcs):
    return not os.path.exists(out) or os.path.getmtime(out) < max(os.path.getmtime(s) for s in srcs)


def build_host(force=False) -> str:
    srcs = [os.path.join(HERE, "synth_host.c"), os.path.join(HERE, "philox.h")]
    if force or _stale(HOST_LIB, *srcs):
        tmp = HOST_LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-I", HERE,
                        srcs[0], "-o", tmp], check=True)
        os.replace(tmp, HOST_LIB)
    return HOST_LIB


def build_dev(force=False, nvcc="nvcc") -> str:
    srcs = [os.path.join(HERE, "synth_dev.cu"), os.path.join(HERE, "philox.h")]
    if force or _stale(DEV_LIB, *srcs):
        tmp = DEV_LIB + f".tmp{os.getpid()}"
        subprocess.run([nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-Xcompiler", "-fPIC", "-shared", "-I", HERE, srcs[0], "-o", tmp,
                        "-lcudart"], check=True)
        os.replace(tmp, DEV_LIB)
    return DEV_LIB


def host_lib():
    global _host
    with _lock:
        if _host is None:
            L = C.CDLL(build_host())
            L.syn_philox_block.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
            L.syn_fill_normal.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64,
                                          C.c_uint64, C.c_float]
            L.syn_fill_u64.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64]
            _host = L
        return _host


def dev_lib():
    global _dev
    with _lock:
        if _dev is None:
            L = C.CDLL(build_dev())
            L.syn_fill_normal_dev.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64,
                                              C.c_uint64, C.c_float, C.c_void_p]
            L.syn_fill_normal_dev.restype = C.c_int
            _dev = L
        return _dev


def stream_id(kind: int, layer: int = 0, expert: int = 0, matrix: int = 0) -> int:
    return (kind << 56) | (layer << 40) | (expert << 16) | matrix


def scale_for(sigma: float) -> float:
    """binary32 factor turning the centred Irwin-Hall integer into a value of std sigma."""
    return float(np.float32(sigma / math.sqrt(8.0 * (65536.0 ** 2 - 1.0) / 12.0)))


def philox_block(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.empty(4, dtype=np.uint64)
    host_lib().syn_philox_block(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def normal_host(n: int, seed: int, st: int, offset: int = 0, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(int(n), dtype=np.float32)
    host_lib().syn_fill_normal(out.ctypes.data, int(n), seed, st, offset, scale_for(sigma))
    return out


def normal_dev(t, seed: int, st: int, offset: int = 0, sigma: float = 1.0, stream=None):
    """Fill a contiguous float32 CUDA tensor ``t`` in place."""
    import torch
    assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    s = torch.cuda.current_stream(t.device).cuda_stream if stream is None else stream
    rc = dev_lib().syn_fill_normal_dev(t.data_ptr(), t.numel(), seed, st, offset,
                                       scale_for(sigma), s)
    if rc != 0:
        raise RuntimeError("synth: device fill failed")
    return t


def u64_host(n: int, seed: int, st: int) -> np.ndarray:
    out = np.empty(int(n), dtype=np.uint64)
    host_lib().syn_fill_u64(out.ctypes.data, int(n), seed, st)
    return out


def permutation(n: int, seed: int, st: int) -> np.ndarray:
    """Fisher-Yates shuffle of 0..n-1 driven by Philox words (modulo bias < 2^-40)."""
    r = u64_host(n, seed, st)
    p = np.arange(n, dtype=np.int64)
    for i in range(n - 1, 0, -1):
        j = int(r[i] % np.uint64(i + 1))
        p[i], p[j] = p[j], p[i]
    return p


# ---------------------------------------------------------------------------------------
# Workload recipes: shapes, distributions and seeds of the five configurations.
# ---------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    I: int
    E: int
    K: int
    bits: int
    seed: int
    layers: int = 1
    tokens: int = 1
    w_sigma: float = 0.02      # expert weights before quantisation
    r_sigma: float = 0.02      # router and shared-gate vector
    routing: str = "natural"   # natural | uniform | skewed
    shared: bool = True
    eps: float = 1e-6
    note: str = ""
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    # hidden 256, 16 experts, top-2, intermediate 128, 1 shared expert, q4, seed 0
    "tiny": Workload("tiny", 256, 128, 16, 2, 4, seed=0, tokens=8),
    # hidden 4096, 512 experts, top-4 + shared, intermediate 1024, q4; 1000 tokens with the
    # router forced to a uniform selection (each expert chosen ~7.8 times)
    "full_q4": Workload("full_q4", 4096, 1024, 512, 4, 4, seed=1, tokens=1000, routing="uniform"),
    "full_q4_natural": Workload("full_q4_natural", 4096, 1024, 512, 4, 4, seed=1, tokens=1000),
    # same layer at 2-bit, 1000 tokens, natural routing
    "full_q2": Workload("full_q2", 4096, 1024, 512, 4, 2, seed=2, tokens=1000),
    # 60-layer 2-bit stack, 256 tokens
    "stack_q2": Workload("stack_q2", 4096, 1024, 512, 4, 2, seed=3, layers=60, tokens=256),
    # 24-layer 4-bit stack, 256 tokens, skewed (32 hot experts/layer take 70%) or uniform
    "stack_q4_skewed": Workload("stack_q4_skewed", 4096, 1024, 512, 4, 4, seed=4, layers=24,
                                tokens=256, routing="skewed"),
    "stack_q4_uniform": Workload("stack_q4_uniform", 4096, 1024, 512, 4, 4, seed=4, layers=24,
                                 tokens=256, routing="uniform"),
}

FORCE_BIAS = 64.0


def forced_experts(wl: Workload, tokens: int | None = None) -> np.ndarray | None:
    """[T, L, K] expert choices forced through the logit bias, or None for natural routing."""
    T = wl.tokens if tokens is None else tokens
    L, E, K = wl.layers, wl.E, wl.K
    if wl.routing == "natural":
        return None
    out = np.empty((T, L, K), dtype=np.int64)
    if wl.routing == "uniform":
        # token t takes positions K*t .. K*t+K-1 (mod E) of a seeded permutation, per layer
        for l in range(L):
            perm = permutation(E, wl.seed, stream_id(KIND_ROUTE, l, 0, 1))
            for t in range(T):
                out[t, l] = perm[(K * t + np.arange(K)) % E]
        return out
    if wl.routing == "skewed":
        hot_n = 32
        for l in range(L):
            perm = permutation(E, wl.seed, stream_id(KIND_ROUTE, l, 0, 2))
            hot, cold = perm[:hot_n], perm[hot_n:]
            r = u64_host(T * K * 2, wl.seed, stream_id(KIND_ROUTE, l, 0, 3))
            for t in range(T):
                chosen: list[int] = []
                for k in range(K):
                    u = float(r[(t * K + k) * 2] >> np.uint64(11)) / float(1 << 53)
                    pool = hot if u < 0.7 else cold
                    avail = [int(e) for e in pool if int(e) not in chosen]
                    j = int(r[(t * K + k) * 2 + 1] % np.uint64(len(avail)))
                    chosen.append(avail[j])
                out[t, l] = chosen
        return out
    raise ValueError(wl.routing)


def logit_bias(wl: Workload, tokens: int | None = None) -> np.ndarray | None:
    """[T, L, E] float32 bias (+64 on the forced experts), or None for natural routing."""
    f = forced_experts(wl, tokens)
    if f is None:
        return None
    T, L, K = f.shape
    b = np.zeros((T, L, wl.E), dtype=np.float32)
    for t in range(T):
        for l in range(L):
            b[t, l, f[t, l]] = FORCE_BIAS
    return b


def token_inputs(wl: Workload, t0: int, n: int, kind: int = KIND_X) -> np.ndarray:
    """[n, H] float32 N(0,1)-shaped token vectors t0 .. t0+n-1 (x or residual)."""
    return normal_host(n * wl.H, wl.seed, stream_id(kind), offset=t0 * wl.H, sigma=1.0).reshape(n, wl.H)


def matrix_host(wl: Workload, layer: int, expert: int, mat: int, shared: bool = False) -> np.ndarray:
    """fp32 weights of one expert matrix (gate/up: [I, H]; down: [H, I])."""
    rows, cols = (wl.I, wl.H) if mat != MAT_DOWN else (wl.H, wl.I)
    kind = KIND_SHARED if shared else KIND_EXPERT
    v = normal_host(rows * cols, wl.seed, stream_id(kind, layer, expert, mat), sigma=wl.w_sigma)
    return v.reshape(rows, cols)


def router_host(wl: Workload, layer: int) -> np.ndarray:
    return normal_host(wl.E * wl.H, wl.seed, stream_id(KIND_ROUTER, layer), sigma=wl.r_sigma).reshape(wl.E, wl.H)


def gatevec_host(wl: Workload, layer: int) -> np.ndarray:
    return normal_host(wl.H, wl.seed, stream_id(KIND_GATEVEC, layer), sigma=wl.r_sigma)
