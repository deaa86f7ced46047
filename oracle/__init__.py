"""CPU oracle of the batch-1 MoE layer (test infrastructure).

The oracle is a plain C implementation in binary64 (``fmoe_oracle.c``) of what the CUDA
library computes. Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg
of ``bench.py`` may import this package; the product library never does, and it shares no
code with it. This module only builds the shared object and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fmoe_oracle.c")
HDR = os.path.join(HERE, "fmoe_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")

_lock = threading.Lock()
_cache: dict[str, "Oracle"] = {}


def build(out: str = LIB, mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle with gcc (``mutant`` != 0 plants a known mistake, for the pin tests)."""
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR))
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           f"-DORC_MUTANT={int(mutant)}", "-I", HERE, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class OrcLayer(C.Structure):
    _fields_ = [("H", C.c_int), ("I", C.c_int), ("E", C.c_int), ("K", C.c_int), ("bits", C.c_int),
                ("experts", C.POINTER(C.c_void_p)), ("shared", C.c_void_p),
                ("router", C.c_void_p), ("shared_gate", C.c_void_p)]


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


class Oracle:
    """ctypes view of one build of the oracle."""

    def __init__(self, path: str):
        self.path = path
        L = C.CDLL(path)
        self.L = L
        vp, i, d, sz = C.c_void_p, C.c_int, C.c_double, C.c_size_t
        sig = {
            "orc_bf16_rne": (C.c_uint16, [C.c_float]),
            "orc_bf16_to_f32": (C.c_float, [C.c_uint16]),
            "orc_qmat_bytes": (sz, [i, i, i]),
            "orc_expert_bytes": (sz, [i, i, i]),
            "orc_quantise": (None, [vp, i, i, i, vp]),
            "orc_code": (i, [vp, i, i, i, i, i]),
            "orc_scale_bias": (None, [vp, i, i, i, i, i, vp, vp]),
            "orc_weight": (d, [vp, i, i, i, i, i]),
            "orc_dequant": (None, [vp, i, i, i, vp]),
            "orc_gemv": (None, [vp, i, i, i, vp, vp]),
            "orc_group_dot": (d, [i, vp, d, d, vp, i]),
            "orc_expert": (None, [vp, i, i, i, vp, vp, vp]),
            "orc_route": (None, [vp, vp, vp, i, i, i, vp, vp, vp, vp]),
            "orc_layer_forward": (i, [vp, vp, vp, vp, vp, vp, vp]),
            "orc_layer_forced": (i, [vp, vp, vp, vp, vp, vp]),
            "orc_rmsnorm": (None, [vp, i, d, vp]),
            "orc_stack": (i, [vp, i, vp, vp, d, vp, vp, vp]),
            "orc_mutant": (i, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args

    # -- sizes and bf16 ------------------------------------------------------------------
    def mutant(self) -> int:
        return self.L.orc_mutant()

    def qmat_bytes(self, rows, cols, bits) -> int:
        return int(self.L.orc_qmat_bytes(rows, cols, bits))

    def expert_bytes(self, hidden, inter, bits) -> int:
        return int(self.L.orc_expert_bytes(hidden, inter, bits))

    def bf16_rne(self, f: float) -> int:
        return int(self.L.orc_bf16_rne(C.c_float(f)))

    def bf16_to_f32(self, h: int) -> float:
        return float(self.L.orc_bf16_to_f32(h))

    # -- quantiser / decoder --------------------------------------------------------------
    def quantise(self, w, bits) -> np.ndarray:
        w = _f32(w)
        rows, cols = w.shape
        n = self.qmat_bytes(rows, cols, bits)
        if n == 0:
            raise ValueError(f"oracle quantise: illegal shape {w.shape} / bits {bits}")
        out = np.zeros(n, dtype=np.uint8)
        self.L.orc_quantise(_p(w), rows, cols, bits, _p(out))
        return out

    def code(self, qm, rows, cols, bits, r, c) -> int:
        return int(self.L.orc_code(_p(qm), rows, cols, bits, r, c))

    def scale_bias(self, qm, rows, cols, bits, r, g):
        s, z = C.c_double(), C.c_double()
        self.L.orc_scale_bias(_p(qm), rows, cols, bits, r, g, C.byref(s), C.byref(z))
        return s.value, z.value

    def dequant(self, qm, rows, cols, bits) -> np.ndarray:
        out = np.empty((rows, cols), dtype=np.float64)
        self.L.orc_dequant(_p(qm), rows, cols, bits, _p(out))
        return out

    def gemv(self, qm, rows, cols, bits, x) -> np.ndarray:
        x = _f64(x)
        y = np.empty(rows, dtype=np.float64)
        self.L.orc_gemv(_p(qm), rows, cols, bits, _p(x), _p(y))
        return y

    def group_dot(self, form, q, s, z, x) -> float:
        q = np.ascontiguousarray(q, dtype=np.int32)
        x = _f64(x)
        return float(self.L.orc_group_dot(form, _p(q), s, z, _p(x), len(q)))

    # -- expert / router / layer ----------------------------------------------------------
    def expert(self, blob, H, I, bits, x, want_h=False):
        x = _f64(x)
        y = np.empty(H, dtype=np.float64)
        h = np.empty(I, dtype=np.float64) if want_h else None
        self.L.orc_expert(_p(blob), H, I, bits, _p(x), _p(y), _p(h))
        return (y, h) if want_h else y

    def route(self, x, router, bias, K):
        x = _f64(x)
        router = _f32(router)
        E, H = router.shape
        bias = _f32(bias)
        idx = np.empty(K, dtype=np.int32)
        w = np.empty(K, dtype=np.float64)
        logits = np.empty(E, dtype=np.float64)
        p = np.empty(E, dtype=np.float64)
        self.L.orc_route(_p(x), _p(router), _p(bias), H, E, K, _p(idx), _p(w), _p(logits), _p(p))
        return idx, w, logits, p

    def _layer_struct(self, layer):
        """layer: dict(H, I, E, K, bits, experts=list of uint8 arrays or None, shared, router,
        shared_gate). Returns (struct, keepalive)."""
        E = layer["E"]
        ptrs = (C.c_void_p * E)()
        keep = []
        for e, blob in enumerate(layer["experts"]):
            if blob is not None:
                ptrs[e] = blob.ctypes.data
                keep.append(blob)
        router = _f32(layer["router"])
        gate = _f32(layer.get("shared_gate"))
        shared = layer.get("shared")
        keep += [router, gate, shared, ptrs]
        st = OrcLayer(layer["H"], layer["I"], E, layer["K"], layer["bits"],
                      C.cast(ptrs, C.POINTER(C.c_void_p)), _p(shared), _p(router), _p(gate))
        return st, keep

    def layer(self, layer, x, res, bias=None):
        st, keep = self._layer_struct(layer)
        x = _f64(x)
        res = None if res is None else _f64(res)
        out = np.empty(layer["H"], dtype=np.float64)
        idx = np.empty(layer["K"], dtype=np.int32)
        w = np.empty(layer["K"], dtype=np.float64)
        b = _f32(bias)
        rc = self.L.orc_layer_forward(C.byref(st), _p(x), _p(res), _p(b), _p(out), _p(idx), _p(w))
        if rc != 0:
            raise ValueError("oracle layer: a selected expert blob was not supplied")
        return out, idx, w

    def layer_forced(self, layer, x, res, idx, w):
        st, keep = self._layer_struct(layer)
        x = _f64(x)
        res = None if res is None else _f64(res)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        w = _f64(w)
        out = np.empty(layer["H"], dtype=np.float64)
        rc = self.L.orc_layer_forced(C.byref(st), _p(x), _p(res), _p(idx), _p(w), _p(out))
        if rc != 0:
            raise ValueError("oracle layer: a selected expert blob was not supplied")
        return out

    def rmsnorm(self, h, eps):
        h = _f64(h)
        x = np.empty_like(h)
        self.L.orc_rmsnorm(_p(h), len(h), eps, _p(x))
        return x

    def stack(self, layers, h_in, bias, eps, want_trace=False):
        Ln = len(layers)
        structs = (OrcLayer * Ln)()
        keep = []
        for l, ly in enumerate(layers):
            st, k = self._layer_struct(ly)
            structs[l] = st
            keep.append(k)
        H, K = layers[0]["H"], layers[0]["K"]
        h_in = _f64(h_in)
        out = np.empty(H, dtype=np.float64)
        idx = np.empty((Ln, K), dtype=np.int32)
        xt = np.empty((Ln, H), dtype=np.float64) if want_trace else None
        b = _f32(bias)
        rc = self.L.orc_stack(structs, Ln, _p(h_in), _p(b), eps, _p(out), _p(idx), _p(xt))
        if rc != 0:
            raise ValueError("oracle stack: a selected expert blob was not supplied")
        return (out, idx, xt) if want_trace else (out, idx)


def load(mutant: int = 0) -> Oracle:
    """Build (if needed) and load the oracle; ``mutant`` selects a planted-mistake build."""
    with _lock:
        key = f"m{mutant}"
        if key not in _cache:
            path = LIB if mutant == 0 else os.path.join(HERE, f"liboracle_m{mutant}.so")
            _cache[key] = Oracle(build(path, mutant))
        return _cache[key]
