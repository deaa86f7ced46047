"""B200 (sm_100a) batch-1 MoE layer with 4-bit / 2-bit group-affine dequantising expert GEMVs.

Thin binding over the C ABI of ``libfmoe.so`` (``include/fmoe.h``): argument marshalling
only. Every step of the computation runs in the library's CUDA kernels; PyTorch only supplies
device memory and streams. There is no CPU fallback: importing the package fails loudly when
the compiled library is missing.
"""
from __future__ import annotations

import ctypes as C
import os

from ._build import LIB, build, stale  # noqa: F401

FMOE_OK, FMOE_ERR_INVALID, FMOE_ERR_ALIGN, FMOE_ERR_CUDA, FMOE_ERR_NOMEM, FMOE_ERR_TIMEOUT, \
    FMOE_ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5, -6


class FmoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


_SIGS = {
    "fmoe_last_error": (C.c_char_p, []),
    "fmoe_version": (C.c_int, []),
    "fmoe_sync_status": (C.c_int, [C.c_void_p]),
    "fmoe_set_wait_budget_ns": (None, [C.c_uint64]),
    "fmoe_set_fault_injection": (None, [C.c_int]),
    "fmoe_qmat_bytes": (C.c_size_t, [C.c_int] * 3),
    "fmoe_expert_bytes": (C.c_size_t, [C.c_int] * 3),
    "fmoe_pack": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "fmoe_pack_q4": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "fmoe_pack_q2": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "fmoe_route": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                             C.c_void_p, C.c_void_p, C.c_void_p]),
    "fmoe_expert_gemv": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p,
                                   C.c_void_p, C.c_void_p]),
    "fmoe_moe_layer": (C.c_int, [C.c_void_p] * 8),
    "fmoe_moe_layer_noalloc": (C.c_int, [C.c_void_p] * 8),
    "fmoe_moe_layer_seq": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "fmoe_moe_layer_seq_host": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int,
                                          C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                          C.c_void_p]),
    "fmoe_moe_stack": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_float,
                                 C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "fmoe_stack_graph_create": (C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p,
                                          C.c_float, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                          C.c_void_p]),
    "fmoe_stack_graph_launch": (C.c_int, [C.c_void_p, C.c_void_p]),
    "fmoe_stack_graph_destroy": (C.c_int, [C.c_void_p]),
    "fmoe_describe_geometry": (C.c_int, [C.c_int] * 8 + [C.c_void_p, C.c_int]),
    "fmoe_set_dot_form": (C.c_int, [C.c_int]),
    "fmoe_launch_count": (C.c_uint64, []),
}
_lib = None


def lib():
    """The loaded libfmoe.so; raises ImportError when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError(f"libfmoe.so is not built ({LIB}); run __graft_entry__.build() "
                              "or python -m bit_dequant_expert_gemv_b200._build")
        L = C.CDLL(LIB)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def last_error() -> str:
    return lib().fmoe_last_error().decode()


def _ck(name: str, rc: int):
    if rc != FMOE_OK:
        raise FmoeError(name, rc, last_error())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


class LayerDesc(C.Structure):
    """Mirror of fmoe_layer_desc; keeps the tensors it points to alive."""
    _fields_ = [("hidden", C.c_int), ("inter", C.c_int), ("n_experts", C.c_int),
                ("top_k", C.c_int), ("bits", C.c_int), ("experts", C.c_void_p),
                ("expert_stride", C.c_size_t), ("shared_expert", C.c_void_p),
                ("router", C.c_void_p), ("shared_gate", C.c_void_p)]

    def __init__(self, hidden, inter, n_experts, top_k, bits, experts, expert_stride, shared,
                 router, shared_gate):
        super().__init__(hidden, inter, n_experts, top_k, bits, experts.data_ptr(), expert_stride,
                         None if shared is None else shared.data_ptr(), router.data_ptr(),
                         None if shared_gate is None else shared_gate.data_ptr())
        self._keep = (experts, shared, router, shared_gate)


def _descs(layers):
    if isinstance(layers, LayerDesc):
        layers = [layers]
    arr = (LayerDesc * len(layers))()
    for i, d in enumerate(layers):
        C.memmove(C.addressof(arr[i]), C.addressof(d), C.sizeof(LayerDesc))
    return arr, len(layers)


# --------------------------------------------------------------------------------- sizes
def qmat_bytes(rows: int, cols: int, bits: int) -> int:
    return int(lib().fmoe_qmat_bytes(rows, cols, bits))


def expert_bytes(hidden: int, inter: int, bits: int) -> int:
    return int(lib().fmoe_expert_bytes(hidden, inter, bits))


GEOMETRY_FIELDS = ("H I E K bits route_on shared_on routed_on gate_on rc_h rs_h rc_i rs_i q_gu nr "
                   "rseg rcols rrows au hr ad dr nseg sh wh gh si wi pi ji stage_bytes nA nB "
                   "o_ringA o_ringB o_x o_h o_red o_oacc o_misc o_bar oacc_n smem_bytes "
                   "consumer_warps max_rows_thread max_rows_warp red_slot gpass").split()


def describe_geometry(H, I, E, K, bits, flags=15, max_smem=232448, sms=148) -> dict:
    buf = (C.c_int64 * len(GEOMETRY_FIELDS))()
    n = lib().fmoe_describe_geometry(H, I, E, K, bits, flags, max_smem, sms, buf,
                                     len(GEOMETRY_FIELDS))
    if n < 0:
        raise FmoeError("fmoe_describe_geometry", n, last_error())
    return {k: int(buf[i]) for i, k in enumerate(GEOMETRY_FIELDS[:n])}


def set_dot_form(form: int):
    """0: digit planes + dp4a (default), 1: literal fma(q, s*x, z*x), 2: naive (q*s + z)*x."""
    _ck("fmoe_set_dot_form", lib().fmoe_set_dot_form(int(form)))


def launch_count() -> int:
    return int(lib().fmoe_launch_count())


def set_wait_budget_ns(ns: int):
    lib().fmoe_set_wait_budget_ns(int(ns))


def set_fault_injection(flags: int):
    lib().fmoe_set_fault_injection(int(flags))


def sync_status(stream=None) -> int:
    """Synchronise `stream`, return (and clear) the sticky device status (0 = OK)."""
    return int(lib().fmoe_sync_status(_stream(stream)))


# --------------------------------------------------------------------------------- entry points
def pack(w, bits: int, out=None, stream=None):
    import torch
    assert w.is_cuda and w.dtype == torch.float32 and w.is_contiguous() and w.dim() == 2
    rows, cols = w.shape
    if out is None:
        out = torch.empty(qmat_bytes(rows, cols, bits), dtype=torch.uint8, device=w.device)
    _ck("fmoe_pack", lib().fmoe_pack(_ptr(w), rows, cols, bits, _ptr(out), _stream(stream)))
    return out


def route(x, router, bias, top_k: int, idx=None, weight=None, stream=None):
    import torch
    E, H = router.shape
    idx = torch.empty(top_k, dtype=torch.int32, device=x.device) if idx is None else idx
    weight = torch.empty(top_k, dtype=torch.float32, device=x.device) if weight is None else weight
    _ck("fmoe_route", lib().fmoe_route(_ptr(x), _ptr(router), _ptr(bias), H, E, top_k, _ptr(idx),
                                      _ptr(weight), _stream(stream)))
    return idx, weight


def expert_gemv(blob, hidden: int, inter: int, bits: int, x, y=None, stream=None):
    import torch
    y = torch.empty(hidden, dtype=torch.float32, device=x.device) if y is None else y
    _ck("fmoe_expert_gemv", lib().fmoe_expert_gemv(_ptr(blob), hidden, inter, bits, _ptr(x), _ptr(y),
                                                  _stream(stream)))
    return y


def moe_layer(desc: LayerDesc, x, residual=None, bias=None, out=None, idx=None, weight=None,
              stream=None):
    import torch
    out = torch.empty_like(x) if out is None else out
    arr, _ = _descs(desc)
    _ck("fmoe_moe_layer", lib().fmoe_moe_layer(arr, _ptr(x), _ptr(residual), _ptr(bias), _ptr(out),
                                              _ptr(idx), _ptr(weight), _stream(stream)))
    return out


def moe_layer_noalloc(desc: LayerDesc, x, residual=None, bias=None, out=None, idx=None,
                      weight=None, stream=None):
    """fmoe_moe_layer_noalloc: one token with the library's fixed scratch array (no device
    allocation inside the call; `out` must be given by callers that allocate nothing)."""
    import torch
    out = torch.empty_like(x) if out is None else out
    arr, _ = _descs(desc)
    _ck("fmoe_moe_layer_noalloc",
        lib().fmoe_moe_layer_noalloc(arr, _ptr(x), _ptr(residual), _ptr(bias), _ptr(out),
                                     _ptr(idx), _ptr(weight), _stream(stream)))
    return out


NOALLOC_SCRATCH_BYTES = 128 * 1024


def moe_layer_seq(descs, x, residual=None, bias=None, out=None, idx=None, weight=None,
                  stream=None):
    import torch
    T = x.shape[0]
    out = torch.empty_like(x) if out is None else out
    arr, n = _descs(descs)
    _ck("fmoe_moe_layer_seq", lib().fmoe_moe_layer_seq(arr, n, _ptr(x), _ptr(residual), T,
                                                      _ptr(bias), _ptr(out), _ptr(idx),
                                                      _ptr(weight), _stream(stream)))
    return out


def moe_layer_seq_host(descs, x, residual, bias, out, idx=None, weight=None, stream=None):
    """Host-buffer variant (pinned torch CPU tensors): copies in, runs, copies out on `stream`."""
    arr, n = _descs(descs)
    _ck("fmoe_moe_layer_seq_host", lib().fmoe_moe_layer_seq_host(
        arr, n, _ptr(x), _ptr(residual), x.shape[0], _ptr(bias), _ptr(out), _ptr(idx), _ptr(weight),
        _stream(stream)))
    return out


def moe_stack(descs, h_in, bias=None, eps: float = 1e-6, h_out=None, idx_trace=None,
              h_trace=None, stream=None):
    import torch
    T = h_in.shape[0]
    h_out = torch.empty_like(h_in) if h_out is None else h_out
    arr, n = _descs(descs)
    _ck("fmoe_moe_stack", lib().fmoe_moe_stack(arr, n, _ptr(h_in), T, _ptr(bias), eps, _ptr(h_out),
                                              _ptr(idx_trace), _ptr(h_trace), _stream(stream)))
    return h_out


class StackGraph:
    """fmoe_moe_stack captured once into a CUDA graph (fixed buffers), replayed by launch()."""

    def __init__(self, descs, h_in, h_out, bias=None, eps: float = 1e-6, idx_trace=None,
                 h_trace=None, tokens_per_launch: int = 0):
        arr, n = _descs(descs)
        self._keep = (descs, h_in, h_out, bias, idx_trace, h_trace)
        self._g = C.c_void_p()
        _ck("fmoe_stack_graph_create", lib().fmoe_stack_graph_create(
            arr, n, _ptr(h_in), h_in.shape[0], _ptr(bias), eps, _ptr(h_out), _ptr(idx_trace),
            _ptr(h_trace), tokens_per_launch, C.byref(self._g)))

    def launch(self, stream=None):
        _ck("fmoe_stack_graph_launch", lib().fmoe_stack_graph_launch(self._g, _stream(stream)))

    def close(self):
        if self._g:
            lib().fmoe_stack_graph_destroy(self._g)
            self._g = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
