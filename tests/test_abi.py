"""The C-ABI library loads on a machine without a GPU and exports every function that
include/fmoe.h declares; the host-only size helpers agree with the packed layout."""
import ctypes
import os
import re

import bit_dequant_expert_gemv_b200 as fmoe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fmoe.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)  # comments
    return sorted(set(re.findall(r"\b(fmoe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fmoe_pack_q4", "fmoe_pack_q2", "fmoe_route", "fmoe_expert_gemv", "fmoe_moe_layer",
              "fmoe_moe_stack", "fmoe_stack_graph_create", "fmoe_stack_graph_launch",
              "fmoe_stack_graph_destroy", "fmoe_moe_layer_noalloc"):
        assert n in names, n


def test_every_declared_function_is_exported():
    lib = ctypes.CDLL(fmoe.LIB)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_python_binding_covers_the_header():
    bound = set(fmoe._SIGS)
    missing = [n for n in declared_functions() if n not in bound]
    assert not missing, missing


def test_host_size_helpers():
    lib = fmoe.lib()
    assert lib.fmoe_expert_bytes(4096, 1024, 4) == 7_077_888
    assert lib.fmoe_expert_bytes(4096, 1024, 2) == 3_932_160
    assert lib.fmoe_qmat_bytes(1024, 4096, 4) == 1024 * 4096 // 2 + 1024 * 4096 // 16
    assert lib.fmoe_qmat_bytes(64, 100, 4) == 0   # columns not a multiple of 64
    assert lib.fmoe_qmat_bytes(64, 64, 3) == 0    # unsupported width
    assert lib.fmoe_version() >= 10000
