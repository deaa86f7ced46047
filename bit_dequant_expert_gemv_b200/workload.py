"""Device-resident synthetic MoE layers: seeded binary32 weights drawn on the GPU (synth) and
packed in place by the library's own pack kernel, so full-size models never pass through the
host. Used by the benchmark and by the GPU tests."""
from __future__ import annotations

from dataclasses import dataclass

import synth
from synth import KIND_GATEVEC, KIND_ROUTER, MAT_DOWN, MAT_GATE, MAT_UP, Workload, stream_id

from . import LayerDesc, expert_bytes, pack, qmat_bytes


@dataclass
class DeviceLayer:
    experts: object          # uint8 [E * stride]
    stride: int
    shared: object           # uint8 blob or None
    router: object           # float32 [E, H]
    gate: object             # float32 [H] or None
    desc: LayerDesc


def _fill_expert(wl: Workload, layer: int, e: int, blob, tmp, shared: bool):
    H, I, bits = wl.H, wl.I, wl.bits
    kind = synth.KIND_SHARED if shared else synth.KIND_EXPERT
    off = 0
    for m, (rows, cols) in ((MAT_GATE, (I, H)), (MAT_UP, (I, H)), (MAT_DOWN, (H, I))):
        w = tmp[: rows * cols]
        synth.normal_dev(w, wl.seed, stream_id(kind, layer, e, m), sigma=wl.w_sigma)
        nb = qmat_bytes(rows, cols, bits)
        pack(w.view(rows, cols), bits, out=blob[off: off + nb])
        off += nb


def build_layer(wl: Workload, layer: int, device="cuda", shared: bool | None = None,
                gate: bool | None = None, experts_tensor=None) -> DeviceLayer:
    """All E experts of layer `layer` (plus shared expert, router, gate) on the device.
    `experts_tensor` may supply one preallocated uint8 buffer of E * expert_bytes."""
    import torch
    H, I, E = wl.H, wl.I, wl.E
    shared = wl.shared if shared is None else shared
    gate = shared if gate is None else gate
    eb = expert_bytes(H, I, wl.bits)
    experts = experts_tensor if experts_tensor is not None else torch.empty(E * eb, dtype=torch.uint8, device=device)
    tmp = torch.empty(I * H, dtype=torch.float32, device=device)
    for e in range(E):
        _fill_expert(wl, layer, e, experts[e * eb:(e + 1) * eb], tmp, shared=False)
    sh = None
    if shared:
        sh = torch.empty(eb, dtype=torch.uint8, device=device)
        _fill_expert(wl, layer, 0, sh, tmp, shared=True)
    router = torch.empty(E * H, dtype=torch.float32, device=device)
    synth.normal_dev(router, wl.seed, stream_id(KIND_ROUTER, layer), sigma=wl.r_sigma)
    router = router.view(E, H)
    g = None
    if gate:
        g = torch.empty(H, dtype=torch.float32, device=device)
        synth.normal_dev(g, wl.seed, stream_id(KIND_GATEVEC, layer), sigma=wl.r_sigma)
    del tmp
    desc = LayerDesc(H, I, E, wl.K, wl.bits, experts, eb, sh, router, g)
    return DeviceLayer(experts, eb, sh, router, g, desc)


def token_inputs_dev(wl: Workload, t0: int, n: int, kind: int = synth.KIND_X, device="cuda"):
    import torch
    t = torch.empty(n * wl.H, dtype=torch.float32, device=device)
    synth.normal_dev(t, wl.seed, stream_id(kind), offset=t0 * wl.H, sigma=1.0)
    return t.view(n, wl.H)
