"""Host-side copies of the synthetic workloads for the oracle (test infrastructure).

Weights come from the same seeded generator as the device side (synth, host implementation)
and are packed by the ORACLE's quantiser, never by the CUDA library. Only the experts a check
needs are materialised, so full-size layers stay cheap on the host."""
from __future__ import annotations

import numpy as np

import synth
from synth import MAT_DOWN, MAT_GATE, MAT_UP, Workload


def expert_blob(o, wl: Workload, layer: int, e: int, shared: bool = False) -> np.ndarray:
    parts = [o.quantise(synth.matrix_host(wl, layer, e, m, shared=shared), wl.bits)
             for m in (MAT_GATE, MAT_UP, MAT_DOWN)]
    return np.concatenate(parts)


class HostLayer:
    """Lazily materialised oracle view of one layer."""

    def __init__(self, o, wl: Workload, layer: int, shared: bool | None = None, gate: bool | None = None):
        self.o, self.wl, self.layer = o, wl, layer
        self.shared_on = wl.shared if shared is None else shared
        self.gate_on = self.shared_on if gate is None else gate
        self.router = synth.router_host(wl, layer)
        self.gate = synth.gatevec_host(wl, layer) if self.gate_on else None
        self.shared = expert_blob(o, wl, layer, 0, shared=True) if self.shared_on else None
        self.blobs: dict[int, np.ndarray] = {}

    def blob(self, e: int) -> np.ndarray:
        if e not in self.blobs:
            self.blobs[e] = expert_blob(self.o, self.wl, self.layer, e)
        return self.blobs[e]

    def as_dict(self, need=()) -> dict:
        for e in need:
            self.blob(int(e))
        wl = self.wl
        return dict(H=wl.H, I=wl.I, E=wl.E, K=wl.K, bits=wl.bits,
                    experts=[self.blobs.get(e) for e in range(wl.E)], shared=self.shared,
                    router=self.router, shared_gate=self.gate)

    def forward(self, x, res, bias=None):
        """Route with the oracle, materialise the chosen experts, run the oracle layer."""
        idx, w, logits, p = self.o.route(x, self.router, bias, self.wl.K)
        out = self.o.layer_forced(self.as_dict(idx), x, res, idx, w)
        return out, idx, w, logits

    def forced(self, x, res, idx, w):
        return self.o.layer_forced(self.as_dict(idx), x, res, idx, w)
