"""Shared checks for the GPU parity tests (CUDA path vs the CPU oracle)."""
from __future__ import annotations

import numpy as np

TIE = 1e-6          # logits closer than this may be ordered either way
W_TOL = 1e-6        # routing weights
ABS_TOL = 2e-3      # output activations: max-abs
REL_L2 = 1e-3       # output activations: relative L2 per token


def check_out(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err <= ABS_TOL and rel <= REL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {rel:.3e}"
    return err, rel


def check_routing(idx_gpu, w_gpu, logits, K):
    """idx bit-exact except inside the tie band; order by oracle logits (ties either way).
    Returns True when the selection is exactly the oracle's."""
    idx_gpu = [int(i) for i in np.asarray(idx_gpu).reshape(-1)]
    logits = np.asarray(logits, dtype=np.float64)
    E = len(logits)
    order = np.lexsort((np.arange(E), -logits))
    want = [int(i) for i in order[:K]]
    assert len(set(idx_gpu)) == K and all(0 <= i < E for i in idx_gpu), idx_gpu
    kth = logits[order[K - 1]]
    nxt = logits[order[K]] if K < E else -np.inf
    if kth - nxt >= TIE:
        assert set(idx_gpu) == set(want), (idx_gpu, want)
    else:  # tie band: every chosen expert must be within TIE of the K-th logit or above it
        assert all(logits[i] >= kth - TIE for i in idx_gpu), (idx_gpu, want)
    for a, b in zip(idx_gpu, idx_gpu[1:]):
        assert logits[a] >= logits[b] - TIE, ("order", idx_gpu)
    exact = idx_gpu == want
    if w_gpu is not None:
        sel = np.array(idx_gpu)
        p = np.exp(logits[sel] - logits.max())
        wref = p / p.sum()
        assert np.abs(np.asarray(w_gpu, dtype=np.float64).reshape(-1) - wref).max() <= W_TOL, (w_gpu, wref)
    return exact


def renorm_weights(logits, idx):
    logits = np.asarray(logits, dtype=np.float64)
    p = np.exp(logits[np.asarray(idx)] - logits.max())
    return p / p.sum()
