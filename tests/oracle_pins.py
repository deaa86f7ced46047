"""Pins of the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes an oracle handle and raises AssertionError when the oracle disagrees
with a fact fixed by the pages (tests/golden/pages_facts.json), by a library routine on a
special case (torch's bfloat16 rounding, numpy's softmax), by construction (weights placed
exactly on the quantisation grid), by a closed form, or by brute force (a dense numpy
evaluation of every expert written from the layout text). ``test_oracle_pins.py`` runs them
on the real oracle; ``test_oracle_mutants.py`` runs them on builds with a planted mistake.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pages_facts.json")
MiB = 1 << 20
GiB = 1 << 30


def facts():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------
# helpers independent of the oracle: numpy decoder and bf16 widening written from the
# layout text ("codes row-major, 32/bits codes per little-endian uint32 word, lowest column
# in the lowest bits; then per row and 64-column group a uint32 with bf16 scale in bits
# 0..15 and bf16 bias in bits 16..31").
# ---------------------------------------------------------------------------------------
def np_bf16_to_f64(u16):
    return (np.asarray(u16, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def np_decode(qm, rows, cols, bits):
    per = 32 // bits
    nbytes = rows * cols * bits // 8
    words = np.frombuffer(qm[:nbytes].tobytes(), dtype="<u4").reshape(rows, cols // per)
    shifts = (np.arange(per, dtype=np.uint32) * bits)
    codes = (words[:, :, None] >> shifts[None, None, :]) & np.uint32((1 << bits) - 1)
    codes = codes.reshape(rows, cols).astype(np.int64)
    sb = np.frombuffer(qm[nbytes:nbytes + rows * cols // 16].tobytes(), dtype="<u4").reshape(rows, cols // 64)
    s = np_bf16_to_f64(sb & 0xFFFF)
    z = np_bf16_to_f64(sb >> 16)
    return codes, s, z


def np_dense(qm, rows, cols, bits):
    q, s, z = np_decode(qm, rows, cols, bits)
    return q * np.repeat(s, 64, axis=1) + np.repeat(z, 64, axis=1)


def bf16_round_torch(v):
    import torch
    t = torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).to(torch.float32)
    return t.numpy().astype(np.float64)


def on_grid_matrix(rows, cols, bits, seed):
    """Weights that lie exactly on a quantisation grid: per group pick a bf16 bias z, a
    power-of-two-times-small-integer scale s (exact in bf16 and in the binary32 division
    (max-min)/(2^bits-1)) and codes spanning 0 .. 2^bits-1, so min = z and max = qmax*s + z."""
    rng = np.random.default_rng(seed)
    qmax = (1 << bits) - 1
    groups = cols // 64
    q = rng.integers(0, qmax + 1, size=(rows, cols))
    for r in range(rows):
        for g in range(groups):
            blk = q[r, g * 64:(g + 1) * 64]
            blk[rng.integers(0, 64)] = 0
            j = rng.integers(0, 64)
            while blk[j] == 0 and np.count_nonzero(blk == 0) == 1:
                j = rng.integers(0, 64)
            blk[j] = qmax
    m = rng.integers(1, 8, size=(rows, groups))            # s = m * 2^-e, m < 8: exact in bf16
    e = rng.integers(6, 12, size=(rows, groups))
    s = m.astype(np.float64) * np.exp2(-e.astype(np.float64))
    zi = rng.integers(-128, 128, size=(rows, groups))       # z = k * 2^-7: exact in bf16
    z = zi.astype(np.float64) / 128.0
    w = q * np.repeat(s, 64, axis=1) + np.repeat(z, 64, axis=1)
    assert np.all(w.astype(np.float32).astype(np.float64) == w)  # exactly representable
    return w.astype(np.float32), q, s, z


# ---------------------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------------------
def pin_bytes_pages(o):
    f = facts()
    H, E, L = f["model"]["hidden"], f["model"]["experts"], f["model"]["layers"]
    I = 1024
    q4 = o.expert_bytes(H, I, 4)
    assert q4 == int(f["expert_mb"]["value"] * MiB), q4          # 6.75 MiB exactly
    assert f["model"]["top_k"] * q4 == f["active_mb_per_layer"]["value"] * MiB
    q2 = o.expert_bytes(H, I, 2)
    non = f["disk_gb"]["non_expert_gb"]
    tot4 = L * E * q4 / GiB + non
    tot2 = L * E * q2 / GiB + non
    assert abs(tot4 - f["disk_gb"]["q4"]) / f["disk_gb"]["q4"] < 0.03, tot4
    assert abs(tot2 - f["disk_gb"]["q2"]) / f["disk_gb"]["q2"] < 0.03, tot2
    assert o.qmat_bytes(64, 64, 4) == 64 * 64 // 2 + 64 * 4
    assert o.qmat_bytes(64, 63, 4) == 0 and o.qmat_bytes(64, 64, 3) == 0


def pin_bf16_library(o):
    rng = np.random.default_rng(5)
    v = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(3.0),
        rng.standard_normal(1000).astype(np.float32) * np.float32(1e-30),
        np.array([1.0, 1.00390625, 1.01171875, -1.00390625, 0.0, -0.0, 3.0e38, 1e-45,
                  65504.0, 2.0 ** -126], dtype=np.float32),
        # exact ties between two bf16 neighbours (low 16 bits 0x8000)
        (rng.integers(0x3f000000 >> 16, 0x4f000000 >> 16, 500).astype(np.uint32) << 16 | 0x8000).view(np.float32),
    ])
    ref = bf16_round_torch(v)
    got = np.array([o.bf16_to_f32(o.bf16_rne(float(x))) for x in v], dtype=np.float64)
    assert np.array_equal(np.signbit(ref), np.signbit(got)) and np.array_equal(ref, got)


def pin_quantise_on_grid(o):
    for bits, shape, seed in [(4, (8, 256), 1), (2, (8, 256), 2), (4, (64, 128), 3), (2, (4, 64), 4)]:
        rows, cols = shape
        w, q, s, z = on_grid_matrix(rows, cols, bits, seed)
        qm = o.quantise(w, bits)
        assert len(qm) == o.qmat_bytes(rows, cols, bits)
        for r in range(rows):
            for c in range(cols):
                assert o.code(qm, rows, cols, bits, r, c) == q[r, c], (bits, r, c)
        for r in range(rows):
            for g in range(cols // 64):
                assert o.scale_bias(qm, rows, cols, bits, r, g) == (s[r, g], z[r, g])
        dq = o.dequant(qm, rows, cols, bits)
        assert np.array_equal(dq, w.astype(np.float64))
        # one-hot x picks column j exactly; x = 1 gives the row sums of the known weights
        for j in (0, 1, cols // 2 + 3, cols - 1):
            x = np.zeros(cols)
            x[j] = 1.0
            assert np.array_equal(o.gemv(qm, rows, cols, bits, x), w[:, j].astype(np.float64))
        y = o.gemv(qm, rows, cols, bits, np.ones(cols))
        exact = (q * np.repeat(s, 64, axis=1)).sum(1) + 64 * z.sum(1)
        assert np.allclose(y, exact, rtol=0, atol=1e-12)


def pin_quantise_constant_codes(o):
    """All codes equal c and x = 1: each row equals sum_g 64 * (c * s_g + z_g)."""
    for bits in (4, 2):
        rows, cols = 4, 192
        c = (1 << bits) - 2
        rng = np.random.default_rng(9 + bits)
        s = np.exp2(-rng.integers(4, 9, size=(rows, cols // 64)).astype(np.float64))
        z = rng.integers(-64, 64, size=(rows, cols // 64)) / 64.0
        # pin min and max of each group to the grid ends, the rest at code c
        q = np.full((rows, cols), c)
        q[:, ::64] = 0
        q[:, 1::64] = (1 << bits) - 1
        w = (q * np.repeat(s, 64, 1) + np.repeat(z, 64, 1)).astype(np.float32)
        qm = o.quantise(w, bits)
        y = o.gemv(qm, rows, cols, bits, np.ones(cols))
        want = (q * np.repeat(s, 64, 1)).sum(1) + 64 * z.sum(1)
        assert np.allclose(y, want, rtol=0, atol=1e-12)


def pin_quantise_ties_even(o):
    # group with min 0 and max 2^bits-1: s = 1, z = 0, so w itself is the scaled value
    for bits in (4, 2):
        qmax = (1 << bits) - 1
        base = np.zeros(64, dtype=np.float32)
        base[0], base[1] = 0.0, float(qmax)
        halves = np.arange(qmax, dtype=np.float32) + np.float32(0.5)  # k + 0.5
        w = np.tile(base, (1, 1))
        w[0, 2:2 + len(halves)] = halves
        qm = o.quantise(w, bits)
        assert o.scale_bias(qm, 1, 64, bits, 0, 0) == (1.0, 0.0)
        for i, h in enumerate(halves):
            k = int(math.floor(h))
            want = k if k % 2 == 0 else k + 1  # round half to even
            assert o.code(qm, 1, 64, bits, 0, 2 + i) == want, (bits, h)


def pin_quantise_clamp(o):
    # bf16(min) rounds above min: the min element must clamp to code 0, not wrap
    mn = np.float32(1.0 + 3 * 2.0 ** -9)          # nearest bf16 is 1.0078125 > mn
    w = np.full((1, 64), 2.0, dtype=np.float32)
    w[0, 0] = mn
    w[0, 5] = np.float32(2.5)
    qm = o.quantise(w, 4)
    s, z = o.scale_bias(qm, 1, 64, 4, 0, 0)
    assert z == 1.0078125 and z > float(mn)
    assert o.code(qm, 1, 64, 4, 0, 0) == 0
    assert 0 <= o.code(qm, 1, 64, 4, 0, 5) <= 15


def pin_roundtrip_bound(o):
    rng = np.random.default_rng(11)
    for bits in (4, 2):
        qmax = (1 << bits) - 1
        w = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
        w[3, 64:128] = np.float32(0.25)  # constant group: s = 0, w_hat = bf16(min)
        qm = o.quantise(w, bits)
        dq = o.dequant(qm, 16, 512, bits)
        for r in range(16):
            for g in range(8):
                v = w[r, g * 64:(g + 1) * 64].astype(np.float64)
                s, z = o.scale_bias(qm, 16, 512, bits, r, g)
                mn, mx = v.min(), v.max()
                assert s == bf16_round_torch([np.float32(np.float32(mx - mn) / np.float32(qmax))])[0]
                assert z == bf16_round_torch([np.float32(mn)])[0]
                step = (mx - mn) / qmax
                bound = 0.5 * s + abs(z - mn) + qmax * abs(s - step) + 1e-12
                err = np.abs(dq[r, g * 64:(g + 1) * 64] - v).max()
                assert err <= bound, (bits, r, g, err, bound)
        assert np.all(dq[3, 64:128] == 0.25)


def pin_fma_identity(o):
    """(q*s + z)*x == fma(q, s*x, z*x) == fma(q*x, s, z*x) == s*sum(qx) + z*sum(x)."""
    rng = np.random.default_rng(13)
    for bits in (4, 2):
        for _ in range(50):
            q = rng.integers(0, 1 << bits, 64)
            s = float(rng.uniform(1e-4, 1e-2))
            z = float(rng.uniform(-0.05, 0.05))
            x = rng.standard_normal(64)
            vals = [o.group_dot(f, q, s, z, x) for f in range(4)]
            scale = np.abs((q * s + z) * x).sum()
            for v in vals[1:]:
                assert abs(v - vals[0]) <= 1e-12 * scale, (vals, scale)


def make_tiny_layer(o, H=256, I=128, E=16, K=2, bits=4, seed=0, shared=True, gate=True):
    rng = np.random.default_rng(seed)
    f32 = lambda *s: (rng.standard_normal(s) * 0.02).astype(np.float32)
    experts = [np.concatenate([o.quantise(f32(I, H), bits), o.quantise(f32(I, H), bits),
                               o.quantise(f32(H, I), bits)]) for _ in range(E)]
    sh = np.concatenate([o.quantise(f32(I, H), bits), o.quantise(f32(I, H), bits),
                         o.quantise(f32(H, I), bits)]) if shared else None
    return dict(H=H, I=I, E=E, K=K, bits=bits, experts=experts, shared=sh,
                router=f32(E, H), shared_gate=f32(H) if gate else None)


def np_expert(blob, H, I, bits):
    g = np_dense(blob, I, H, bits)
    qb = (I * H * bits // 8) + I * H // 16
    up = np_dense(blob[qb:2 * qb], I, H, bits)
    dn = np_dense(blob[2 * qb:], H, I, bits)

    def f(x):
        a = g @ x
        u = up @ x
        h = a / (1.0 + np.exp(-a)) * u
        return dn @ h
    return f


def brute_force_layer(ly, x, res, bias=None):
    """Dense numpy evaluation: every expert evaluated, all logits sorted."""
    H, I, E, K, bits = ly["H"], ly["I"], ly["E"], ly["K"], ly["bits"]
    R = ly["router"].astype(np.float64)
    logits = R @ x + (0.0 if bias is None else bias.astype(np.float64))
    p = np.exp(logits - logits.max())
    p /= p.sum()
    order = np.lexsort((np.arange(E), -logits))       # logit desc, index asc
    sel = order[:K]
    w = p[sel] / p[sel].sum()
    ys = [np_expert(b, H, I, bits)(x) for b in ly["experts"]]   # all experts, densely
    out = (res.copy() if res is not None else np.zeros(H))
    for k in range(K):
        out = out + w[k] * ys[sel[k]]
    if ly["shared"] is not None:
        gsig = 1.0
        if ly["shared_gate"] is not None:
            gsig = 1.0 / (1.0 + np.exp(-(ly["shared_gate"].astype(np.float64) @ x)))
        out = out + gsig * np_expert(ly["shared"], H, I, bits)(x)
    return out, sel, w


def pin_brute_force_tiny(o):
    for bits, shared, gate, seed in [(4, True, True, 0), (2, True, True, 1), (4, False, False, 2),
                                     (4, True, False, 3)]:
        ly = make_tiny_layer(o, bits=bits, shared=shared, gate=gate, seed=seed)
        rng = np.random.default_rng(100 + seed)
        for t in range(3):
            x = rng.standard_normal(ly["H"]).astype(np.float32).astype(np.float64)
            res = rng.standard_normal(ly["H"]).astype(np.float32).astype(np.float64)
            want, sel, w = brute_force_layer(ly, x, res)
            got, idx, gw = o.layer(ly, x, res)
            assert list(idx) == list(sel), (idx, sel)
            assert np.allclose(gw, w, rtol=1e-12, atol=0)
            assert np.allclose(got, want, rtol=1e-11, atol=1e-12), np.abs(got - want).max()
        # the expert alone, and one GEMV, against the dense matrices
        blob = ly["experts"][3]
        y = o.expert(blob, ly["H"], ly["I"], bits, x)
        assert np.allclose(y, np_expert(blob, ly["H"], ly["I"], bits)(x), rtol=1e-11, atol=1e-13)


def pin_routing_invariants(o):
    rng = np.random.default_rng(17)
    H, E = 64, 12
    for K in (1, 3, E):
        router = (rng.standard_normal((E, H)) * 0.3).astype(np.float32)
        x = rng.standard_normal(H)
        idx, w, logits, p = o.route(x, router, None, K)
        assert abs(w.sum() - 1.0) <= 1e-12 and np.all(w > 0)
        assert len(set(idx.tolist())) == K
    # K = E is the full softmax; logits chosen exactly through a one-hot x
    lv = np.array([0.5, -1.25, 2.0, 0.0, 3.5, -0.75, 1.0, 2.0, -3.0, 0.25, 1.5, -2.5], dtype=np.float32)
    router = np.zeros((E, H), dtype=np.float32)
    router[:, 7] = lv
    x = np.zeros(H)
    x[7] = 1.0
    idx, w, logits, p = o.route(x, router, None, E)
    sm = np.exp(lv.astype(np.float64) - lv.max())
    sm /= sm.sum()
    assert np.allclose(w, sm[idx], rtol=1e-14, atol=0)
    assert np.array_equal(logits, lv.astype(np.float64))
    # the two equal logits (2.0 at 2 and 7) come out lower index first
    assert list(idx[:3]) == [4, 2, 7]
    # a bias is added before the softmax
    bias = np.zeros(E, dtype=np.float32)
    bias[8] = 10.0
    idx, w, logits, p = o.route(x, router, bias, 2)
    assert idx[0] == 8 and logits[8] == 7.0


def pin_ties_lower_index(o):
    H, E = 64, 9
    router = np.zeros((E, H), dtype=np.float32)
    for K in (1, 4, 9):
        idx, w, _, _ = o.route(np.ones(H), router, None, K)
        assert list(idx) == list(range(K)) and np.allclose(w, 1.0 / K, rtol=1e-15, atol=0)


def pin_zero_input(o):
    for bits in (4, 2):
        ly = make_tiny_layer(o, bits=bits, seed=21 + bits)
        res = np.random.default_rng(3).standard_normal(ly["H"])
        out, idx, w = o.layer(ly, np.zeros(ly["H"]), res)
        assert np.array_equal(out, res)
        assert list(idx) == list(range(ly["K"]))


def pin_rmsnorm(o):
    rng = np.random.default_rng(23)
    h = rng.standard_normal(256) * 3.0
    ms = float(np.mean(h * h))
    for eps in (1e-6, 0.5, 4.0):
        x = o.rmsnorm(h, eps)
        assert abs(np.mean(x * x) - ms / (ms + eps)) <= 1e-12
        assert np.allclose(x / h, x[0] / h[0], rtol=1e-13, atol=0)  # one common factor
    assert np.allclose(o.rmsnorm(h * 7.0, 0.0), o.rmsnorm(h, 0.0), rtol=1e-13, atol=0)


def pin_stack_composition(o):
    """Layer 0 takes h_in as it is; layer l >= 1 takes rmsnorm(h_l); residual is h_l."""
    lys = [make_tiny_layer(o, seed=31 + l) for l in range(3)]
    h0 = np.random.default_rng(5).standard_normal(256) * 2.5     # rms far from 1
    eps = 1e-6
    out1, idx1 = o.stack(lys[:1], h0, None, eps)
    want1, sel1, _ = brute_force_layer(lys[0], h0, h0)
    assert np.allclose(out1, want1, rtol=1e-11, atol=1e-12) and list(idx1[0]) == list(sel1)
    out3, idx3, xt = o.stack(lys, h0, None, eps, want_trace=True)
    h = h0
    for l in range(3):
        x = h if l == 0 else h / math.sqrt(np.mean(h * h) + eps)
        assert np.allclose(xt[l], x, rtol=1e-13, atol=1e-15)
        h, sel, _ = brute_force_layer(lys[l], x, h)
        assert list(idx3[l]) == list(sel)
    assert np.allclose(out3, h, rtol=1e-11, atol=1e-12)


ALL_PINS = [pin_bytes_pages, pin_bf16_library, pin_quantise_on_grid, pin_quantise_constant_codes,
            pin_quantise_ties_even, pin_quantise_clamp, pin_roundtrip_bound, pin_fma_identity,
            pin_brute_force_tiny, pin_routing_invariants, pin_ties_lower_index, pin_zero_input,
            pin_rmsnorm, pin_stack_composition]
