"""GPU: multi-layer decode stacks (RMSNorm between layers) against the oracle."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle.workload import HostLayer
from gpu_helpers import ABS_TOL, REL_L2, check_out, check_routing, renorm_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    import bit_dequant_expert_gemv_b200 as f
    f.build()
    return f


def build_stack(wl):
    from bit_dequant_expert_gemv_b200.workload import build_layer
    return [build_layer(wl, l) for l in range(wl.layers)]


def run_stack(fmoe, wl, dls, T, bias=None, scale=1.0):
    L = wl.layers
    h_in = torch.from_numpy(synth.token_inputs(wl, 0, T) * np.float32(scale)).cuda()
    idx = torch.empty(T, L, wl.K, dtype=torch.int32, device="cuda")
    ht = torch.empty(T, L, wl.H, dtype=torch.float32, device="cuda")
    b = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias[:T])).cuda()
    h_out = fmoe.moe_stack([d.desc for d in dls], h_in, b, wl.eps, idx_trace=idx, h_trace=ht)
    assert fmoe.sync_status() == 0
    return h_in.cpu().numpy(), idx.cpu().numpy(), ht.cpu().numpy(), h_out.cpu().numpy()


def teacher_force(orc, wl, hls, pairs, h_in, idx, ht, h_out, bias=None):
    """Layer l of token t recomputed by the oracle from the GPU's recorded input h_l."""
    L = wl.layers
    for t, l in pairs:
        hl = hls.setdefault(l, HostLayer(orc, wl, l))
        h = ht[t, l].astype(np.float64)
        if l == 0:
            assert np.array_equal(ht[t, 0], h_in[t])
        x = h if l == 0 else orc.rmsnorm(h, wl.eps)
        bb = None if bias is None else bias[t, l]
        oi, ow, logits, _ = orc.route(x, hl.router, bb, wl.K)
        if check_routing(idx[t, l], None, logits, wl.K):
            want = hl.forced(x, h, oi, ow)
        else:
            want = hl.forced(x, h, idx[t, l], renorm_weights(logits, idx[t, l]))
        nxt = h_out[t] if l == L - 1 else ht[t, l + 1]
        check_out(nxt, want, f"{wl.name} token {t} layer {l}")


def test_stack_tiny_end_to_end(fmoe, orc):
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], layers=3, tokens=4)
    dls = build_stack(wl)
    h_in, idx, ht, h_out = run_stack(fmoe, wl, dls, wl.tokens, scale=2.0)
    hls = [HostLayer(orc, wl, l) for l in range(wl.layers)]
    for t in range(wl.tokens):
        layers = [hl.as_dict(range(wl.E)) for hl in hls]
        want, widx = orc.stack(layers, h_in[t], None, wl.eps)
        assert np.array_equal(idx[t], widx)
        check_out(h_out[t], want, f"stack token {t}")
    teacher_force(orc, wl, dict(enumerate(hls)), [(t, l) for t in range(4) for l in range(3)],
                  h_in, idx, ht, h_out)


def test_stack_graph_matches_direct(fmoe):
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], layers=4, tokens=5)
    dls = build_stack(wl)
    h_in = torch.from_numpy(synth.token_inputs(wl, 0, wl.tokens)).cuda()
    ref = fmoe.moe_stack([d.desc for d in dls], h_in, None, wl.eps)
    for tpl in (0, 1, 2):
        h2 = torch.empty_like(ref)
        g = fmoe.StackGraph([d.desc for d in dls], h_in, h2, eps=wl.eps, tokens_per_launch=tpl)
        g.launch()
        g.launch()
        assert fmoe.sync_status() == 0
        check_out(h2.cpu().numpy(), ref.cpu().numpy(), f"graph tokens_per_launch={tpl}")
        g.close()


@pytest.mark.parametrize("name", ["stack_q4_skewed", "stack_q4_uniform", "stack_q2"])
def test_stack_full_size(fmoe, orc, name):
    wl = synth.WORKLOADS[name]
    free, _ = torch.cuda.mem_get_info()
    need = wl.layers * (wl.E + 1) * fmoe.expert_bytes(wl.H, wl.I, wl.bits) * 1.02 + 4e9
    if need > free:
        pytest.skip(f"needs {need / 1e9:.1f} GB, {free / 1e9:.1f} GB free")
    dls = build_stack(wl)
    T = 3
    bias = synth.logit_bias(wl, tokens=T)
    h_in, idx, ht, h_out = run_stack(fmoe, wl, dls, T, bias=bias)
    assert np.isfinite(h_out).all()
    if bias is not None:
        forced = synth.forced_experts(wl, tokens=T)
        for t in range(T):
            for l in range(wl.layers):
                assert set(idx[t, l].tolist()) == set(forced[t, l].tolist())
    L = wl.layers
    pairs = [(0, 0), (0, 1), (1, L // 2), (2, L - 1)]
    hls = {}
    teacher_force(orc, wl, hls, pairs, h_in, idx, ht, h_out, bias=bias)
    if name != "stack_q4_skewed":
        end_to_end(orc, wl, hls, 0, h_in, idx, h_out, bias=bias)
    del dls
    torch.cuda.empty_cache()


def end_to_end(orc, wl, hls, t, h_in, idx, h_out, bias=None):
    """Token t through every layer by the oracle alone, from the same input: the oracle's own
    chain of h, not the GPU's recorded layer inputs. The selection is the oracle's wherever it
    is unambiguous; inside the tie band the chain takes the GPU's (both are correct there),
    so that the two chains stay comparable. The per-layer bounds hold for one layer; over a
    chain each layer adds its own rounding error to the residual stream, and independent
    errors grow like the square root of the depth: the end-to-end output is held to the same
    relative-L2 bound (1e-3) and to max-abs <= 2e-3 * sqrt(L). Its error is reported."""
    L = wl.layers
    h = h_in[t].astype(np.float64)
    for l in range(L):
        hl = hls.setdefault(l, HostLayer(orc, wl, l))
        x = h if l == 0 else orc.rmsnorm(h, wl.eps)
        bb = None if bias is None else bias[t, l]
        oi, ow, logits, _ = orc.route(x, hl.router, bb, wl.K)
        if check_routing(idx[t, l], None, logits, wl.K):
            h = hl.forced(x, h, oi, ow)
        else:
            h = hl.forced(x, h, idx[t, l], renorm_weights(logits, idx[t, l]))
    got, want = h_out[t].astype(np.float64), h
    err = np.abs(got - want).max()
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    print(f"{wl.name} token {t}, {L} layers end to end: max-abs {err:.3e}, rel-L2 {rel:.3e}")
    assert err <= ABS_TOL * np.sqrt(L) and rel <= REL_L2, (wl.name, t, err, rel)
