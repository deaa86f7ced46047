"""GPU: one expert, one MoE layer and token sequences against the oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle.workload import HostLayer, expert_blob
from gpu_helpers import check_out, check_routing, renorm_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    import bit_dequant_expert_gemv_b200 as f
    f.build()
    return f


def wl_variant(name, **kw):
    import dataclasses
    return dataclasses.replace(synth.WORKLOADS[name], **kw)


@pytest.mark.parametrize("shape", [(256, 128, 4), (256, 128, 2), (4096, 1024, 4), (4096, 1024, 2),
                                   (192, 320, 4), (64, 64, 2)])
def test_expert_gemv(fmoe, orc, shape):
    from bit_dequant_expert_gemv_b200.workload import _fill_expert
    H, I, bits = shape
    wl = wl_variant("tiny", H=H, I=I, bits=bits, E=1, K=1)
    blob = torch.empty(fmoe.expert_bytes(H, I, bits), dtype=torch.uint8, device="cuda")
    tmp = torch.empty(H * I, dtype=torch.float32, device="cuda")
    _fill_expert(wl, 0, 0, blob, tmp, shared=False)
    host_blob = expert_blob(orc, wl, 0, 0)
    assert np.array_equal(blob.cpu().numpy(), host_blob)  # pack parity on a whole expert
    xs = synth.token_inputs(wl, 0, 3)
    for t in range(3):
        y = fmoe.expert_gemv(blob, H, I, bits, torch.from_numpy(xs[t]).cuda())
        check_out(y.cpu().numpy(), orc.expert(host_blob, H, I, bits, xs[t]), f"expert {shape}")


def run_seq(fmoe, wl, T, shared=True, gate=True, bias=None, replicas=1, t0=0):
    from bit_dequant_expert_gemv_b200.workload import build_layer, token_inputs_dev
    dl = build_layer(wl, 0, shared=shared, gate=gate)
    descs = [dl.desc]
    keep = []
    for r in range(1, replicas):   # copies of the data-independent tensors, shared experts
        router = dl.router.clone()
        g = None if dl.gate is None else dl.gate.clone()
        sh = None if dl.shared is None else dl.shared.clone()
        keep += [router, g, sh]
        descs.append(fmoe.LayerDesc(wl.H, wl.I, wl.E, wl.K, wl.bits, dl.experts, dl.stride, sh, router, g))
    x = token_inputs_dev(wl, t0, T)
    res = token_inputs_dev(wl, t0, T, kind=synth.KIND_RES)
    idx = torch.empty(T, wl.K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.K, dtype=torch.float32, device="cuda")
    b = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias)).cuda()
    out = fmoe.moe_layer_seq(descs, x, res, b, idx=idx, weight=w)
    assert fmoe.sync_status() == 0
    return out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(), x.cpu().numpy(), res.cpu().numpy()


def check_tokens(orc, wl, tokens, out, idx, w, x, res, bias=None, shared=True, gate=True):
    hl = HostLayer(orc, wl, 0, shared=shared, gate=gate)
    for t in tokens:
        b = None if bias is None else bias[t]
        oi, ow = orc.route(x[t], hl.router, b, wl.K)[:2]
        logits = orc.route(x[t], hl.router, b, wl.K)[2]
        exact = check_routing(idx[t], w[t], logits, wl.K)
        if exact:
            want = hl.forced(x[t], res[t], oi, ow)
        else:   # tie band: the oracle combine with the GPU's selection
            want = hl.forced(x[t], res[t], idx[t], renorm_weights(logits, idx[t]))
        check_out(out[t], want, f"{wl.name} token {t}")


@pytest.mark.parametrize("bits", [4, 2])
def test_layer_tiny(fmoe, orc, bits):
    wl = wl_variant("tiny", bits=bits)
    out, idx, w, x, res = run_seq(fmoe, wl, 8)
    check_tokens(orc, wl, range(8), out, idx, w, x, res)


@pytest.mark.parametrize("shared,gate", [(False, False), (True, False)])
def test_layer_tiny_without_shared_or_gate(fmoe, orc, shared, gate):
    wl = wl_variant("tiny", shared=shared)
    out, idx, w, x, res = run_seq(fmoe, wl, 4, shared=shared, gate=gate)
    check_tokens(orc, wl, range(4), out, idx, w, x, res, shared=shared, gate=gate)


@pytest.mark.parametrize("shape", [(192, 320, 7, 3, 4), (64, 64, 1, 1, 2), (128, 64, 40, 8, 4),
                                   (1024, 576, 33, 5, 2),
                                   # more than 512 experts: the top-K keeps 16 keys per lane
                                   # across passes of 512 (a merge per pass)
                                   (128, 64, 1100, 8, 4), (256, 128, 513, 2, 2)])
def test_layer_odd_shapes(fmoe, orc, shape):
    H, I, E, K, bits = shape
    wl = wl_variant("tiny", H=H, I=I, E=E, K=K, bits=bits)
    out, idx, w, x, res = run_seq(fmoe, wl, 3)
    check_tokens(orc, wl, range(3), out, idx, w, x, res)


def test_layer_zero_input_gives_residual(fmoe):
    from bit_dequant_expert_gemv_b200.workload import build_layer
    for bits in (4, 2):
        wl = wl_variant("tiny", bits=bits)
        dl = build_layer(wl, 0)
        x = torch.zeros(wl.H, device="cuda")
        res = torch.randn(wl.H, device="cuda")
        idx = torch.empty(wl.K, dtype=torch.int32, device="cuda")
        out = fmoe.moe_layer(dl.desc, x, res, idx=idx)
        assert torch.equal(out, res)
        assert idx.cpu().tolist() == list(range(wl.K))


def test_layer_residual_may_alias_out(fmoe, orc):
    from bit_dequant_expert_gemv_b200.workload import build_layer
    wl = synth.WORKLOADS["tiny"]
    dl = build_layer(wl, 0)
    x = torch.from_numpy(synth.token_inputs(wl, 0, 1)[0]).cuda()
    res = torch.from_numpy(synth.token_inputs(wl, 0, 1, kind=synth.KIND_RES)[0]).cuda()
    ref = fmoe.moe_layer(dl.desc, x, res.clone())
    inplace = res.clone()
    fmoe.moe_layer(dl.desc, x, inplace, out=inplace)
    assert torch.equal(ref, inplace)


def test_layer_full_q4_natural(fmoe, orc):
    wl = synth.WORKLOADS["full_q4_natural"]
    out, idx, w, x, res = run_seq(fmoe, wl, 6)
    check_tokens(orc, wl, [0, 3, 5], out, idx, w, x, res)


def test_layer_full_q4_forced_bench_launch(fmoe, orc):
    """The benchmark's launch: 1000 tokens in one launch, forced-uniform routing, 4 replicas of
    the router / shared expert; sampled tokens checked against the oracle."""
    wl = synth.WORKLOADS["full_q4"]
    T = wl.tokens
    bias = synth.logit_bias(wl, tokens=T)[:, 0]
    out, idx, w, x, res = run_seq(fmoe, wl, T, bias=bias, replicas=4)
    forced = synth.forced_experts(wl, tokens=T)[:, 0]
    assert all(set(idx[t].tolist()) == set(forced[t].tolist()) for t in range(T))
    check_tokens(orc, wl, sample_tokens(T, 32, seed=5), out, idx, w, x, res, bias=bias)
    assert np.isfinite(out).all()


def sample_tokens(T, n, seed):
    """The first and last token and n - 2 others drawn without replacement (seeded)."""
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, T - 1), size=n - 2, replace=False)
    return [0, *sorted(int(t) for t in mid), T - 1]


def test_layer_full_q2(fmoe, orc):
    """The 2-bit layer's whole token sequence (1000 tokens, natural routing) in one launch;
    32 sampled tokens against the oracle."""
    wl = synth.WORKLOADS["full_q2"]
    T = wl.tokens
    out, idx, w, x, res = run_seq(fmoe, wl, T)
    check_tokens(orc, wl, sample_tokens(T, 32, seed=6), out, idx, w, x, res)
    assert np.isfinite(out).all()
