"""GPU: the top-K decision at the edge of the 1e-6 tie band, at large logit magnitudes.

The K-th and (K+1)-th logits are placed at about 20 and about 64 (through the logit bias)
and separated by 0.5e-6 (inside the band: either order is correct), 1.5e-6 and 3e-6 (outside:
the selection must be the oracle's exactly). The router is one-hot on column 7, so the
logits are l_e = router[e, 7] * x[7] + bias[e] with x[7] = 1, exact in binary64 on both sides;
the (K+1)-th expert has the LOWER index, so a kernel that merged the two logits (for instance
by ranking on binary32-rounded values, whose spacing is 1.9e-6 at 20 and 7.6e-6 at 64) would
pick it by the lower-index tie rule and fail. Both top-K paths are covered (<= 512 experts
and > 512 experts), through fmoe_route and through fmoe_moe_layer."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle.workload import HostLayer
from gpu_helpers import TIE, check_out, check_routing, renorm_weights

pytestmark = pytest.mark.gpu

COL = 7


@pytest.fixture(scope="module")
def fmoe():
    import bit_dequant_expert_gemv_b200 as f
    f.build()
    return f


def band_case(E, K, H, M, gap):
    """(router [E, H] fp32, bias [E] fp32, p, q): experts 1..K-1 sit at M + 5, expert p at
    M + gap, expert q < p at M, every other expert at 0."""
    router = np.zeros((E, H), dtype=np.float32)
    bias = np.zeros(E, dtype=np.float32)
    top = list(range(1, K))
    q, p = K + 1, E - 3            # q has the lower index
    bias[top] = np.float32(M + 5.0)
    bias[p] = np.float32(M)
    bias[q] = np.float32(M)
    router[p, COL] = np.float32(gap)
    return router, bias, p, q


CASES = [(E, K, H, M, gap) for (E, K, H) in [(16, 3, 256), (600, 4, 128)]
         for M in (20.0, 64.0) for gap in (0.5e-6, 1.5e-6, 3e-6)]


def _x(H, seed):
    x = synth.normal_host(H, 11, synth.stream_id(synth.KIND_X), offset=seed * H, sigma=1.0)
    x[COL] = 1.0
    return x


@pytest.mark.parametrize("E,K,H,M,gap", CASES)
def test_route_tie_band(fmoe, orc, E, K, H, M, gap):
    router, bias, p, q = band_case(E, K, H, M, gap)
    x = _x(H, 0)
    idx, w = fmoe.route(torch.from_numpy(x).cuda(), torch.from_numpy(router).cuda(),
                        torch.from_numpy(bias).cuda(), K)
    _, _, logits, _ = orc.route(x, router, bias, K)
    d = logits[p] - logits[q]
    assert abs(d - np.float64(np.float32(gap))) < 1e-12  # the band geometry is what we built
    exact = check_routing(idx.cpu().numpy(), w.cpu().numpy(), logits, K)
    if gap >= TIE:
        assert exact and p in idx.cpu().tolist() and q not in idx.cpu().tolist()


@pytest.mark.parametrize("E,K,H,M,gap", CASES)
def test_layer_tie_band(fmoe, orc, E, K, H, M, gap):
    from bit_dequant_expert_gemv_b200.workload import build_layer
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], H=H, E=E, K=K)
    dl = build_layer(wl, 0)
    router, bias, p, q = band_case(E, K, H, M, gap)
    rd = torch.from_numpy(router).cuda()
    desc = fmoe.LayerDesc(wl.H, wl.I, wl.E, wl.K, wl.bits, dl.experts, dl.stride, dl.shared, rd,
                          dl.gate)
    x = _x(H, 1)
    res = synth.token_inputs(wl, 0, 1, kind=synth.KIND_RES)[0]
    idx = torch.empty(K, dtype=torch.int32, device="cuda")
    w = torch.empty(K, dtype=torch.float32, device="cuda")
    out = fmoe.moe_layer(desc, torch.from_numpy(x).cuda(), torch.from_numpy(res).cuda(),
                         torch.from_numpy(bias).cuda(), idx=idx, weight=w)
    assert fmoe.sync_status() == 0
    hl = HostLayer(orc, wl, 0)
    hl.router = router
    oi, ow, logits, _ = orc.route(x, router, bias, K)
    gi = idx.cpu().numpy()
    exact = check_routing(gi, w.cpu().numpy(), logits, K)
    if gap >= TIE:
        assert exact
        want = hl.forced(x, res, oi, ow)
    else:
        want = hl.forced(x, res, gi, renorm_weights(logits, gi))
    check_out(out.cpu().numpy(), want, f"layer E={E} M={M} gap={gap}")
