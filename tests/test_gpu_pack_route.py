"""GPU: input generator, pack kernel and router against the oracle."""
import numpy as np
import pytest
import torch

import synth
import oracle_pins as P
from gpu_helpers import check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    import bit_dequant_expert_gemv_b200 as f
    f.build()
    return f


def test_device_generator_matches_host():
    for st, off, n, sigma in [(synth.stream_id(1, 0, 3, 2), 0, 1 << 20, 0.02),
                              (synth.stream_id(5), 4096 * 17, 4096 * 3, 1.0),
                              (synth.stream_id(3, 59, 0, 0), 123, 999, 0.02)]:
        d = torch.empty(n, dtype=torch.float32, device="cuda")
        synth.normal_dev(d, 7, st, offset=off, sigma=sigma)
        h = synth.normal_host(n, 7, st, offset=off, sigma=sigma)
        assert np.array_equal(d.cpu().numpy().view(np.uint32), h.view(np.uint32))


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("shape", [(64, 64), (128, 256), (256, 128), (192, 320), (64, 4096)])
def test_pack_bit_exact(fmoe, orc, bits, shape):
    w = synth.normal_host(shape[0] * shape[1], 3, synth.stream_id(1, 0, shape[0], shape[1]),
                          sigma=0.02).reshape(shape)
    got = fmoe.pack(torch.from_numpy(w).cuda(), bits).cpu().numpy()
    assert np.array_equal(got, orc.quantise(w, bits))


@pytest.mark.parametrize("bits", [4, 2])
def test_pack_special_groups(fmoe, orc, bits):
    # on-grid groups, half-way ties, a constant group and a group whose bf16(min) > min
    w, _, _, _ = P.on_grid_matrix(64, 256, bits, seed=bits)
    qmax = (1 << bits) - 1
    w[0, :64] = 0.0
    w[0, 1] = qmax
    w[0, 2:2 + qmax] = np.arange(qmax) + 0.5
    w[1, 64:128] = 0.25
    w[2, :64] = 2.0
    w[2, 0] = np.float32(1.0 + 3 * 2.0 ** -9)
    w = np.ascontiguousarray(w, dtype=np.float32)
    got = fmoe.pack(torch.from_numpy(w).cuda(), bits).cpu().numpy()
    assert np.array_equal(got, orc.quantise(w, bits))


@pytest.mark.parametrize("bits", [4, 2])
def test_pack_full_expert_matrices(fmoe, orc, bits):
    wl = synth.WORKLOADS["full_q4"]
    for m in (synth.MAT_GATE, synth.MAT_DOWN):
        w = synth.matrix_host(wl, 0, 5, m)
        got = fmoe.pack(torch.from_numpy(w).cuda(), bits).cpu().numpy()
        assert np.array_equal(got, orc.quantise(w, bits)), m


@pytest.mark.parametrize("name", ["tiny", "full_q4"])
def test_route_natural(fmoe, orc, name):
    wl = synth.WORKLOADS[name]
    router = synth.router_host(wl, 0)
    rd = torch.from_numpy(router).cuda()
    xs = synth.token_inputs(wl, 0, 6)
    for t in range(6):
        x = xs[t]
        idx, w = fmoe.route(torch.from_numpy(x).cuda(), rd, None, wl.K)
        _, _, logits, _ = orc.route(x, router, None, wl.K)
        check_routing(idx.cpu().numpy(), w.cpu().numpy(), logits, wl.K)


def test_route_bias_forces_selection(fmoe, orc):
    wl = synth.WORKLOADS["full_q4"]
    router = synth.router_host(wl, 0)
    bias = synth.logit_bias(wl, tokens=4)[:, 0]
    forced = synth.forced_experts(wl, tokens=4)[:, 0]
    xs = synth.token_inputs(wl, 0, 4)
    for t in range(4):
        b = torch.from_numpy(bias[t]).cuda()
        idx, w = fmoe.route(torch.from_numpy(xs[t]).cuda(), torch.from_numpy(router).cuda(), b, wl.K)
        assert set(idx.cpu().tolist()) == set(forced[t].tolist())
        _, _, logits, _ = orc.route(xs[t], router, bias[t], wl.K)
        check_routing(idx.cpu().numpy(), w.cpu().numpy(), logits, wl.K)


def test_route_ties_and_full_softmax(fmoe, orc):
    H, E = 128, 8
    router = torch.zeros(E, H, device="cuda")
    x = torch.ones(H, device="cuda")
    for K in (1, 3, 8):
        idx, w = fmoe.route(x, router, None, K)
        assert idx.cpu().tolist() == list(range(K))
        assert np.allclose(w.cpu().numpy(), 1.0 / K, rtol=0, atol=1e-7)
    lv = np.array([0.5, -1.25, 2.0, 0.0, 3.5, -0.75, 1.0, 2.0], dtype=np.float32)
    r = np.zeros((E, H), dtype=np.float32)
    r[:, 7] = lv
    xh = np.zeros(H, dtype=np.float32)
    xh[7] = 1.0
    idx, w = fmoe.route(torch.from_numpy(xh).cuda(), torch.from_numpy(r).cuda(), None, E)
    assert idx.cpu().tolist()[:3] == [4, 2, 7]
    sm = np.exp(lv.astype(np.float64) - lv.max())
    sm /= sm.sum()
    assert np.abs(w.cpu().numpy() - sm[idx.cpu().numpy()]).max() <= 1e-6
