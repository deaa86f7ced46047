"""GPU: the status-code contract, and the bounded-wait timeout path made on the host."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    import bit_dequant_expert_gemv_b200 as f
    f.build()
    return f


def test_validation_errors_launch_nothing(fmoe):
    from bit_dequant_expert_gemv_b200.workload import build_layer
    wl = synth.WORKLOADS["tiny"]
    dl = build_layer(wl, 0)
    x = torch.randn(wl.H, device="cuda")
    n0 = fmoe.launch_count()
    bad = fmoe.LayerDesc(wl.H, wl.I, wl.E, wl.K, 3, dl.experts, dl.stride, dl.shared, dl.router, dl.gate)
    with pytest.raises(fmoe.FmoeError) as e:
        fmoe.moe_layer(bad, x)
    assert e.value.code == fmoe.FMOE_ERR_INVALID
    bad = fmoe.LayerDesc(wl.H, wl.I, wl.E, wl.E + 1, 4, dl.experts, dl.stride, dl.shared, dl.router, dl.gate)
    with pytest.raises(fmoe.FmoeError) as e:
        fmoe.moe_layer(bad, x)
    assert e.value.code == fmoe.FMOE_ERR_INVALID
    xs = torch.empty(wl.H + 1, device="cuda")[1:]
    with pytest.raises(fmoe.FmoeError) as e:
        fmoe.moe_layer(dl.desc, xs)
    assert e.value.code == fmoe.FMOE_ERR_ALIGN
    with pytest.raises(fmoe.FmoeError) as e:
        fmoe.pack(torch.empty(64, 96, device="cuda"), 4)
    assert e.value.code == fmoe.FMOE_ERR_INVALID
    assert fmoe.launch_count() == n0


def test_timeout_path_reports_and_recovers(fmoe):
    """The routing decision is withheld (host-set test flag), so the waits that depend on it
    run out of a short budget; the kernel must return, the status must say TIMEOUT, and the
    next normal call must work."""
    from bit_dequant_expert_gemv_b200.workload import build_layer
    wl = synth.WORKLOADS["tiny"]
    dl = build_layer(wl, 0)
    x = torch.from_numpy(synth.token_inputs(wl, 0, 1)[0]).cuda()
    ref = fmoe.moe_layer(dl.desc, x, x)
    assert fmoe.sync_status() == 0
    fmoe.set_wait_budget_ns(2_000_000)
    fmoe.set_fault_injection(1)
    try:
        fmoe.moe_layer(dl.desc, x, x)
        assert fmoe.sync_status() == fmoe.FMOE_ERR_TIMEOUT
        assert "budget" in fmoe.last_error()
    finally:
        fmoe.set_fault_injection(0)
        fmoe.set_wait_budget_ns(1_000_000_000)
    again = fmoe.moe_layer(dl.desc, x, x)
    assert fmoe.sync_status() == 0
    assert torch.equal(again, ref)
