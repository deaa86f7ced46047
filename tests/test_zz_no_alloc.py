"""GPU: fmoe_moe_layer_noalloc (one token, scratch in the library's fixed device array)
against fmoe_moe_layer (pool scratch), called twice in a row through the C ABI.

Collected last on purpose (file name), so it runs both after every other GPU test in the
same process and alone (``pytest tests/test_zz_no_alloc.py``)."""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import check_out, W_TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fmoe():
    import bit_dequant_expert_gemv_b200 as f
    f.build()
    return f


def _layer_inputs(fmoe, name, t):
    from bit_dequant_expert_gemv_b200.workload import build_layer, token_inputs_dev
    wl = synth.WORKLOADS[name]
    dl = build_layer(wl, 0)
    x = token_inputs_dev(wl, t, 1)[0]
    res = token_inputs_dev(wl, t, 1, kind=synth.KIND_RES)[0]
    return wl, dl, x, res


@pytest.mark.parametrize("name", ["tiny", "full_q4_natural", "full_q2"])
def test_noalloc_matches_layer(fmoe, orc, name):
    from oracle.workload import HostLayer
    from gpu_helpers import check_routing
    wl, dl, x, res = _layer_inputs(fmoe, name, 3)
    K = wl.K
    idx_ref = torch.empty(K, dtype=torch.int32, device="cuda")
    w_ref = torch.empty(K, dtype=torch.float32, device="cuda")
    ref = fmoe.moe_layer(dl.desc, x, res, None, idx=idx_ref, weight=w_ref)
    assert fmoe.sync_status() == 0
    outs = [torch.full_like(x, float("nan")) for _ in range(3)]
    idxs = [torch.full((K,), -1, dtype=torch.int32, device="cuda") for _ in range(3)]
    ws = [torch.full((K,), float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
    free_before = None
    for call in range(3):  # calls in a row reuse the same fixed scratch
        fmoe.moe_layer_noalloc(dl.desc, x, res, None, out=outs[call], idx=idxs[call],
                               weight=ws[call])
        assert fmoe.sync_status() == 0, fmoe.last_error()
        if call == 0:  # the first call on the device did the set-up; later calls allocate nothing
            free_before = torch.cuda.mem_get_info()[0]
    assert torch.cuda.mem_get_info()[0] == free_before
    # the oracle, for the same token
    hl = HostLayer(orc, wl, 0)
    xh, rh = x.cpu().numpy(), res.cpu().numpy()
    want, oi, ow, logits = hl.forward(xh, rh)
    for call in range(3):
        out, idx, w = outs[call].cpu().numpy(), idxs[call].cpu().numpy(), ws[call].cpu().numpy()
        check_out(out, ref.cpu().numpy(), f"{name} call {call} vs fmoe_moe_layer")
        assert idx.tolist() == idx_ref.cpu().tolist()
        assert np.abs(w - w_ref.cpu().numpy()).max() <= W_TOL
        assert check_routing(idx, w, logits, K)
        check_out(out, want, f"{name} call {call} vs oracle")


def test_noalloc_rejects_oversized_scratch(fmoe):
    # 4096 experts with top_k = 8 and I = 1024 need more scratch than the fixed array holds.
    # Validation happens on the host before anything is enqueued, so these small buffers are
    # never read.
    H, I, E, K, bits = 1024, 1024, 4096, 8, 4
    buf = torch.zeros(1024, dtype=torch.float32, device="cuda")
    stride = fmoe.expert_bytes(H, I, bits)
    d = fmoe.LayerDesc(H, I, E, K, bits, buf, stride, None, buf, None)
    before = fmoe.launch_count()
    with pytest.raises(fmoe.FmoeError, match="fixed area"):
        fmoe.moe_layer_noalloc(d, buf, None, None, out=torch.empty_like(buf))
    assert fmoe.launch_count() == before
