"""Expert parallelism on one GPU: the ranks' shares (moe_layer_forward_partial
over each rank's expert range, the shared expert on rank 0) are computed one
after the other on the same device and summed on the host -- what the
all-reduce of an expert-parallel group adds up -- and compared with the
layer forward and with the oracle.  Covers the fused small-batch path (T <=
4), the multi-kernel path and the batched tensor-core path (T >= 64), and
the adaptive top-p.  No rank waits for another: nothing here needs several
GPUs."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity_helpers import OUT_TOL, build_pair, make_workload, rel_rms_err
from quantized_routed_expert_group_b200 import ep, moe, synth

pytestmark = pytest.mark.gpu

TC4 = synth.LayerShape(512, 256, 32, 4, 2, 4, 1, 2.5, 4)
GROUP32_TOPP = synth.LayerShape(512, 128, 128, 4, 2, 8, 1, 2.5, 4, topp=0.7)


@pytest.mark.parametrize("shape,T,world", [(TC4, 1, 2), (TC4, 3, 3), (TC4, 17, 2), (TC4, 100, 4),
                                           (GROUP32_TOPP, 2, 2), (GROUP32_TOPP, 70, 3)])
def test_partial_shares_sum_to_the_layer(shape, T, world):
    pair = build_pair(make_workload("ep", shape, T, 91 + T), T_max=T)
    layer = pair.layer
    x = torch.from_numpy(pair.x).cuda()
    full = layer.forward(x).clone()
    idx_full = layer.view(T)["idx"].clone()
    total = torch.zeros_like(full, dtype=torch.float64)
    for r in range(world):
        lo, hi = ep.expert_range(r, world, shape.n_experts)
        part = layer.forward_partial(x, lo, hi, ep.owns_shared(r))
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        assert torch.equal(layer.view(T)["idx"], idx_full)  # every rank routes every token the same
        total += part.double()
    got = total.float().cpu().numpy()
    ref = full.cpu().numpy()
    assert rel_rms_err(got, ref) <= 1e-5
    tr = orc.layer_forward(shape, pair.x, pair.router_w, pair.bias, pair.orc_routed, pair.orc_shared)
    assert rel_rms_err(got, tr.out) <= OUT_TOL


def test_partial_rejects_bad_ranges():
    pair = build_pair(make_workload("ep_bad", TC4, 2, 5), T_max=2)
    x = torch.from_numpy(pair.x).cuda()
    for lo, hi, sh in ((-1, 4, True), (5, 4, True), (0, TC4.n_experts + 1, False)):
        with pytest.raises(moe.MoeError):
            pair.layer.forward_partial(x, lo, hi, sh)
    import ctypes
    L = pair.layer
    out = torch.empty_like(x)
    st = moe.lib().moe_layer_forward_partial(
        ctypes.byref(L.cfg), ctypes.c_void_p(x.data_ptr()), 2, ctypes.c_void_p(L.router_w.data_ptr()),
        ctypes.c_void_p(L.bias.data_ptr()), ctypes.byref(L._routed_s), ctypes.byref(L._shared_s), 0, 4, 2,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(L.workspace.data_ptr()), L.workspace.numel(), None)
    assert st == moe.MOE_EINVAL  # with_shared is 0 or 1
