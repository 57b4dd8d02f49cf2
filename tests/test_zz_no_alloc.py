"""The allocation-free forward (moe_layer_forward_noalloc) against the
workspace forward, through the C ABI.

It exists for callers that cannot allocate device memory at call time (a host
framework that owns the device's memory, a plugin handed only its input and
output buffers, a loop where cudaMalloc's possible device synchronisation is
not allowed); it uses a fixed 8 MiB device array inside the library instead of
a caller workspace.  This file is collected last so that, run after the other
tests, it sees a process whose device state they have already exercised; it
also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity_helpers import OUT_TOL, build_pair, make_workload, rel_rms_err
from quantized_routed_expert_group_b200 import moe, synth

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 8 << 20


def _call(layer, x, out):
    return moe.lib().moe_layer_forward_noalloc(
        ctypes.byref(layer.cfg), ctypes.c_void_p(x.data_ptr()), x.shape[0],
        ctypes.c_void_p(layer.router_w.data_ptr()), ctypes.c_void_p(layer.bias.data_ptr()),
        ctypes.byref(layer._routed_s), ctypes.byref(layer._shared_s), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("shape,T", [
    (synth.TINY, 4),
    (synth.LayerShape(1056, 160, 32, 4, 2, 4, 1, 2.5, 4), 5),
])
def test_noalloc_matches_workspace_forward_twice(shape, T):
    wl = make_workload("noalloc", shape, T, 21)
    pair = build_pair(wl, T_max=T)
    layer = pair.layer
    for call in range(2):
        # a different batch each call, so the second call cannot pass on the
        # first call's leftovers in the shared scratch
        x = torch.from_numpy(synth.make_x(make_workload("noalloc", shape, T, 100 + call))).cuda()
        ref = layer.forward(x).clone()
        out = torch.full_like(x, float("nan"))
        assert _call(layer, x, out) == moe.MOE_OK
        torch.cuda.synchronize()
        code = ctypes.c_int32(-1)
        assert moe.lib().moe_noalloc_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                                  ctypes.byref(code)) == moe.MOE_OK
        assert code.value == 0
        assert torch.isfinite(out).all()
        assert rel_rms_err(out.cpu().numpy(), ref.cpu().numpy()) <= OUT_TOL
        # the same deterministic kernels on the same inputs: bit-identical
        assert torch.equal(out, ref)


def test_noalloc_rejects_batches_beyond_its_scratch():
    shape = synth.GLM_INT4
    cfg = moe.config(shape)
    T_max = max(T for T in range(1, 256) if moe.lib().moe_workspace_bytes(ctypes.byref(cfg), T) <= NOALLOC_BYTES)
    assert moe.lib().moe_workspace_bytes(ctypes.byref(cfg), T_max + 1) > NOALLOC_BYTES
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    ex = moe.MoeExperts(*([dummy.data_ptr()] * 6))
    x = torch.zeros((T_max + 1, shape.hidden), dtype=torch.float32, device="cuda")
    st = moe.lib().moe_layer_forward_noalloc(ctypes.byref(cfg), ctypes.c_void_p(x.data_ptr()), T_max + 1,
                                             ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()),
                                             ctypes.byref(ex), ctypes.byref(ex), ctypes.c_void_p(x.data_ptr()),
                                             None)
    assert st == moe.MOE_EWORKSPACE
    assert "workspace" in moe.status_string(st)
