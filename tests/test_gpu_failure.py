"""Failure detection on the GPU without a fault: a device-side wait that runs
out must end the kernel with an error status that the host reads, leave the
context usable, and leave the next forward correct.

The fused small-batch kernel's down projection waits for other CTAs' h codes.
The test hook moe_debug_fault_injection makes one entry's first gate/up unit
skip its publication (nothing else changes), with a short wait bound, so that
wait runs out on every CTA: the kernel records code 2 (a wait ran out) and
returns.  Every wait in the kernel is bounded by the GPU's global timer, so
the forward ends in about the bound, not after a hang."""
import time

import pytest
import torch

from parity_helpers import build_pair, check_layer, make_workload
from quantized_routed_expert_group_b200 import moe, synth

pytestmark = pytest.mark.gpu

MID4 = synth.LayerShape(1056, 160, 32, 4, 2, 4, 1, 2.5, 4)
GROUP32 = synth.LayerShape(512, 96, 128, 4, 2, 8, 1, 2.5, 4)
BUDGET_NS = 2_000_000  # 2 ms for the producer's waits (the others: 8 ms)


@pytest.fixture(autouse=True)
def _hook_off():
    yield
    moe.debug_fault_injection(-1, 0)


@pytest.mark.parametrize("shape,T,entry", [(MID4, 1, 0), (MID4, 4, 1), (GROUP32, 2, 0), (GROUP32, 3, 2)])
def test_withheld_publication_times_out_then_recovers(shape, T, entry):
    pair = build_pair(make_workload("fault", shape, T, 31), T_max=T)
    layer = pair.layer
    assert moe.forward_phases(layer.cfg, T) == ["fused"]
    x = torch.from_numpy(pair.x).cuda()
    layer.forward(x)
    torch.cuda.synchronize()
    assert layer.device_error() == 0

    moe.debug_fault_injection(entry, BUDGET_NS)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    layer.forward(x)  # returns MOE_OK: the fault is found on the device
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert layer.device_error() == 2, "the withheld wait must record a timeout"
    assert dt < 1.0, f"the forward took {dt:.3f} s: the waits must end near their bound"

    # the context is still usable and the next forward is correct
    moe.debug_fault_injection(-1, 0)
    check_layer(pair)
    assert layer.device_error() == 0


def test_fault_hook_rejects_bad_arguments():
    assert moe.lib().moe_debug_fault_injection(-2, 0) == moe.MOE_EINVAL
    assert moe.lib().moe_debug_fault_injection(0, -1) == moe.MOE_EINVAL
    assert moe.lib().moe_debug_fault_injection(-1, 0) == moe.MOE_OK
