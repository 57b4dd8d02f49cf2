"""Host-side checks of the C ABI (no GPU needed).

The library loads on a machine without a GPU; every function declared in
include/moe.h is exported; argument validation answers with the documented
status before anything touches the device (the pointers passed here are never
dereferenced).
"""
import ctypes
import os
import re

import pytest

from quantized_routed_expert_group_b200 import build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    build.build_lib()
    from quantized_routed_expert_group_b200 import moe
    return moe


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("moe_quantize_act_q8_0", "moe_router_select", "moe_layer_forward", "moe_workspace_bytes",
                     "moe_bucket_tokens", "moe_pack_weights", "moe_block_dots", "moe_get_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    lib = ctypes.CDLL(build.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_python_binding_covers_every_symbol(L):
    assert set(declared_functions()) <= set(L._SIGS)


def test_status_strings(L):
    for st in (0, -1, -2, -3, -4, -5):
        assert L.status_string(st).startswith("MOE_")
    assert "unknown" in L.status_string(42)


def _cfg(L, **kw):
    s = synth.GLM_INT4
    c = L.config(s)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("kw,status", [
    ({"hidden": 6000}, -2), ({"inter": 100}, -2), ({"wbits": 3}, -2), ({"wbits": 1}, -2),
    ({"n_groups": 7}, -1), ({"topk_groups": 9}, -1), ({"top_k": 129}, -1), ({"top_k": 33, "topk_groups": 8}, -2),
    ({"n_experts": 2048, "n_groups": 16}, -2), ({"n_shared": 2}, -2), ({"n_experts": 8, "n_groups": 8, "top_k": 2}, -2),
    ({"top_k": 0}, -1), ({"routed_scaling_factor": float("nan")}, -1),
    ({"expert_topp": float("nan")}, -1), ({"expert_topp": -0.5}, -1), ({"expert_topp": float("inf")}, -1),
])
def test_config_validation(L, kw, status):
    c = _cfg(L, **kw)
    assert L.lib().moe_workspace_bytes(ctypes.byref(c), 4) == 0
    ex = L.MoeExperts(*([0x1000] * 6))
    st = L.lib().moe_layer_forward(ctypes.byref(c), 0x1000, 1, 0x1000, 0x1000, ctypes.byref(ex), ctypes.byref(ex),
                                   0x1000, 0x1000, 1 << 40, None)
    assert st == status


def test_workspace_bytes_monotone_and_aligned(L):
    c = _cfg(L)
    sizes = [L.lib().moe_workspace_bytes(ctypes.byref(c), T) for T in (0, 1, 4, 16, 512)]
    assert all(s % 256 == 0 for s in sizes)
    assert sizes == sorted(sizes) and sizes[0] > 0
    # T=512 holds at least the per-slot expert outputs (fp32) and h codes
    slots = 512 * 9
    assert sizes[-1] >= slots * 6144 * 4 + slots * 2048


def test_forward_argument_errors(L):
    c = _cfg(L)
    lib = L.lib()
    ex = L.MoeExperts(*([0x1000] * 6))
    need = lib.moe_workspace_bytes(ctypes.byref(c), 4)
    args = dict(x=0x1000, T=4, rw=0x1000, rb=0x1000, out=0x1000, ws=0x1000, nbytes=need)

    def call(**kw):
        a = dict(args, **kw)
        return lib.moe_layer_forward(ctypes.byref(c), a["x"], a["T"], a["rw"], a["rb"], ctypes.byref(ex),
                                     ctypes.byref(ex), a["out"], a["ws"], a["nbytes"], None)

    assert call(x=0) == -1                 # null x
    assert call(x=0x1004) == -1            # x not 16-byte aligned
    assert call(ws=0x1010) == -1           # workspace not 256-byte aligned
    assert call(rw=0x1008) == -1           # router weight not 16-byte aligned
    assert call(T=-1) == -1
    assert call(nbytes=need - 1) == -3     # workspace too small
    assert call(T=5000) == -2              # beyond the bucketing limit
    bad = L.MoeExperts(0x1008, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    assert lib.moe_layer_forward(ctypes.byref(c), 0x1000, 4, 0x1000, 0x1000, ctypes.byref(bad), ctypes.byref(ex),
                                 0x1000, 0x1000, need, None) == -1
    assert lib.moe_layer_forward(ctypes.byref(c), 0x1000, 4, 0x1000, 0x1000, None, ctypes.byref(ex),
                                 0x1000, 0x1000, need, None) == -1


def test_other_entry_point_errors(L):
    lib = L.lib()
    c = _cfg(L)
    assert lib.moe_quantize_act_q8_0(0x1000, 1, 33, 0x1000, 0x1000, None) == -1
    assert lib.moe_quantize_act_q8_0(0x1000, -1, 32, 0x1000, 0x1000, None) == -1
    assert lib.moe_quantize_act_q8_0(0x1000, 0, 32, 0x1000, 0x1000, None) == 0   # nothing to do
    assert lib.moe_pack_weights(0x1000, 4, 64, 3, 0x1000, 0x1000, None) == -2
    assert lib.moe_pack_weights(0x1004, 4, 64, 4, 0x1000, 0x1000, None) == -1
    assert lib.moe_block_dots(0x1000, 4, 48, 4, 0x1000, 1, 0x1000, None) == -1
    assert lib.moe_block_dots(0x1000, 4, 64, 3, 0x1000, 1, 0x1000, None) == -2
    ex = L.MoeExperts(*([0x1000] * 6))
    big = 1 << 40
    for lo, hi, sh in ((-1, 3, 1), (4, 3, 1), (0, c.n_experts + 1, 1), (0, 3, 2)):
        assert lib.moe_layer_forward_partial(ctypes.byref(c), 0x1000, 1, 0x1000, 0x1000, ctypes.byref(ex),
                                             ctypes.byref(ex), lo, hi, sh, 0x1000, 0x1000, big, None) == -1
    assert lib.moe_layer_forward_partial(ctypes.byref(c), 0x1000, 0, 0x1000, 0x1000, ctypes.byref(ex),
                                         ctypes.byref(ex), 0, 3, 0, 0x1000, 0x1000, big, None) == 0  # T = 0
    assert lib.moe_block_dots_routine(0x1000, 4, 64, 4, 0x1000, 1, 7, 0x1000, None) == -2   # unknown routine
    assert lib.moe_block_dots_routine(0x1000, 4, 48, 4, 0x1000, 1, 1, 0x1000, None) == -1   # cols % 32
    assert lib.moe_block_dots_routine(0x1000, 0, 64, 4, 0x1000, 1, 1, 0x1000, None) == 0    # nothing to do
    assert lib.moe_requant_fp8(0x1000, 0x1000, 4, 48, 128, 4, 0x1000, 0x1000, None) == -1   # cols % 32
    assert lib.moe_requant_fp8(0x1000, 0x1000, 4, 64, 100, 4, 0x1000, 0x1000, None) == -1   # block % 32
    assert lib.moe_requant_fp8(0x1000, 0x1000, 4, 64, 128, 3, 0x1000, 0x1000, None) == -2   # wbits
    assert lib.moe_requant_fp8(0x1000, 0x1000, 0, 64, 128, 4, 0x1000, 0x1000, None) == 0    # nothing to do
    assert lib.moe_requant_fp8(0x1000, 0x1000, 4, 64, 128, 4, 0x1004, 0x1000, None) == -1   # packed alignment
    assert lib.moe_requant_fp8(None, 0x1000, 4, 64, 128, 4, 0x1000, 0x1000, None) == -1
    assert lib.moe_router_select(ctypes.byref(c), 0x1000, 4, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 16, None) == -3
    assert lib.moe_router_workspace_bytes(ctypes.byref(c), 4) >= 4 * 256 * 8
    assert lib.moe_synth_normal(1, 2, -1, 4, 1.0, 0x1000, None) == -1
    code = ctypes.c_int32(0)
    assert lib.moe_get_device_error(None, None, ctypes.byref(code)) == -1


def test_forward_paths_and_phases(L):
    """T <= 4 takes the fused small-batch path (one launch, one traced phase);
    larger batches the multi-kernel path (five phases; 8 launches at 16
    tokens: the router's split-K logits add their reduction from 5 tokens)."""
    c = _cfg(L)
    assert L.forward_phases(c, 1) == ["fused"] and L.forward_launches(c, 1) == 1
    assert L.forward_phases(c, 4) == ["fused"]
    assert L.forward_phases(c, 5) == ["route", "bucket", "gate_up", "down", "combine"]
    assert L.forward_launches(c, 16) == 8 and L.forward_launches(c, 0) == 0
    big = _cfg(L, n_experts=512, n_groups=16)   # beyond the fused path's 256 experts
    assert L.forward_phases(big, 1) == ["route", "bucket", "gate_up", "down", "combine"]
    assert L.lib().moe_profile_events(None, 3) == -1


@pytest.mark.parametrize("shape,T,fused", [
    (synth.GLM_INT4, 1, True), (synth.GLM_INT4, 4, True), (synth.GLM_INT4, 5, False),
    (synth.GLM_INT8, 4, True), (synth.GLM_INT2, 1, True),
    # int2 rows of 264 / 40 bytes are not 16-byte multiples: the multi-kernel path
    (synth.LayerShape(1056, 160, 32, 4, 2, 4, 1, 2.5, 2), 3, False),
    (synth.LayerShape(1088, 192, 32, 4, 2, 4, 1, 2.5, 2), 4, True),
    (synth.LayerShape(1056, 160, 32, 4, 2, 4, 1, 2.5, 4), 4, True),
])
def test_path_selection(L, shape, T, fused):
    """Which path a forward takes (host logic, the device's sizes defaulting to
    a B200's 148 SMs and 227 KB of shared memory per block without a GPU)."""
    c = L.config(shape)
    phases = L.forward_phases(c, T)
    assert (phases == ["fused"]) == fused, phases
    # multi-kernel: 7 launches, one more (the split-K router reduction) from 5 tokens
    assert L.forward_launches(c, T) == (1 if fused else 8 if T >= 5 else 7)
