"""The one-token fused forward's down-row split (host export of the split
every CTA computes; no GPU): the CTAs' row ranges tile [0, hidden) exactly,
in order, within the per-CTA cap, and the CTAs that stream one routed
gate/up unit more own no more rows than the others.  At 2-4 tokens the split
is even."""
import pytest

from quantized_routed_expert_group_b200 import moe, synth

SHAPES = [synth.WORKLOADS[n].shape for n in ("glm52_decode_int4_t1", "glm52_decode_int2_t1", "glm52_int8_t16_outliers",
                                             "tiny_h256_e16_int8_t4")] + [
    synth.LayerShape(512, 256, 32, 4, 2, 4, 1, 2.5, 4),
    synth.LayerShape(256, 128, 16, 2, 1, 4, 0, 1.5, 4),
    synth.LayerShape(640, 128, 32, 4, 2, 4, 1, 2.5, 2),
]


def _check_tiling(starts, H, cap):
    assert starts[0] == 0 and starts[-1] == H
    sizes = starts[1:] - starts[:-1]
    assert (sizes >= 0).all()
    if cap > 0:
        assert sizes.max() <= cap
    return sizes


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"h{s.hidden}_i{s.inter}_e{s.n_experts}_w{s.wbits}_ns{s.n_shared}")
@pytest.mark.parametrize("grid", [148, 132, 64])
def test_one_token_split_tiles_the_rows(shape, grid):
    cfg = moe.config(shape)
    max_ent = 1 + min(shape.n_experts, shape.top_k)
    for n_entries in range(1, max_ent + 1):
        starts, cap = moe.debug_down_rows(cfg, 1, n_entries, grid)
        _check_tiling(starts, shape.hidden, cap)


def test_glm_decode_split_balances_the_units():
    s = synth.WORKLOADS["glm52_decode_int4_t1"].shape
    starts, cap = moe.debug_down_rows(moe.config(s), 1, s.top_k + s.n_shared, 148)
    sizes = _check_tiling(starts, s.hidden, cap)
    # 9 experts x 64 units dealt round robin over 148 CTAs, the shared
    # expert's 64 first: CTAs 64-131 stream 4 routed units, the others 3
    assert cap == 48
    assert sizes[64:132].max() <= sizes[:64].min()
    assert sizes[64:132].max() <= sizes[132:].min()


@pytest.mark.parametrize("T", [2, 3, 4])
def test_several_tokens_split_evenly(T):
    s = synth.WORKLOADS["glm52_verify_int4_t4"].shape
    starts, cap = moe.debug_down_rows(moe.config(s), T, 1 + min(s.n_experts, T * s.top_k), 148)
    assert cap == 0
    assert list(starts) == [s.hidden * c // 148 for c in range(149)]


def test_bad_arguments_are_rejected():
    s = synth.WORKLOADS["glm52_decode_int4_t1"].shape
    cfg = moe.config(s)
    for T, n, grid in ((0, 2, 148), (5, 2, 148), (1, 0, 148), (1, s.top_k + 2, 148), (1, 2, 0)):
        with pytest.raises(moe.MoeError):
            moe.debug_down_rows(cfg, T, n, grid)
