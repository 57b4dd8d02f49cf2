"""The batched expert path on the tcgen05 tensor cores (T >= 64 tokens) against
the oracle, through the C ABI.

At these batch sizes every selected expert meets several tokens per weight
row, so the layer runs the grouped int8 GEMMs.  Each token's block-scaled
Q8_0 activations (and each row's h) are split exactly into five signed int8
digit planes (block scales as integers over the token's smallest exponent,
while the exponents lie within 8 of each other), so the tensor core sums
the whole K in int32 per plane and the epilogue forms the exact sum once per
output, scales it by the row scale in fp64 and rounds to fp32 -- what the
oracle computes when its fp64 block sum is exact.  Tokens whose block scales
spread wider take the fp64-epilogue GEMM (exact int32 block dots, fp64 block
order).  SwiGLU is fp64, the combine fp64.  So beyond the 1e-3 output bound,
the h codes, the per-slot expert outputs y and the layer output are compared
bit for bit, and the test checks which GEMM form ran.

Shapes: hidden and intermediate multiples of 128 (one MMA tile of rows); 1-3
weight tiles per matrix and 2-5 pipeline stages per unit; token counts that
leave ragged 16-token groups and 48-token chunks; int8, int4 and int2 weights;
no shared expert; the adaptive top-p dropping picks."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity_helpers import OUT_TOL, build_pair, check_layer, make_workload, rel_rms_err
from quantized_routed_expert_group_b200 import moe, synth

pytestmark = pytest.mark.gpu

TC4 = synth.LayerShape(512, 256, 32, 4, 2, 4, 1, 2.5, 4)
TC8 = synth.LayerShape(384, 256, 24, 4, 2, 3, 1, 1.0, 8)
TC2 = synth.LayerShape(640, 128, 32, 4, 2, 4, 1, 2.5, 2)
TC4_NOSHARED = synth.LayerShape(256, 128, 16, 2, 1, 4, 0, 1.5, 4)
TC4_TOPP = synth.LayerShape(512, 256, 32, 4, 2, 4, 1, 2.5, 4, topp=0.6)
TC4_G32 = synth.LayerShape(256, 128, 128, 4, 2, 8, 1, 2.5, 4)   # groups of 32 experts, top-8, as GLM-5.2


def _strict(pair, x, fallback=(0, 0)):
    s = pair.wl.shape
    T = x.shape[0]
    assert moe.forward_launches(pair.layer.cfg, T) == moe.TC_LAUNCHES, "expected the tensor-core path"
    out = pair.layer.forward(torch.from_numpy(np.ascontiguousarray(x)).cuda())
    torch.cuda.synchronize()
    assert pair.layer.device_error() == 0
    # which GEMM form ran: the digit planes (0) or the fp64 epilogue (1), for x and h
    assert tuple(pair.layer.view(T)["fp64_fallback"].cpu().tolist()) == fallback
    tr = orc.layer_forward(s, x, pair.router_w, pair.bias, pair.orc_routed, pair.orc_shared)
    v = {k: t.cpu().numpy() for k, t in pair.layer.view(T).items()}
    got = out.cpu().numpy()
    assert rel_rms_err(got, tr.out) <= OUT_TOL
    np.testing.assert_array_equal(v["idx"], tr.idx)
    counts, offsets, perm = orc.bucket(tr.idx, s.n_experts)
    np.testing.assert_array_equal(v["perm"], perm)
    k = s.top_k
    n = int(offsets[-1])
    live = perm[:n]
    t_of = np.concatenate([live // k, np.arange(T)]) if s.n_shared else live // k
    j_of = np.concatenate([live % k, np.full(T, k)]) if s.n_shared else live % k
    slots = np.concatenate([np.arange(n), T * k + np.arange(T)]) if s.n_shared else np.arange(n)
    hq_mis = int((v["hq"][slots] != tr.hq[t_of, j_of]).sum())
    hd_mis = int((v["hd"][slots].view(np.uint32) != tr.hd[t_of, j_of].view(np.uint32)).sum())
    y_mis = int((v["y"][slots].view(np.uint32) != tr.ys[t_of, j_of].view(np.uint32)).sum())
    out_mis = int((got.view(np.uint32) != tr.out.view(np.uint32)).sum())
    print(f"{pair.wl.name} T={T}: h codes {hq_mis}/{v['hq'][slots].size} differ, h scales {hd_mis}, "
          f"y {y_mis}/{v['y'][slots].size}, out {out_mis}/{got.size}")
    assert hq_mis == 0 and hd_mis == 0
    assert y_mis == 0
    assert out_mis == 0


@pytest.mark.parametrize("shape,T", [(TC4, 64), (TC4, 100), (TC4, 300), (TC8, 64), (TC8, 257), (TC2, 96),
                                     (TC4_NOSHARED, 130), (TC4_TOPP, 200), (TC4_G32, 128)])
def test_tc_layer_bitexact(shape, T):
    pair = build_pair(make_workload(f"tc_{shape.wbits}", shape, T, 41 + T), T_max=T)
    st = check_layer(pair)
    print(st)
    _strict(pair, pair.x)


def test_tc_then_small_batches_share_a_workspace():
    """One workspace sized for 300 tokens serves the tensor-core path and the
    smaller batches' paths one after the other."""
    pair = build_pair(make_workload("tc_mixed", TC4, 300, 77), T_max=300)
    for T in (300, 3, 17, 64):
        x = synth.make_x(make_workload("tc_mixed", TC4, T, 500 + T))
        check_layer(pair, x)


def test_tc_wide_block_scales_take_the_fp64_epilogue():
    """Tokens whose block-scale exponents lie more than 8 apart do not fit the
    five digit planes and take the fp64-epilogue GEMM: x with some blocks
    scaled by 2^-12 on every third token (gate/up side), and a shared expert
    whose first 32 up rows are scaled by 1e-4, so that h's first block is tiny
    on every token (down side).  Still bit-identical."""
    def mutate(mats, shm):
        shm[1][:32] *= np.float32(1e-4)

    T = 80
    pair = build_pair(make_workload("tc_wide", TC4, T, 123), T_max=T, mutate=mutate)
    x = pair.x.copy()
    for t in range(0, T, 3):
        for b in range(0, TC4.hidden // 32, 5):
            x[t, 32 * b:32 * (b + 1)] *= np.float32(2.0 ** -12)
    _strict(pair, x, fallback=(1, 1))
