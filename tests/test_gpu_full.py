"""GPU vs oracle at the GLM-5.2 layer's full sizes (hidden 6144, intermediate
2048, 256 experts resident in HBM), in the launch configuration bench.py times.

All 256 experts are drawn and packed on the GPU; the oracle regenerates on the
host only the experts the sampled tokens need and packs them itself.  Checked:
packed bytes of those experts (bit-exact), expert indices and bucketing for
every token (bit-exact), per-block int32 dots of gate/up and down rows
(bit-exact), and the sampled tokens' fp32 outputs (1e-3 of their RMS)."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity_helpers import OUT_TOL, host_expert_mats, rel_rms_err
from quantized_routed_expert_group_b200 import moe, synth

pytestmark = pytest.mark.gpu

FULL = ["glm52_decode_int4_t1", "glm52_verify_int4_t4", "glm52_int8_t16_outliers", "glm52_prefill_int4_t512_zipf",
        "glm52_decode_int4_t1_topp07", "glm52_decode_int2_t1"]


@pytest.fixture(scope="module", params=FULL)
def full(request):
    wl = synth.WORKLOADS[request.param]
    layer = moe.synth_layer(wl)
    x = synth.make_x(wl)
    out = layer.forward(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    view = {k: v.cpu().numpy() for k, v in layer.view(wl.T).items()}
    yield wl, layer, x, out.cpu().numpy(), view
    del layer, out
    torch.cuda.empty_cache()


def _sample_tokens(T):
    """Every token of a batch of at most 16, else 16 spread over the batch
    (first and last included)."""
    if T <= 16:
        return list(range(T))
    return sorted(set(np.linspace(0, T - 1, 16).round().astype(int).tolist()))


def test_full_router_and_bucket(full):
    wl, layer, x, out, v = full
    s = wl.shape
    io, wo, c, gs = orc.router(x, synth.make_router_w(wl), synth.make_bias(wl), s.n_groups, s.topk_groups,
                               s.top_k, s.rsf, want_scores=True, topp=s.topp)
    np.testing.assert_array_equal(v["idx"], io)
    np.testing.assert_allclose(v["w"], wo, rtol=1e-6)
    counts, offsets, perm = orc.bucket(io, s.n_experts)
    np.testing.assert_array_equal(v["counts"], counts)
    np.testing.assert_array_equal(v["offsets"], offsets)
    np.testing.assert_array_equal(v["perm"], perm)
    print(wl.name, "unique experts:", int((counts > 0).sum()), "max tokens/expert:", int(counts.max()))


def test_full_sampled_outputs(full):
    wl, layer, x, out, v = full
    s = wl.shape
    toks = _sample_tokens(wl.T)
    need = sorted(set(v["idx"][toks].reshape(-1).tolist()) - {-1})  # -1: dropped by the top-p
    routed = {}
    for e in need:
        ex = orc.pack_expert(*host_expert_mats(wl, e), s.wbits)
        routed[e] = ex
        # the GPU packed the device-generated weights to the same bytes
        np.testing.assert_array_equal(layer.routed.w_gate[e].cpu().numpy(), ex.wg)
        np.testing.assert_array_equal(layer.routed.w_up[e].cpu().numpy(), ex.wu)
        np.testing.assert_array_equal(layer.routed.w_down[e].cpu().numpy(), ex.wd)
        np.testing.assert_array_equal(layer.routed.s_down[e].cpu().numpy().view(np.uint32), ex.sd.view(np.uint32))
    shared = orc.pack_expert(*host_expert_mats(wl, 0, shared=True), s.wbits)
    np.testing.assert_array_equal(layer.shared.w_gate[0].cpu().numpy(), shared.wg)
    tr = orc.layer_forward(s, x[toks], synth.make_router_w(wl), synth.make_bias(wl), routed, shared)
    err = rel_rms_err(out[toks], tr.out)
    print(wl.name, "tokens", toks, "max err / rms =", err)
    assert err <= OUT_TOL
    # per-block int32 dots, bit-exact: gate rows on x's codes, down rows on the
    # oracle's own h codes (h itself may round differently by a few ulp)
    t0 = toks[0]
    j0 = int(np.nonzero(v["idx"][t0] >= 0)[0][0])  # the first pick the top-p kept (0 without it)
    e0 = int(v["idx"][t0, j0])
    ex = routed[e0]
    xq = torch.from_numpy(tr.xq[0:1]).cuda()
    ref_g = orc.block_dots(ex.wg, s.hidden, s.wbits, tr.xq[0:1])
    hq = np.ascontiguousarray(tr.hq[0, j0:j0 + 1])
    ref_d = orc.block_dots(ex.wd, s.inter, s.wbits, hq)
    factor = {8: 1, 4: 16, 2: 64}[s.wbits]
    for routine, f in ((None, 1), (moe.DOTS_FUSED, factor)):
        got = moe.block_dots(layer.routed.w_gate[e0], s.hidden, s.wbits, xq, routine=routine).cpu().numpy()
        np.testing.assert_array_equal(got.astype(np.int64), f * ref_g.astype(np.int64))
        got = moe.block_dots(layer.routed.w_down[e0], s.inter, s.wbits, torch.from_numpy(hq).cuda(),
                             routine=routine).cpu().numpy()
        np.testing.assert_array_equal(got.astype(np.int64), f * ref_d.astype(np.int64))


def test_full_hot_expert_slots(full):
    """Per-slot expert outputs y (before the combine) of EVERY token routed to
    the two most loaded experts, and of the shared expert on every token,
    against the oracle's expert FFN on the oracle's own Q8_0 codes of x."""
    wl, layer, x, out, v = full
    s = wl.shape
    if wl.T < 2:
        pytest.skip("one token: the sampled-output test covers every slot")
    counts, offsets, perm = v["counts"], v["offsets"], v["perm"]
    hot = [int(e) for e in np.argsort(-counts, kind="stable")[:2] if counts[e] > 0]
    xq, xd = orc.q8_0_quantize(x)
    checked = 0
    for e in hot:
        ex = orc.pack_expert(*host_expert_mats(wl, e), s.wbits)
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        toks = perm[lo:hi] // s.top_k
        ref = np.stack([orc.expert_ffn(ex, s.hidden, s.inter, s.wbits, xq[t], xd[t])[0] for t in toks])
        err = rel_rms_err(v["y"][lo:hi], ref)
        print(wl.name, "expert", e, "tokens", hi - lo, "y err / rms =", err)
        assert err <= OUT_TOL
        checked += hi - lo
    if s.n_shared:
        sh = orc.pack_expert(*host_expert_mats(wl, 0, shared=True), s.wbits)
        base = wl.T * s.top_k
        ref = np.stack([orc.expert_ffn(sh, s.hidden, s.inter, s.wbits, xq[t], xd[t])[0] for t in range(wl.T)])
        err = rel_rms_err(v["y"][base:base + wl.T], ref)
        print(wl.name, "shared expert y err / rms =", err)
        assert err <= OUT_TOL
        checked += wl.T
    assert checked >= min(wl.T, 16)
