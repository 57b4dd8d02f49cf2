"""Pins of the oracle's adaptive expert top-p (CPU only).

The pages name the option (an adaptive expert top-p, 0.7 in their example)
but give no rule; the oracle reads it as nucleus selection over the k picks:
order the picks by their share q = s / sum(s) (ties: the earlier pick), keep
the shortest prefix whose running sum reaches topp (at least one pick), drop
the rest (idx -1, w 0) and renormalise the kept weights to the scaling
factor.  Fixed here by hand-worked cases, by the definition's properties
checked against the plain router's picks (minimal prefix, coverage,
renormalisation, kept picks in place), by the degenerate settings that must
reduce to the plain router, and, for the layer, by recombining the plain
layer's per-slot expert outputs with the top-p weights.
"""
import numpy as np
import pytest

from quantized_routed_expert_group_b200 import synth


def _one_token(logits, bias):
    E = len(logits)
    x = np.ones((1, 1), np.float32)
    Wr = np.array(logits, np.float32).reshape(E, 1)
    return x, Wr, np.array(bias, np.float32)


S3 = [np.log(9.0), np.log(1.5), np.log(3.0 / 7.0), -5.0]  # s = 0.9, 0.6, 0.3, ~0.0067


@pytest.mark.parametrize("topp,idx,w", [
    # shares 0.5, 0.333, 0.167: 0.5 < 0.7 <= 0.833 -> two picks, w = 0.9 : 0.6
    (0.7, [0, 1, -1], [0.6, 0.4, 0.0]),
    # 0.45 <= 0.5 -> the first pick alone carries the whole scaling factor
    (0.45, [0, -1, -1], [1.0, 0.0, 0.0]),
    # 0.9 > 0.833 -> every pick, the plain weights s / sum(s)
    (0.9, [0, 1, 2], [0.5, 1.0 / 3.0, 1.0 / 6.0]),
])
def test_topp_hand_worked(orc, topp, idx, w):
    x, Wr, bias = _one_token(S3, [0.0] * 4)
    gi, gw = orc.router(x, Wr, bias, 1, 1, 3, 1.0, topp=topp)
    assert gi[0].tolist() == idx
    np.testing.assert_allclose(gw[0], w, rtol=1e-6, atol=1e-7)


def test_topp_orders_by_share_not_by_biased_score(orc):
    # s = 0.3, 0.9, 0.6, ~0; the bias puts expert 0 first among the picks, but
    # its share is the smallest, so the top-p drops it and keeps 1 and 2
    x, Wr, bias = _one_token([np.log(3.0 / 7.0), np.log(9.0), np.log(1.5), -5.0], [1.0, 0.0, 0.0, 0.0])
    gi, gw = orc.router(x, Wr, bias, 1, 1, 3, 2.5)
    assert gi[0].tolist() == [0, 1, 2]
    gi, gw = orc.router(x, Wr, bias, 1, 1, 3, 2.5, topp=0.7)
    assert gi[0].tolist() == [-1, 1, 2]
    np.testing.assert_allclose(gw[0], [0.0, 1.5, 1.0], rtol=1e-6)


def test_topp_ties_keep_the_earlier_pick(orc):
    # three equal shares of 1/3: 0.5 is reached after two picks; the equal
    # scores make the picks 0, 1, 2 (lower index first) and the earlier two stay
    x, Wr, bias = _one_token([0.4, 0.4, 0.4, -5.0], [0.0] * 4)
    gi, gw = orc.router(x, Wr, bias, 1, 1, 3, 2.0, topp=0.5)
    assert gi[0].tolist() == [0, 1, -1]
    np.testing.assert_allclose(gw[0], [1.0, 1.0, 0.0], rtol=1e-6)


@pytest.mark.parametrize("topp", [0.0, 1.0, 1.5])
def test_topp_off_is_the_plain_router(orc, topp):
    wl = synth.WORKLOADS["glm52_decode_int4_t1"].with_tokens(6)
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    i0, w0 = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf)
    i1, w1 = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf, topp=topp)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_array_equal(w0.view(np.uint32), w1.view(np.uint32))


@pytest.mark.parametrize("name,T", [("tiny_h256_e16_int8_t4", 64), ("glm52_decode_int4_t1", 8)])
@pytest.mark.parametrize("topp", [0.3, 0.7, 0.95])
def test_topp_properties(orc, name, T, topp):
    wl = synth.WORKLOADS[name].with_tokens(T)
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    i0, w0 = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf)
    i1, w1 = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf, topp=topp)
    logit = x.astype(np.float64) @ Wr.astype(np.float64).T
    sig = 1.0 / (1.0 + np.exp(-logit))
    for t in range(T):
        kept = i1[t] >= 0
        # kept picks stay in place; dropped ones carry no weight
        assert kept.any()
        np.testing.assert_array_equal(i1[t][kept], i0[t][kept])
        assert np.all(w1[t][~kept] == 0.0)
        sv = sig[t, i0[t]]
        q = sv / sv.sum()
        # the kept picks are the largest shares, and the shortest such prefix
        # that reaches topp
        order = sorted(range(s.top_k), key=lambda j: (-q[j], j))
        m = int(kept.sum())
        assert set(np.nonzero(kept)[0].tolist()) == set(order[:m])
        assert q[order[:m]].sum() >= topp - 1e-12
        assert q[order[:m - 1]].sum() < topp + 1e-12
        # renormalised to the scaling factor, in the ratio of the kept s
        np.testing.assert_allclose(w1[t][kept].sum(), s.rsf, rtol=1e-6)
        np.testing.assert_allclose(w1[t][kept], sv[kept] / sv[kept].sum() * s.rsf, rtol=1e-6)


def test_topp_drops_picks_on_the_decode_workload(orc):
    # with near-uniform shares 0.7 needs about 0.7 * 8 picks: some are dropped
    wl = synth.WORKLOADS["glm52_decode_int4_t1_topp07"].with_tokens(16)
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    i1, _ = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf, topp=s.topp)
    kept = (i1 >= 0).sum(axis=1)
    assert kept.min() >= 1 and kept.max() < s.top_k


def test_bucket_skips_dropped_picks(orc):
    rng = np.random.default_rng(5)
    T, k, E = 9, 4, 16
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[rng.random((T, k)) < 0.4] = -1
    counts, offsets, perm = orc.bucket(idx, E)
    flat = idx.reshape(-1)
    live = np.nonzero(flat >= 0)[0]
    np.testing.assert_array_equal(counts, np.bincount(flat[live], minlength=E))
    assert offsets[-1] == len(live)
    # stable: by expert, then by (token, slot)
    ref = live[np.argsort(flat[live], kind="stable")]
    np.testing.assert_array_equal(perm[: len(live)], ref)
    assert np.all(perm[len(live):] == -1)


def test_topp_layer_is_the_plain_layer_reweighted(orc):
    """The top-p layer reads the same experts at the kept positions, so its
    output is the plain layer's per-slot expert outputs recombined with the
    top-p weights (plus the shared expert)."""
    from parity_helpers import host_expert_mats
    base = synth.WORKLOADS["tiny_h256_e16_int8_t4"].with_tokens(12)
    shp = base.shape
    wl = synth.Workload("tiny_topp", synth.LayerShape(shp.hidden, shp.inter, shp.n_experts, shp.n_groups,
                                                      shp.topk_groups, 4, shp.n_shared, shp.rsf, shp.wbits,
                                                      topp=0.6), 12, base.seed)
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    routed = {e: orc.pack_expert(*host_expert_mats(wl, e), s.wbits) for e in range(s.n_experts)}
    shared = orc.pack_expert(*host_expert_mats(wl, 0, True), s.wbits)
    plain = orc.layer_forward(synth.LayerShape(*[getattr(s, f) for f in
                                                 ("hidden", "inter", "n_experts", "n_groups", "topk_groups",
                                                  "top_k", "n_shared", "rsf", "wbits")]),
                              x, Wr, bias, routed, shared)
    tp = orc.layer_forward(s, x, Wr, bias, routed, shared)
    kept = tp.idx >= 0
    assert (~kept).any() and kept.any()
    np.testing.assert_array_equal(tp.idx[kept], plain.idx[kept])
    ref = np.einsum("tj,tjh->th", np.where(kept, tp.w, 0.0).astype(np.float64),
                    plain.ys[:, : s.top_k].astype(np.float64)) + plain.ys[:, s.top_k].astype(np.float64)
    np.testing.assert_allclose(tp.out, ref, rtol=0, atol=1e-5 * np.abs(ref).max())
    # the dropped slots read nothing
    assert np.all(tp.ys[:, : s.top_k][~kept] == 0.0)
