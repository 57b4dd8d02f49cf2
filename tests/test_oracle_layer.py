"""Pins of the oracle's integer dots, expert FFN and layer forward (CPU only).

Fixed by: brute-force int64 sums on codes unpacked with numpy bit operations
(the bit layout itself is pinned by tests/golden/packing.json), numpy fp64
matmuls of dequantised weights and activations, and consistency between the
layer's trace and its separately pinned steps.
"""
import numpy as np
import pytest

from quantized_routed_expert_group_b200 import synth


def np_unpack(packed, cols, wbits):
    """Codes of a packed [rows][bytes] matrix, by numpy bit extraction."""
    p = packed.astype(np.int32)
    if wbits == 8:
        v = p
    else:
        per = 8 // wbits
        fields = (p[..., None] >> (wbits * np.arange(per))) & ((1 << wbits) - 1)
        v = fields.reshape(p.shape[0], -1)
    half = 1 << (wbits - 1)
    v = np.where(v >= half, v - 2 * half, v) if wbits < 8 else np.where(v >= 128, v - 256, v)
    return v[:, :cols].astype(np.int64)


@pytest.mark.parametrize("wbits", [8, 4, 2])
def test_block_dots_bruteforce(orc, wbits):
    rng = np.random.default_rng(10 + wbits)
    rows, cols, n = 24, 160, 3
    w = rng.standard_normal((rows, cols)).astype(np.float32)
    packed, _ = orc.quantize_rows(w, wbits)
    q = rng.integers(-127, 128, size=(n, cols), dtype=np.int64).astype(np.int8)
    q[0, :32] = 127  # extreme block
    got = orc.block_dots(packed, cols, wbits, q)
    codes = np_unpack(packed, cols, wbits)
    ref = np.einsum("rbi,tbi->trb", codes.reshape(rows, -1, 32), q.astype(np.int64).reshape(n, -1, 32))
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("wbits", [8, 4, 2])
def test_qmatvec_is_dequantised_dot(orc, wbits):
    """s * sum_b d_b * isum_b equals sum_i (s q_w,i)(d_b q_x,i) (fp64), rounded once to fp32."""
    rng = np.random.default_rng(20 + wbits)
    rows, cols = 64, 512
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    x = rng.standard_normal(cols).astype(np.float32)
    packed, s = orc.quantize_rows(w, wbits)
    xq, xd = orc.q8_0_quantize(x)
    y = orc.qmatvec(packed, s, cols, wbits, xq, xd)
    wdeq = s.astype(np.float64)[:, None] * np_unpack(packed, cols, wbits)
    xdeq = np.repeat(xd.astype(np.float64), 32) * xq.astype(np.float64)
    ref = wdeq @ xdeq
    np.testing.assert_allclose(y, ref, rtol=2e-7 * 4, atol=1e-12 * np.abs(ref).max())
    assert np.max(np.abs(y.astype(np.float64) - ref) / np.maximum(np.abs(ref), 1e-30)) < 1e-6


def _tiny_expert(orc, wl, e, shared=False):
    m = [synth.make_expert_matrix(wl, e, k, shared) for k in (0, 1, 2)]
    return m, orc.pack_expert(*m, wl.shape.wbits)


def _silu(v):
    return v / (1.0 + np.exp(-v))


@pytest.mark.parametrize("wbits", [8, 4, 2])
def test_expert_ffn_dequantised_fp64(orc, wbits):
    from dataclasses import replace
    base = synth.WORKLOADS["tiny_h256_e16_int8_t4"]
    wl = replace(base, shape=replace(base.shape, wbits=wbits))
    s = wl.shape
    x = synth.make_x(wl)
    (_, ex) = _tiny_expert(orc, wl, 3)
    for t in range(wl.T):
        xq, xd = orc.q8_0_quantize(x[t])
        y, h, hq, hd = orc.expert_ffn(ex, s.hidden, s.inter, s.wbits, xq, xd)
        xdeq = np.repeat(xd.astype(np.float64), 32) * xq.astype(np.float64)
        g = (ex.sg.astype(np.float64)[:, None] * np_unpack(ex.wg, s.hidden, s.wbits)) @ xdeq
        u = (ex.su.astype(np.float64)[:, None] * np_unpack(ex.wu, s.hidden, s.wbits)) @ xdeq
        href = _silu(g) * u
        np.testing.assert_allclose(h, href, rtol=1e-5, atol=1e-6 * np.abs(href).max())
        # the down projection consumes Q8_0(h): hq/hd are that quantisation of h
        hq2, hd2 = orc.q8_0_quantize(h)
        np.testing.assert_array_equal(hq, hq2)
        np.testing.assert_array_equal(hd, hd2)
        hdeq = np.repeat(hd.astype(np.float64), 32) * hq.astype(np.float64)
        yref = (ex.sd.astype(np.float64)[:, None] * np_unpack(ex.wd, s.inter, s.wbits)) @ hdeq
        np.testing.assert_allclose(y, yref, rtol=1e-5, atol=1e-6 * np.abs(yref).max())


def _tiny_layer(orc, wl):
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    mats, routed = {}, {}
    for e in range(s.n_experts):
        mats[e], routed[e] = _tiny_expert(orc, wl, e)
    shm, shared = _tiny_expert(orc, wl, 0, shared=True)
    tr = orc.layer_forward(s, x, Wr, bias, routed, shared)
    return x, Wr, bias, mats, routed, shm, shared, tr


def test_layer_trace_consistent_with_steps(orc):
    wl = synth.WORKLOADS["tiny_h256_e16_int8_t4"]
    s = wl.shape
    x, Wr, bias, mats, routed, shm, shared, tr = _tiny_layer(orc, wl)
    idx, w = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf)
    np.testing.assert_array_equal(tr.idx, idx)
    np.testing.assert_array_equal(tr.w, w)
    xq, xd = orc.q8_0_quantize(x)
    np.testing.assert_array_equal(tr.xq, xq)
    np.testing.assert_array_equal(tr.xd, xd)
    for t in range(wl.T):
        for j in range(s.top_k + s.n_shared):
            ex = routed[int(idx[t, j])] if j < s.top_k else shared
            y, h, hq, hd = orc.expert_ffn(ex, s.hidden, s.inter, s.wbits, xq[t], xd[t])
            np.testing.assert_array_equal(tr.ys[t, j], y)
            np.testing.assert_array_equal(tr.hq[t, j], hq)
        # combine: sum_j w_j y_j + y_shared in fp64, rounded once
        ref = (w[t].astype(np.float64)[:, None] * tr.ys[t, :s.top_k].astype(np.float64)).sum(0) \
            + tr.ys[t, s.top_k].astype(np.float64)
        np.testing.assert_allclose(tr.out[t], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


def test_layer_against_unquantised_fp64(orc):
    """Quantisation error of the whole layer against an fp64 float MoE with the
    same routing (reported; bounded loosely as a sanity check)."""
    wl = synth.WORKLOADS["tiny_h256_e16_int8_t4"]
    s = wl.shape
    x, Wr, bias, mats, routed, shm, shared, tr = _tiny_layer(orc, wl)
    for t in range(wl.T):
        xt = x[t].astype(np.float64)
        acc = np.zeros(s.hidden)
        for j in range(s.top_k + 1):
            m = mats[int(tr.idx[t, j])] if j < s.top_k else shm
            g, u = m[0].astype(np.float64) @ xt, m[1].astype(np.float64) @ xt
            y = m[2].astype(np.float64) @ (_silu(g) * u)
            acc += (float(tr.w[t, j]) if j < s.top_k else 1.0) * y
        rel = np.abs(tr.out[t] - acc).max() / np.sqrt(np.mean(acc ** 2))
        print(f"token {t}: int8 layer vs fp64 float layer, max error / rms = {rel:.4f}")
        assert rel < 0.1


def test_layer_missing_expert_raises(orc):
    wl = synth.WORKLOADS["tiny_h256_e16_int8_t4"]
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    idx, _ = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf)
    _, sh = _tiny_expert(orc, wl, 0, shared=True)
    partial = {}
    for e in set(idx.reshape(-1).tolist()) - {int(idx[0, 0])}:
        partial[e] = _tiny_expert(orc, wl, e)[1]
    with pytest.raises(ValueError):
        orc.layer_forward(s, x, Wr, bias, partial, sh)
