"""GPU parity of the individual steps against the oracle (bit-exact where the
result is integer or bytes).  Calls go through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from quantized_routed_expert_group_b200 import moe, synth

pytestmark = pytest.mark.gpu


def test_device_generator_matches_host():
    for seed, tid, off, n, sigma in ((1, 1000, 0, 100003, 0.02), (4, 3, 12345, 5000, 1.0), (0, 7, 2**33, 777, 0.5)):
        dev = moe.synth_normal(seed, tid, n, sigma, offset=off).cpu().numpy()
        host = synth.normal(seed, tid, n, sigma, offset=off)
        np.testing.assert_array_equal(dev.view(np.uint32), host.view(np.uint32))


@pytest.mark.parametrize("rows,cols,scale", [(1, 6144, 1.0), (37, 256, 1e-3), (16, 6144, 20.0), (3, 1056, 1e4)])
def test_q8_0_bitexact(rows, cols, scale):
    rng = np.random.default_rng(rows * cols)
    x = (rng.standard_normal((rows, cols)) * scale).astype(np.float32)
    x[0, :32] = 0.0                       # zero block
    x[-1, 32:64] = np.float32(1e-39)      # subnormal block
    x[0, 64:96] = np.arange(32, dtype=np.float32) - 15.5  # .5 ties after scaling
    q, d = moe.quantize_act_q8_0(torch.from_numpy(x).cuda())
    qo, do = orc.q8_0_quantize(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(d.cpu().numpy().view(np.uint32), do.view(np.uint32))


def test_q8_0_golden_on_gpu():
    import json, os
    doc = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "q8_0_blocks.json")))
    x = np.array([b["x"] for b in doc["blocks"]], np.float32).reshape(1, -1)
    q, d = moe.quantize_act_q8_0(torch.from_numpy(x).cuda())
    for i, b in enumerate(doc["blocks"]):
        assert float(d[0, i]) == np.float32(b["d"])
        np.testing.assert_array_equal(q[0, 32 * i:32 * (i + 1)].cpu().numpy(), np.array(b["q"], np.int8))


@pytest.mark.parametrize("wbits", [8, 4, 2])
@pytest.mark.parametrize("rows,cols", [(2048, 6144), (77, 96), (5, 2048)])
def test_pack_weights_bitexact(wbits, rows, cols):
    w = synth.normal(9, 1000 + wbits, rows * cols, 0.02).reshape(rows, cols)
    w[1] = 0.0
    if rows > 3:
        w[3, 5] = 0.5  # one outlier row
    p, s = moe.pack_weights(torch.from_numpy(w).cuda(), wbits)
    po, so = orc.quantize_rows(w, wbits)
    np.testing.assert_array_equal(p.cpu().numpy(), po)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("wbits", [8, 4, 2])
@pytest.mark.parametrize("rows,cols,n", [(64, 6144, 1), (33, 1056, 5), (200, 2048, 3)])
def test_block_dots_bitexact(wbits, rows, cols, n):
    rng = np.random.default_rng(rows + cols + wbits)
    w = synth.normal(3, 5000 + wbits, rows * cols, 0.02).reshape(rows, cols)
    po, _ = orc.quantize_rows(w, wbits)
    q = rng.integers(-127, 128, size=(n, cols)).astype(np.int8)
    q[0, :32] = 127
    q[-1, -32:] = -127
    got = moe.block_dots(torch.from_numpy(po).cuda(), cols, wbits, torch.from_numpy(q).cuda())
    np.testing.assert_array_equal(got.cpu().numpy(), orc.block_dots(po, cols, wbits, q))


def _router_case(name, T):
    wl = synth.WORKLOADS[name].with_tokens(T)
    return wl, synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)


@pytest.mark.parametrize("name,T", [("tiny_h256_e16_int8_t4", 4), ("tiny_h256_e16_int8_t4", 133),
                                    ("glm52_decode_int4_t1", 1), ("glm52_verify_int4_t4", 4),
                                    ("glm52_int8_t16_outliers", 16), ("glm52_prefill_int4_t512_zipf", 512),
                                    ("glm52_decode_int4_t1_topp07", 1), ("glm52_decode_int4_t1_topp07", 64)])
def test_router_bitexact(name, T):
    wl, x, Wr, bias = _router_case(name, T)
    s = wl.shape
    cfg = moe.config(s)
    idx, w = moe.router_select(cfg, torch.from_numpy(x).cuda(), torch.from_numpy(Wr).cuda(),
                               torch.from_numpy(bias).cuda())
    io, wo, c, gs = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf, want_scores=True,
                               topp=s.topp)
    got = idx.cpu().numpy()
    # The logits are summed in different orders on the two sides (oracle: fp64;
    # GPU: compensated fp32 pairs, ~2^-48 relative); only candidates closer than
    # ~1e-12 could swap.  A seed that close would be degenerate.
    top = -np.sort(-c, axis=1)[:, : s.top_k + 1]
    gtop = -np.sort(-gs, axis=1)[:, : s.topk_groups + 1]
    margin = min(np.abs(np.diff(top, axis=1)).min(), np.abs(np.diff(gtop, axis=1)).min())
    if 0 < s.topp < 1:  # the top-p's decision: the running shares against topp
        i0, _ = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf)
        sig = 1.0 / (1.0 + np.exp(-(x.astype(np.float64) @ Wr.astype(np.float64).T)))
        for t in range(T):
            q = np.sort(sig[t, i0[t]])[::-1] / sig[t, i0[t]].sum()
            margin = min(margin, np.abs(np.cumsum(q) - s.topp).min())
    if margin < 1e-10:
        pytest.skip(f"degenerate seed: selection margin {margin:.3g}")
    np.testing.assert_array_equal(got, io)
    np.testing.assert_allclose(w.cpu().numpy(), wo, rtol=1e-6)


@pytest.mark.parametrize("T,k,E,drop", [(1, 8, 256, 0.0), (4, 2, 16, 0.0), (37, 8, 256, 0.0), (512, 8, 256, 0.0),
                                        (3000, 8, 256, 0.0), (0, 8, 256, 0.0), (37, 8, 256, 0.3), (5, 4, 16, 0.5)])
def test_bucket_bitexact(T, k, E, drop):
    rng = np.random.default_rng(T + E)
    rows = [rng.choice(E, size=k, replace=False) for _ in range(T)]
    idx = (np.stack(rows) if rows else np.zeros((0, k))).astype(np.int32).reshape(T, k)
    if drop:  # pairs the adaptive top-p dropped
        idx[rng.random(idx.shape) < drop] = -1
    shape = synth.LayerShape(256, 128, E, 8 if E >= 16 else 2, 4 if E >= 16 else 1, k, 1, 1.0, 4)
    cfg = moe.config(shape)
    counts, offsets, perm = moe.bucket_tokens(cfg, torch.from_numpy(idx).cuda() if T else
                                              torch.zeros((0, k), dtype=torch.int32, device="cuda"))
    co, oo, po = orc.bucket(idx, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), co)
    np.testing.assert_array_equal(offsets.cpu().numpy(), oo)
    np.testing.assert_array_equal(perm.cpu().numpy(), po)


def _fp8_case(rng, rows, cols, block):
    w8 = rng.integers(0, 256, size=(rows, cols), dtype=np.uint8)
    w8[(w8 & 0x7F) == 0x7F] = 0x3A  # no NaN codes
    nb = (-(-rows // block), -(-cols // block))
    bs = (np.exp2(rng.uniform(-12, -4, size=nb)) * rng.uniform(0.5, 1.0, size=nb)).astype(np.float32)
    return w8, bs


@pytest.mark.parametrize("wbits", [8, 4, 2])
@pytest.mark.parametrize("rows,cols,block", [(2048, 6144, 128), (6144, 2048, 128), (200, 1056, 128), (37, 96, 32)])
def test_requant_fp8_bitexact(wbits, rows, cols, block):
    """The converter step: FP8 E4M3 with block scales -> packed codes and row
    scales, bit-exact against the oracle (a full GLM-5.2 gate/up and down
    matrix, a ragged last block, a block smaller than the checkpoint's)."""
    rng = np.random.default_rng(rows + cols + wbits + block)
    w8, bs = _fp8_case(rng, rows, cols, block)
    packed, scales = moe.requant_fp8(torch.from_numpy(w8).cuda(), torch.from_numpy(bs).cuda(), block, wbits)
    po, so = orc.requant_fp8(w8, bs, block, wbits)
    np.testing.assert_array_equal(packed.cpu().numpy(), po)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint32), so.view(np.uint32))


def test_requant_fp8_every_code():
    """Each of the 254 finite codes, one row per block scale of 1.0 and 2^-7:
    the row scales and int8 codes agree with the oracle bit for bit."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    row = np.zeros(256, np.uint8)
    row[: len(codes)] = codes
    w8 = np.tile(row, (256, 1))  # rows 0..127 in block row 0, rows 128..255 in block row 1
    bs = np.array([[1.0, 1.0], [2.0 ** -7, 2.0 ** -7]], np.float32)
    packed, scales = moe.requant_fp8(torch.from_numpy(np.ascontiguousarray(w8)).cuda(), torch.from_numpy(bs).cuda(), 128, 8)
    po, so = orc.requant_fp8(w8, bs, 128, 8)
    np.testing.assert_array_equal(packed.cpu().numpy(), po)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint32), so.view(np.uint32))
