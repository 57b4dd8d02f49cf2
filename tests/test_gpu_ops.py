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


# The factor each routine's stored value carries (see moe_block_dots_routine).
DOT_FACTOR = {(moe.DOTS_MULTI_KERNEL, 8): 1, (moe.DOTS_MULTI_KERNEL, 4): 1, (moe.DOTS_MULTI_KERNEL, 2): 1,
              (moe.DOTS_FUSED, 8): 1, (moe.DOTS_FUSED, 4): 16, (moe.DOTS_FUSED, 2): 64,
              (moe.DOTS_TENSOR, 8): 1, (moe.DOTS_TENSOR, 4): 1, (moe.DOTS_TENSOR, 2): 1}


def _random_dot_inputs(wbits, rows, cols, n, seed):
    """Random packed bytes (every nibble / 2-bit field, including the codes -8
    and -2 that the quantiser never writes) and int8 codes in [-127, 127] with
    saturated blocks: rows 0-1 all -8 / -2 codes, row 2 all +7 / +1, block 0 of
    token 0 all +127, the last block of the last token all -127, one block
    alternating +-127."""
    rng = np.random.default_rng(seed)
    packed = rng.integers(0, 256, size=(rows, cols * wbits // 8), dtype=np.uint8)
    lowest = {8: 0x80, 4: 0x88, 2: 0xAA}[wbits]
    highest = {8: 0x7F, 4: 0x77, 2: 0x55}[wbits]
    packed[0] = lowest
    packed[1 % rows] = lowest
    packed[2 % rows] = highest
    q = rng.integers(-127, 128, size=(n, cols)).astype(np.int8)
    q[0, :32] = 127
    q[-1, -32:] = -127
    if cols >= 96:
        q[0, 64:96] = np.where(np.arange(32) % 2 == 0, 127, -127)
    return packed, q


@pytest.mark.parametrize("routine", [moe.DOTS_MULTI_KERNEL, moe.DOTS_FUSED])
@pytest.mark.parametrize("wbits", [8, 4, 2])
@pytest.mark.parametrize("rows,cols,n", [(48, 6144, 2), (37, 2048, 4), (5, 96, 3)])
def test_dot_routines_random_bytes(routine, wbits, rows, cols, n):
    """Each device dot routine the kernels call, bit-exact against the oracle's
    brute-force block dots on arbitrary packed bytes; the fused routine's
    scaled value is checked as the exact product first."""
    packed, q = _random_dot_inputs(wbits, rows, cols, n, seed=rows * 7 + cols + wbits + 100 * routine)
    ref = orc.block_dots(packed, cols, wbits, q).astype(np.int64)
    got = moe.block_dots(torch.from_numpy(packed).cuda(), cols, wbits, torch.from_numpy(q).cuda(),
                         routine=routine).cpu().numpy().astype(np.int64)
    f = DOT_FACTOR[(routine, wbits)]
    np.testing.assert_array_equal(got, f * ref)
    np.testing.assert_array_equal(got // f, ref)
    # the saturated rows reach the extremes the routines must carry exactly
    assert np.abs(ref).max() >= 32 * 127 * {8: 128, 4: 8, 2: 2}[wbits] // 2


@pytest.mark.parametrize("wbits", [8, 4, 2])
@pytest.mark.parametrize("rows,cols,n", [(128, 128, 16), (300, 6144, 64), (77, 2048, 17), (200, 192, 1),
                                         (129, 320, 48)])
def test_tensor_dot_routine_random_bytes(wbits, rows, cols, n):
    """The tensor-core routine (widening in shared memory, one kind::i8 MMA per
    Q8_0 block, int32 read back from TMEM), bit-exact against the oracle on
    arbitrary packed bytes: ragged row tiles (77, 129, 300 rows), partial
    last stages (192, 320 codes), token counts that are not multiples of 16."""
    if (cols * wbits // 8) % 16:
        pytest.skip("rows of the tensor routine are multiples of 16 bytes")
    packed, q = _random_dot_inputs(wbits, rows, cols, n, seed=rows * 11 + cols + wbits + n)
    ref = orc.block_dots(packed, cols, wbits, q)
    got = moe.block_dots(torch.from_numpy(packed).cuda(), cols, wbits, torch.from_numpy(q).cuda(),
                         routine=moe.DOTS_TENSOR).cpu().numpy()
    np.testing.assert_array_equal(got, ref)


def test_tensor_dot_routine_limits():
    p = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    q = torch.zeros((65, 128), dtype=torch.int8, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.block_dots(p, 128, 4, q, routine=moe.DOTS_TENSOR)  # more than 64 tokens
    p2 = torch.zeros((4, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.block_dots(p2, 32, 2, q[:1, :32].contiguous(), routine=moe.DOTS_TENSOR)  # 8-byte rows


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
