"""Pins of the oracle's FP8 requantiser (CPU only).

The converter step the pages describe: an FP8 checkpoint with 128 x 128
block scales is dequantised and requantised into per-row int8/int4/int2.
Fixed here by values of the E4M3 format worked out from its definition,
by torch's own float8_e4m3fn conversion over every code, by the block
indexing on a case whose dequantised values are exactly the block scales,
and by the composition with the separately pinned per-row quantiser on a
dequantisation computed with numpy.
"""
import numpy as np
import pytest
import torch


@pytest.mark.parametrize("code,value", [
    (0x38, 1.0),            # exponent 7 (bias 7), mantissa 0
    (0x3C, 1.5),            # mantissa 4/8
    (0x7E, 448.0),          # largest finite: (1 + 6/8) * 2^8
    (0xFE, -448.0),
    (0x08, 2.0 ** -6),      # smallest normal
    (0x01, 2.0 ** -9),      # smallest subnormal: 1/8 * 2^-6
    (0x07, 7 * 2.0 ** -9),  # largest subnormal
    (0x00, 0.0),
])
def test_fp8_known_values(orc, code, value):
    assert orc.fp8_e4m3_decode(np.array([code], np.uint8))[0] == np.float32(value)


def test_fp8_negative_zero_and_nan(orc):
    v = orc.fp8_e4m3_decode(np.array([0x80, 0x7F, 0xFF], np.uint8))
    assert v[0] == 0.0 and np.signbit(v[0])
    assert np.isnan(v[1]) and np.isnan(v[2])


def test_fp8_every_code_matches_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = orc.fp8_e4m3_decode(codes)
    finite = ~np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), ~finite)
    np.testing.assert_array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))


def _random_fp8(rng, rows, cols):
    codes = rng.integers(0, 256, size=(rows, cols), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3A  # no NaN codes
    return codes


def _block_scales(rng, rows, cols, block):
    nbr, nbc = -(-rows // block), -(-cols // block)
    return (np.exp2(rng.uniform(-12, -4, size=(nbr, nbc))) * rng.uniform(0.5, 1.0, size=(nbr, nbc))).astype(np.float32)


@pytest.mark.parametrize("wbits", [8, 4, 2])
@pytest.mark.parametrize("rows,cols,block", [(200, 1056, 128), (128, 256, 128), (37, 96, 32)])
def test_requant_is_quantise_of_block_dequant(orc, wbits, rows, cols, block):
    rng = np.random.default_rng(rows * 7 + cols + wbits)
    w8 = _random_fp8(rng, rows, cols)
    bs = _block_scales(rng, rows, cols, block)
    packed, scales = orc.requant_fp8(w8, bs, block, wbits)
    vals = torch.from_numpy(w8).view(torch.float8_e4m3fn).float().numpy()
    full = np.repeat(np.repeat(bs, block, axis=0), block, axis=1)[:rows, :cols]
    deq = (vals * full).astype(np.float32)  # one fp32 multiply per element
    ref_p, ref_s = orc.quantize_rows(deq, wbits)
    np.testing.assert_array_equal(packed, ref_p)
    np.testing.assert_array_equal(scales.view(np.uint32), ref_s.view(np.uint32))


def test_requant_block_indexing(orc):
    # every code is 1.0, so each dequantised value is its block's scale; the
    # row scale is the row's largest block scale / qmax, and int8 codes are
    # round(scale_of_block / row_scale)
    rows, cols, block = 256, 384, 128
    w8 = np.full((rows, cols), 0x38, np.uint8)
    bs = np.exp2(-np.arange(6, dtype=np.float32)).reshape(2, 3)  # 1, 1/2, ..., 1/32
    packed, scales = orc.requant_fp8(w8, bs, block, 8)
    np.testing.assert_array_equal(scales[:128], np.float32(1.0) / np.float32(127.0))
    np.testing.assert_array_equal(scales[128:], np.float32(0.125) / np.float32(127.0))
    codes = packed.view(np.int8)
    assert codes[0, 0] == 127 and codes[0, 128] == 64 and codes[0, 256] == 32
    assert codes[200, 0] == 127 and codes[200, 128] == 64 and codes[200, 256] == 32


def test_requant_rejects_nan_codes(orc):
    w8 = np.full((2, 32), 0x38, np.uint8)
    w8[1, 5] = 0x7F
    with pytest.raises(ValueError, match="status -2"):  # ORC_ENONFINITE
        orc.requant_fp8(w8, np.ones((1, 1), np.float32), 128, 4)
