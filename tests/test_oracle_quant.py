"""Pins of the oracle's quantisers and packers (CPU only).

Each check is fixed by something other than the oracle's own formula: values
worked by hand in tests/golden/, exhaustive round trips over every code and
byte, and error bounds that follow from rounding to nearest.
"""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_q8_0_golden_blocks(orc):
    doc = _load("q8_0_blocks.json")
    x = np.array([b["x"] for b in doc["blocks"]], np.float32).reshape(-1)
    q, d = orc.q8_0_quantize(x.reshape(1, -1))
    for i, b in enumerate(doc["blocks"]):
        assert d[0, i] == np.float32(b["d"]), b["note"]
        np.testing.assert_array_equal(q[0, 32 * i:32 * (i + 1)], np.array(b["q"], np.int8), err_msg=b["note"])


def test_q8_0_bounds_random(orc):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((64, 512)) * rng.uniform(1e-3, 1e3, size=(64, 1))).astype(np.float32)
    x[3, 64:96] = 0.0
    q, d = orc.q8_0_quantize(x)
    xb = x.reshape(64, -1, 32).astype(np.float64)
    qb = q.reshape(64, -1, 32).astype(np.float64)
    db = d.astype(np.float64)[..., None]
    assert np.all(np.abs(qb) <= 127)
    err = np.abs(xb - db * qb)
    # round to nearest of x*id with id ~ 1/d: |x - d q| <= d/2 up to a few ulp
    assert np.all(err <= db * (0.5 + 1e-5))
    # the element holding the block maximum maps to +-127
    amax_pos = np.abs(xb).argmax(axis=-1)
    top = np.take_along_axis(qb, amax_pos[..., None], -1)[..., 0]
    nz = db[..., 0] > 0
    assert np.all(np.abs(top[nz]) == 127)
    # a block of zeros has d = 0 and q = 0
    assert d[3, 2] == 0.0
    assert np.all(q[3, 64:96] == 0)


def test_q8_0_rejects_nonfinite_and_ragged(orc):
    x = np.zeros((1, 32), np.float32)
    x[0, 5] = np.inf
    with pytest.raises(ValueError):
        orc.q8_0_quantize(x)
    with pytest.raises(ValueError):
        orc.q8_0_quantize(np.zeros((1, 33), np.float32))


def test_pack_golden(orc):
    doc = _load("packing.json")
    for wbits, key in ((4, "int4"), (2, "int2")):
        for case in doc[key]:
            codes = np.array(case["codes"], np.int8)
            packed = orc.pack_codes(codes, wbits)
            np.testing.assert_array_equal(packed, np.array(case["bytes"], np.uint8), err_msg=str(case))
            np.testing.assert_array_equal(orc.unpack_codes(packed, codes.size, wbits), codes)


def test_quantize_rows_golden(orc):
    doc = _load("packing.json")
    for case in doc["rows"]:
        w = np.array(case["w"], np.float32).reshape(1, -1)
        packed, scales = orc.quantize_rows(w, case["wbits"])
        assert scales[0] == np.float32(case["scale"]), case["note"]
        codes = orc.unpack_codes(packed.reshape(-1), w.shape[1], case["wbits"])
        np.testing.assert_array_equal(codes, np.array(case["codes"], np.int8), err_msg=case["note"])


@pytest.mark.parametrize("wbits,lo,hi", [(4, -8, 7), (2, -2, 1), (8, -128, 127)])
def test_pack_roundtrip_exhaustive(orc, wbits, lo, hi):
    per = 8 // wbits
    # every code value in every position of a byte
    vals = np.arange(lo, hi + 1, dtype=np.int8)
    grid = np.stack(np.meshgrid(*([vals] * per), indexing="ij"), -1).reshape(-1)
    packed = orc.pack_codes(grid, wbits)
    np.testing.assert_array_equal(orc.unpack_codes(packed, grid.size, wbits), grid)
    # every byte pattern unpacks and repacks to itself
    allbytes = np.arange(256, dtype=np.uint8)
    codes = orc.unpack_codes(allbytes, 256 * per, wbits)
    assert codes.min() >= lo and codes.max() <= hi
    np.testing.assert_array_equal(orc.pack_codes(codes, wbits), allbytes)
    # position check against numpy bit extraction of the byte values
    if wbits < 8:
        fields = (allbytes[:, None].astype(np.int32) >> (wbits * np.arange(per))) & ((1 << wbits) - 1)
        signed = np.where(fields >= (1 << (wbits - 1)), fields - (1 << wbits), fields)
        np.testing.assert_array_equal(codes.reshape(256, per), signed)


@pytest.mark.parametrize("wbits,qmax", [(8, 127), (4, 7), (2, 1)])
def test_quantize_rows_bounds(orc, wbits, qmax):
    rng = np.random.default_rng(wbits)
    w = (rng.standard_normal((40, 96)) * 0.02).astype(np.float32)
    w[5] = 0.0
    packed, s = orc.quantize_rows(w, wbits)
    assert packed.shape == (40, 96 * wbits // 8)
    codes = orc.unpack_codes(packed.reshape(-1), w.size, wbits).reshape(w.shape).astype(np.float64)
    assert np.all(codes <= qmax) and np.all(codes >= -qmax)
    s64 = s.astype(np.float64)[:, None]
    assert np.all(np.abs(w - s64 * codes) <= s64 * (0.5 + 1e-5))
    amax = np.abs(w).max(axis=1)
    np.testing.assert_allclose(s, amax / qmax, rtol=1e-6)
    assert s[5] == 0 and np.all(codes[5] == 0)
    top = codes[np.arange(40), np.abs(w).argmax(axis=1)]
    assert np.all(np.abs(top[np.arange(40) != 5]) == qmax)
