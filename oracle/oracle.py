"""ctypes binding of the C oracle (moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the package smoke check and by
the CPU-baseline leg of bench.py.  The product path never imports it.

Each function is a thin marshalling wrapper around one C function; the
arithmetic, and the citations of the pages each step follows, live in the C
file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.c")
LIB_PATH = os.path.join(HERE, "libmoe_oracle.so")

ORC_OK, ORC_EINVAL, ORC_ENONFINITE, ORC_EMISSING = 0, -1, -2, -3

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_flt = ctypes.c_float


def build(force: bool = False) -> str:
    """Compile the oracle (plain C99, separately rounded fp ops, OpenMP rows)."""
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC):
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-std=c99",
                           "-Wall", "-shared", "-fPIC", "-o", tmp, SRC, "-lm"])
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


class _OrcExpert(ctypes.Structure):
    _fields_ = [("wg", _vp), ("wu", _vp), ("wd", _vp), ("sg", _vp), ("su", _vp), ("sd", _vp)]


_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        L = ctypes.CDLL(build())
        sig = {
            "orc_q8_0_quantize": [_vp, _i64, _vp, _vp],
            "orc_pack_codes": [_vp, _i64, _int, _vp],
            "orc_unpack_codes": [_vp, _i64, _int, _vp],
            "orc_quantize_rows": [_vp, _i64, _i64, _int, _vp, _vp],
            "orc_block_dots": [_vp, _i64, _i64, _int, _vp, _i64, _vp],
            "orc_qmatvec": [_vp, _vp, _i64, _i64, _int, _vp, _vp, _vp],
            "orc_router": [_vp, _int, _int, _vp, _vp, _int, _int, _int, _int, _flt, _vp, _vp, _vp, _vp],
            "orc_router_topp": [_vp, _int, _int, _vp, _vp, _int, _int, _int, _int, _flt, _flt,
                                _vp, _vp, _vp, _vp],
            "orc_bucket": [_vp, _int, _int, _int, _vp, _vp, _vp],
            "orc_expert_ffn": [ctypes.POINTER(_OrcExpert), _int, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp],
            "orc_layer_forward": [_int, _int, _int, _int, _int, _int, _int, _flt, _int,
                                  _vp, _int, _vp, _vp, ctypes.POINTER(_OrcExpert), ctypes.POINTER(_OrcExpert),
                                  _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
            "orc_layer_forward_topp": [_int, _int, _int, _int, _int, _int, _int, _flt, _int, _flt,
                                       _vp, _int, _vp, _vp, ctypes.POINTER(_OrcExpert),
                                       ctypes.POINTER(_OrcExpert), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
            "orc_fp8_e4m3_decode": [_vp, _i64, _vp],
            "orc_requant_fp8": [_vp, _vp, _i64, _i64, _int, _int, _vp, _vp],
            "orc_num_threads": [],
            "orc_set_num_threads": [_int],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = None if name == "orc_set_num_threads" else _int
        _LIB = L
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(_vp)


def _check(rc: int, what: str):
    if rc != ORC_OK:
        raise ValueError(f"oracle {what} failed with status {rc}")


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().orc_num_threads()


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


def q8_0_quantize(x):
    x = _c(x, np.float32)
    n = x.size
    q = np.empty(x.shape, np.int8)
    d = np.empty(x.shape[:-1] + (x.shape[-1] // 32,), np.float32)
    _check(lib().orc_q8_0_quantize(_p(x), n, _p(q), _p(d)), "q8_0_quantize")
    return q, d


def pack_codes(codes, wbits: int):
    codes = _c(codes, np.int8)
    out = np.empty(codes.size * wbits // 8, np.uint8)
    _check(lib().orc_pack_codes(_p(codes), codes.size, wbits, _p(out)), "pack_codes")
    return out


def unpack_codes(packed, n: int, wbits: int):
    packed = _c(packed, np.uint8)
    out = np.empty(n, np.int8)
    _check(lib().orc_unpack_codes(_p(packed), n, wbits, _p(out)), "unpack_codes")
    return out


def quantize_rows(w, wbits: int):
    """Per-row quantise and pack: returns (packed [rows][cols*wbits/8] uint8, scales [rows] fp32)."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    packed = np.empty((rows, cols * wbits // 8), np.uint8)
    scales = np.empty(rows, np.float32)
    _check(lib().orc_quantize_rows(_p(w), rows, cols, wbits, _p(packed), _p(scales)), "quantize_rows")
    return packed, scales


def block_dots(packed, cols: int, wbits: int, q):
    """int32 per-block dots [n_tok][rows][cols/32] of a packed matrix with int8 vectors q [n_tok][cols]."""
    packed = _c(packed, np.uint8)
    q = _c(q, np.int8).reshape(-1, cols)
    rows = packed.shape[0]
    out = np.empty((q.shape[0], rows, cols // 32), np.int32)
    _check(lib().orc_block_dots(_p(packed), rows, cols, wbits, _p(q), q.shape[0], _p(out)), "block_dots")
    return out


def qmatvec(packed, scales, cols: int, wbits: int, q, d):
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.float32)
    q = _c(q, np.int8)
    d = _c(d, np.float32)
    y = np.empty(packed.shape[0], np.float32)
    _check(lib().orc_qmatvec(_p(packed), _p(scales), packed.shape[0], cols, wbits, _p(q), _p(d), _p(y)), "qmatvec")
    return y


def router(x, Wr, bias, n_groups: int, topk_groups: int, top_k: int, rsf: float, want_scores: bool = False,
           topp: float = 0.0):
    """Routing of every token: idx, w [T][top_k] (with topp in (0, 1), dropped
    picks have idx -1 and w 0)."""
    x = _c(x, np.float32)
    Wr = _c(Wr, np.float32)
    bias = _c(bias, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float32)
    c = np.empty((T, E), np.float64) if want_scores else None
    gs = np.empty((T, n_groups), np.float64) if want_scores else None
    _check(lib().orc_router_topp(_p(x), T, H, _p(Wr), _p(bias), E, n_groups, topk_groups, top_k, rsf, topp,
                                 _p(idx), _p(w), _p(c), _p(gs)), "router")
    if want_scores:
        return idx, w, c, gs
    return idx, w


def bucket(idx, n_experts: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(n_experts, np.int32)
    offsets = np.empty(n_experts + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    _check(lib().orc_bucket(_p(idx), T, k, n_experts, _p(counts), _p(offsets), _p(perm)), "bucket")
    return counts, offsets, perm


def fp8_e4m3_decode(codes):
    codes = _c(codes, np.uint8)
    out = np.empty(codes.shape, np.float32)
    _check(lib().orc_fp8_e4m3_decode(_p(codes), codes.size, _p(out)), "fp8_e4m3_decode")
    return out


def requant_fp8(w8, block_scales, block: int, wbits: int):
    """FP8 E4M3 [rows][cols] with [ceil(rows/block)][ceil(cols/block)] fp32
    scales -> (packed [rows][cols*wbits/8], row scales [rows])."""
    w8 = _c(w8, np.uint8)
    block_scales = _c(block_scales, np.float32)
    rows, cols = w8.shape
    packed = np.empty((rows, cols * wbits // 8), np.uint8)
    scales = np.empty(rows, np.float32)
    _check(lib().orc_requant_fp8(_p(w8), _p(block_scales), rows, cols, block, wbits, _p(packed), _p(scales)),
           "requant_fp8")
    return packed, scales


@dataclass
class PackedExpert:
    """Packed codes and fp32 row scales of one expert (gate, up: [inter][hidden]; down: [hidden][inter])."""
    wg: np.ndarray
    wu: np.ndarray
    wd: np.ndarray
    sg: np.ndarray
    su: np.ndarray
    sd: np.ndarray

    def as_struct(self) -> _OrcExpert:
        return _OrcExpert(_p(self.wg), _p(self.wu), _p(self.wd), _p(self.sg), _p(self.su), _p(self.sd))


def pack_expert(wg, wu, wd, wbits: int) -> PackedExpert:
    pg, sg = quantize_rows(wg, wbits)
    pu, su = quantize_rows(wu, wbits)
    pd, sd = quantize_rows(wd, wbits)
    return PackedExpert(pg, pu, pd, sg, su, sd)


def expert_ffn(ex: PackedExpert, H: int, I: int, wbits: int, xq, xd):
    """One expert on one token: returns (y [H], h [I], hq [I], hd [I/32])."""
    xq = _c(xq, np.int8)
    xd = _c(xd, np.float32)
    y = np.empty(H, np.float32)
    h = np.empty(I, np.float32)
    hq = np.empty(I, np.int8)
    hd = np.empty(I // 32, np.float32)
    st = ex.as_struct()
    _check(lib().orc_expert_ffn(ctypes.byref(st), H, I, wbits, _p(xq), _p(xd), _p(y), _p(h), _p(hq), _p(hd)),
           "expert_ffn")
    return y, h, hq, hd


@dataclass
class LayerTrace:
    out: np.ndarray
    idx: np.ndarray
    w: np.ndarray
    xq: np.ndarray
    xd: np.ndarray
    ys: np.ndarray   # [T][k+n_shared][H] per-slot expert outputs (slot k = shared)
    hq: np.ndarray   # [T][k+n_shared][I]
    hd: np.ndarray   # [T][k+n_shared][I/32]


def layer_forward(shape, x, Wr, bias, routed: dict, shared: PackedExpert | None) -> LayerTrace:
    """Full layer forward.  ``routed`` maps expert id -> PackedExpert (experts that
    are never selected may be left out; selecting one raises)."""
    x = _c(x, np.float32)
    Wr = _c(Wr, np.float32)
    bias = _c(bias, np.float32)
    T, H = x.shape
    I, E, k, ns = shape.inter, shape.n_experts, shape.top_k, shape.n_shared
    S = k + ns
    arr = (_OrcExpert * E)()
    for e, ex in routed.items():
        arr[e] = ex.as_struct()
    sh = shared.as_struct() if shared is not None else _OrcExpert()
    out = np.empty((T, H), np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    xq = np.empty((T, H), np.int8)
    xd = np.empty((T, H // 32), np.float32)
    ys = np.empty((T, S, H), np.float32)
    hq = np.empty((T, S, I), np.int8)
    hd = np.empty((T, S, I // 32), np.float32)
    topp = float(getattr(shape, "topp", 0.0))
    rc = lib().orc_layer_forward_topp(H, I, E, shape.n_groups, shape.topk_groups, k, ns, shape.rsf, shape.wbits,
                                      topp, _p(x), T, _p(Wr), _p(bias), arr, ctypes.byref(sh), _p(out),
                                      _p(idx), _p(w), _p(xq), _p(xd), _p(ys), _p(hq), _p(hd))
    _check(rc, "layer_forward")
    return LayerTrace(out, idx, w, xq, xd, ys, hq, hd)
