"""Seeded synthetic inputs for the MoE layer (no arithmetic of the method here).

Every tensor is a pure function of ``(seed, tensor id, element index)`` through
a counter-based SplitMix64 generator (Steele, Lea and Flood, OOPSLA 2014).  The
host side is numpy (small tensors) or the C helper ``libsynth_host.so`` (large
ones); the CUDA library holds a device copy of the same generator so that the
multi-GB expert weights of the GLM-5.2-shape layer can be drawn in HBM.  Both
sides produce identical bits, which the tests check.

Value recipes (the pages run a real GLM-5.2 checkpoint; no weights exist here,
so these seeded tensors stand in for them):

* "normal(sigma)": Irwin-Hall sum of twelve 16-bit uniforms, centred, times
  sigma -- mean 0, variance sigma^2, tails cut at 6 sigma.  Exact integer
  arithmetic up to one fp32 multiply, so host and device agree bit for bit.
* "uniform(lo, lo+width)": 24-bit uniform, one fp32 multiply and one add.
* activations x ~ normal(1); router weight ~ normal(0.02); expert weights
  ~ normal(0.02); correction bias ~ uniform(-0.1, 0.1).
* speculative-verify batch: x_t = sqrt(0.8) z_0 + sqrt(0.2) z_t (pairwise
  correlation 0.8 between the 1 + 3 draft positions).
* int8 small batch: 1% of the hidden channels (61 of 6144, a seeded choice)
  are scaled by 20 in every token.
* prefill: bias_e = -1.1 * alpha * ln(rank_e) with ranks a seeded permutation
  of 1..E, i.e. alpha * ln(p_e / p_max) for Zipf(1.1) popularity p_e.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, replace

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB

# Tensor ids (stream numbers) of the generator.
TID_X = 1
TID_X_COMMON = 2
TID_ROUTER_W = 3
TID_BIAS = 4
TID_OUTLIERS = 5
TID_ZIPF_RANKS = 6
TID_EXPERT_BASE = 1000  # + 4 * expert + matrix (0 gate, 1 up, 2 down); shared experts follow the routed ones

MAT_GATE, MAT_UP, MAT_DOWN = 0, 1, 2

# Calibrated once so that the realised per-expert token counts of the prefill
# workload fall off with a log-log slope close to -1.1 (checked by a test).
ZIPF_ALPHA = 0.133


def _mix_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * _M1) & MASK64
    z = ((z ^ (z >> 27)) * _M2) & MASK64
    return z ^ (z >> 31)


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tid: int) -> int:
    """Output number ``tid`` of the SplitMix64 stream seeded with ``seed``."""
    return _mix_int((seed + (tid + 1) * GAMMA) & MASK64)


def words(seed: int, tid: int, n0: int, n: int) -> np.ndarray:
    """Outputs n0 .. n0+n-1 of the stream seeded with ``stream_key(seed, tid)``."""
    key = np.uint64(stream_key(seed, tid))
    idx = np.arange(n0, n0 + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix_np(key + (idx + np.uint64(1)) * np.uint64(GAMMA))


def normal(seed: int, tid: int, n: int, sigma: float, offset: int = 0, backend: str = "auto") -> np.ndarray:
    """fp32 normal-like values (Irwin-Hall 12) for elements offset..offset+n-1.

    backend: "auto" (C helper for large n), "numpy" or "c".
    """
    lib = _host_lib() if backend != "numpy" else None
    if backend == "c" and lib is None:
        raise RuntimeError("libsynth_host.so is not available")
    out = np.empty(n, dtype=np.float32)
    if lib is not None and (n > 4096 or backend == "c"):
        lib.synth_normal(ctypes.c_uint64(seed), ctypes.c_uint64(tid), ctypes.c_int64(offset),
                         ctypes.c_int64(n), ctypes.c_float(sigma),
                         out.ctypes.data_as(ctypes.c_void_p))
        return out
    w = words(seed, tid, 3 * offset, 3 * n).reshape(n, 3)
    s = np.zeros(n, dtype=np.int64)
    for sh in (0, 16, 32, 48):
        s += ((w >> np.uint64(sh)) & np.uint64(0xFFFF)).astype(np.int64).sum(axis=1)
    z = (s - 393210).astype(np.float32) / np.float32(65536.0)
    out[:] = z * np.float32(sigma)
    return out


def uniform(seed: int, tid: int, n: int, lo: float, width: float, offset: int = 0) -> np.ndarray:
    """fp32 values f*width + lo with f a 24-bit uniform in [0, 1)."""
    w = words(seed, tid, offset, n)
    f = (w >> np.uint64(40)).astype(np.float32) * np.float32(2.0 ** -24)
    return (f * np.float32(width)) + np.float32(lo)


def permutation(seed: int, tid: int, n: int) -> np.ndarray:
    """Seeded Fisher-Yates shuffle of 0..n-1 (word i picks the swap for position n-1-i)."""
    w = words(seed, tid, 0, max(n - 1, 0))
    p = np.arange(n, dtype=np.int64)
    for i in range(n - 1, 0, -1):
        j = int(w[n - 1 - i] % np.uint64(i + 1))
        p[i], p[j] = p[j], p[i]
    return p


# ----------------------------------------------------------------------------
# Layer shapes and workloads
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class LayerShape:
    hidden: int
    inter: int
    n_experts: int
    n_groups: int
    topk_groups: int
    top_k: int
    n_shared: int
    rsf: float
    wbits: int
    topp: float = 0.0  # adaptive expert top-p in (0, 1); 0 keeps all top_k picks

    def matrix_bytes(self, rows: int, cols: int) -> int:
        return rows * cols * self.wbits // 8

    @property
    def expert_bytes(self) -> int:
        """Weight bytes plus row-scale bytes of one expert (gate, up, down)."""
        h, i = self.hidden, self.inter
        return 2 * self.matrix_bytes(i, h) + self.matrix_bytes(h, i) + 4 * (2 * i + h)


@dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    T: int
    seed: int
    x_kind: str = "normal"      # normal | correlated | outliers
    bias_kind: str = "uniform"  # uniform | zipf
    description: str = ""

    def with_tokens(self, T: int) -> "Workload":
        return replace(self, T=T)


GLM_INT4 = LayerShape(6144, 2048, 256, 8, 4, 8, 1, 2.5, 4)
GLM_INT8 = replace(GLM_INT4, wbits=8)
GLM_INT2 = replace(GLM_INT4, wbits=2)
TINY = LayerShape(256, 128, 16, 4, 2, 2, 1, 2.5, 8)

WORKLOADS = {
    "tiny_h256_e16_int8_t4": Workload(
        "tiny_h256_e16_int8_t4", TINY, 4, 0,
        description="hidden 256, intermediate 128, 16 experts in 4 groups, top-2 groups, top-2 + 1 shared, int8, 4 tokens"),
    "glm52_decode_int4_t1": Workload(
        "glm52_decode_int4_t1", GLM_INT4, 1, 1,
        description="GLM-5.2 shape (6144/2048, 256 experts, 8 groups, top-4 groups, top-8 + 1 shared), int4, 1 token"),
    "glm52_decode_int4_t1_topp07": Workload(
        "glm52_decode_int4_t1_topp07", replace(GLM_INT4, topp=0.7), 1, 1,
        description="glm52_decode_int4_t1 with the adaptive expert top-p at 0.7 (the kept picks' shares reach 0.7)"),
    "glm52_decode_int2_t1": Workload(
        "glm52_decode_int2_t1", GLM_INT2, 1, 1,
        description="glm52_decode_int4_t1 with packed int2 experts (codes -2..1, per-row scale amax/1): 9.46 MB per expert"),
    "glm52_verify_int4_t4": Workload(
        "glm52_verify_int4_t4", GLM_INT4, 4, 2, x_kind="correlated",
        description="GLM-5.2 shape, int4, 4 tokens (1 + 3 drafts) with 0.8-correlated activations"),
    "glm52_int8_t16_outliers": Workload(
        "glm52_int8_t16_outliers", GLM_INT8, 16, 3, x_kind="outliers",
        description="GLM-5.2 shape, int8, 16 tokens, 1% outlier channels x20"),
    "glm52_prefill_int4_t512_zipf": Workload(
        "glm52_prefill_int4_t512_zipf", GLM_INT4, 512, 4, bias_kind="zipf",
        description="GLM-5.2 shape, int4, 512 tokens, Zipf(1.1) expert popularity through the correction bias"),
}
WORKLOAD_ORDER = list(WORKLOADS)


def expert_tid(shape: LayerShape, expert: int, mat: int, shared: bool = False) -> int:
    e = expert + (shape.n_experts if shared else 0)
    return TID_EXPERT_BASE + 4 * e + mat


def matrix_dims(shape: LayerShape, mat: int) -> tuple[int, int]:
    """(rows, cols) of an expert matrix: gate/up are [inter][hidden], down is [hidden][inter]."""
    if mat == MAT_DOWN:
        return shape.hidden, shape.inter
    return shape.inter, shape.hidden


def make_x(wl: Workload) -> np.ndarray:
    H, T = wl.shape.hidden, wl.T
    if wl.x_kind == "normal":
        return normal(wl.seed, TID_X, T * H, 1.0).reshape(T, H)
    if wl.x_kind == "correlated":
        z0 = normal(wl.seed, TID_X_COMMON, H, 1.0)
        zt = normal(wl.seed, TID_X, T * H, 1.0).reshape(T, H)
        a, b = np.float32(np.sqrt(0.8)), np.float32(np.sqrt(0.2))
        return (a * z0[None, :]) + (b * zt)
    if wl.x_kind == "outliers":
        x = normal(wl.seed, TID_X, T * H, 1.0).reshape(T, H)
        n_out = int(round(0.01 * H))
        ch = permutation(wl.seed, TID_OUTLIERS, H)[:n_out]
        x[:, ch] *= np.float32(20.0)
        return x
    raise ValueError(wl.x_kind)


def outlier_channels(wl: Workload) -> np.ndarray:
    H = wl.shape.hidden
    return np.sort(permutation(wl.seed, TID_OUTLIERS, H)[: int(round(0.01 * H))])


def make_router_w(wl: Workload) -> np.ndarray:
    s = wl.shape
    return normal(wl.seed, TID_ROUTER_W, s.n_experts * s.hidden, 0.02).reshape(s.n_experts, s.hidden)


def make_bias(wl: Workload) -> np.ndarray:
    E = wl.shape.n_experts
    if wl.bias_kind == "uniform":
        return uniform(wl.seed, TID_BIAS, E, -0.1, 0.2)
    if wl.bias_kind == "zipf":
        rank = permutation(wl.seed, TID_ZIPF_RANKS, E) + 1
        return (-1.1 * ZIPF_ALPHA * np.log(rank.astype(np.float64))).astype(np.float32)
    raise ValueError(wl.bias_kind)


def make_expert_matrix(wl: Workload, expert: int, mat: int, shared: bool = False) -> np.ndarray:
    rows, cols = matrix_dims(wl.shape, mat)
    return normal(wl.seed, expert_tid(wl.shape, expert, mat, shared), rows * cols, 0.02).reshape(rows, cols)


# ----------------------------------------------------------------------------
# Optional C accelerator for the host generator (same definition as above).
# ----------------------------------------------------------------------------
_HOST_LIB = None
_HOST_LIB_TRIED = False
_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB_PATH = os.path.join(_HERE, "libsynth_host.so")


def _host_lib():
    global _HOST_LIB, _HOST_LIB_TRIED
    if _HOST_LIB_TRIED:
        return _HOST_LIB
    _HOST_LIB_TRIED = True
    if not os.path.exists(HOST_LIB_PATH):
        try:
            build_host_lib()
        except Exception:  # numpy path still works, only slower
            return None
    lib = ctypes.CDLL(HOST_LIB_PATH)
    lib.synth_normal.restype = None
    lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_float, ctypes.c_void_p]
    lib.synth_words.restype = None
    lib.synth_words.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                ctypes.c_void_p]
    _HOST_LIB = lib
    return lib


def build_host_lib() -> str:
    import subprocess
    src = os.path.join(_HERE, "csrc", "synth_host.c")
    tmp = HOST_LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-std=c99",
                           "-shared", "-fPIC", "-o", tmp, src])
    os.replace(tmp, HOST_LIB_PATH)
    return HOST_LIB_PATH
