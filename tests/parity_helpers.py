"""Shared set-up for the GPU-vs-oracle parity tests.

Both sides start from the same seeded fp32 tensors of the input generator; the
oracle packs the weights with its own C quantiser, the GPU with the library's
pack kernel, and the tests check the packed bytes agree before comparing any
output.  No oracle input or expected value comes from the CUDA path.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch

from oracle import oracle as orc
from quantized_routed_expert_group_b200 import moe, synth

# Tolerance on fp32 layer outputs: max |gpu - oracle| / rms(oracle).
OUT_TOL = 1e-3


def rel_rms_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.abs(got - ref).max() / rms) if rms > 0 else float(np.abs(got - ref).max())


@dataclass
class Pair:
    wl: synth.Workload
    x: np.ndarray
    router_w: np.ndarray
    bias: np.ndarray
    mats: dict               # expert -> (g, u, d) fp32
    shared_mats: tuple | None
    orc_routed: dict         # expert -> oracle PackedExpert
    orc_shared: object
    layer: moe.MoeLayer


def make_workload(name: str, shape: synth.LayerShape, T: int, seed: int, **kw) -> synth.Workload:
    return synth.Workload(name, shape, T, seed, **kw)


def build_pair(wl: synth.Workload, T_max: int | None = None, device="cuda", mutate=None) -> Pair:
    """mutate(mats, shared_mats), if given, edits the fp32 matrices (tuples
    of gate, up, down arrays) in place before either side packs them."""
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    mats = {e: tuple(synth.make_expert_matrix(wl, e, m) for m in range(3)) for e in range(s.n_experts)}
    shm = tuple(synth.make_expert_matrix(wl, 0, m, shared=True) for m in range(3)) if s.n_shared else None
    if mutate is not None:
        mutate(mats, shm)
    orc_routed = {e: orc.pack_expert(*mats[e], s.wbits) for e in range(s.n_experts)}
    orc_shared = orc.pack_expert(*shm, s.wbits) if shm else None
    routed = moe.bank_from_host_matrices(s, [mats[e] for e in range(s.n_experts)], device)
    shared = moe.bank_from_host_matrices(s, [shm], device) if shm else None
    layer = moe.MoeLayer(s, torch.from_numpy(Wr).to(device), torch.from_numpy(bias).to(device), routed, shared,
                         T_max or max(wl.T, 1))
    return Pair(wl, x, Wr, bias, mats, shm, orc_routed, orc_shared, layer)


def check_banks_equal(pair: Pair) -> None:
    """GPU-packed bytes and scales == oracle-packed, for every expert."""
    b = pair.layer.routed
    for e, ex in pair.orc_routed.items():
        np.testing.assert_array_equal(b.w_gate[e].cpu().numpy(), ex.wg)
        np.testing.assert_array_equal(b.w_up[e].cpu().numpy(), ex.wu)
        np.testing.assert_array_equal(b.w_down[e].cpu().numpy(), ex.wd)
        np.testing.assert_array_equal(b.s_gate[e].cpu().numpy().view(np.uint32), ex.sg.view(np.uint32))
        np.testing.assert_array_equal(b.s_up[e].cpu().numpy().view(np.uint32), ex.su.view(np.uint32))
        np.testing.assert_array_equal(b.s_down[e].cpu().numpy().view(np.uint32), ex.sd.view(np.uint32))
    if pair.orc_shared is not None:
        sh = pair.layer.shared
        np.testing.assert_array_equal(sh.w_gate[0].cpu().numpy(), pair.orc_shared.wg)
        np.testing.assert_array_equal(sh.w_down[0].cpu().numpy(), pair.orc_shared.wd)


def check_layer(pair: Pair, x: np.ndarray | None = None, check_intermediates: bool = True) -> dict:
    """Run GPU and oracle on the same tokens and compare.  Returns stats."""
    s = pair.wl.shape
    x = pair.x if x is None else x
    T = x.shape[0]
    xt = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    out = pair.layer.forward(xt)
    torch.cuda.synchronize()
    assert pair.layer.device_error() == 0
    tr = orc.layer_forward(s, x, pair.router_w, pair.bias, pair.orc_routed, pair.orc_shared)
    got = out.cpu().numpy()
    stats = {"out_err": rel_rms_err(got, tr.out) if T else 0.0}
    assert stats["out_err"] <= OUT_TOL, stats
    if not check_intermediates or T == 0:
        return stats
    v = {k: t.cpu().numpy() for k, t in pair.layer.view(T).items()}
    np.testing.assert_array_equal(v["xq"], tr.xq)
    np.testing.assert_array_equal(v["xd"].view(np.uint32), tr.xd.view(np.uint32))
    np.testing.assert_array_equal(v["idx"], tr.idx)
    np.testing.assert_allclose(v["w"], tr.w, rtol=1e-6)
    counts, offsets, perm = orc.bucket(tr.idx, s.n_experts)
    np.testing.assert_array_equal(v["counts"], counts)
    np.testing.assert_array_equal(v["offsets"], offsets)
    np.testing.assert_array_equal(v["perm"], perm)
    k, S = s.top_k, s.top_k + s.n_shared
    # slot p < n of the GPU holds pair perm[p] = t*k + j (n = routed pairs: the
    # top-p leaves slots n .. T*k-1 unused); shared slot T*k + t
    n = int(offsets[-1])
    live = perm[:n]
    t_of = np.concatenate([live // k, np.arange(T)]) if s.n_shared else live // k
    j_of = np.concatenate([live % k, np.full(T, k)]) if s.n_shared else live % k
    slots = np.concatenate([np.arange(n), T * k + np.arange(T)]) if s.n_shared else np.arange(n)
    v["hq"], v["y"] = v["hq"][slots], v["y"][slots]
    hq_ref = tr.hq[t_of, j_of]
    dq = np.abs(v["hq"].astype(np.int32) - hq_ref.astype(np.int32))
    assert dq.max() <= 1
    stats["hq_mismatch"] = float((dq != 0).mean())
    assert stats["hq_mismatch"] <= 0.01, stats
    ys_ref = tr.ys[t_of, j_of]
    stats["y_err"] = rel_rms_err(v["y"], ys_ref)
    assert stats["y_err"] <= OUT_TOL, stats
    return stats


def host_expert_mats(wl: synth.Workload, e: int, shared: bool = False):
    return tuple(synth.make_expert_matrix(wl, e, m, shared) for m in range(3))
