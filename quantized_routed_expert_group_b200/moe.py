"""Python binding of the C ABI in include/moe.h (argument marshalling only).

Every function takes torch tensors that live on a CUDA device (unless the
name says host), passes their data pointers and the current stream to the C
library, and raises ``MoeError`` on a non-zero status.  There is no fallback:
if the CUDA library has not been built, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from . import synth
from .build import LIB_PATH

_vp, _i64, _int, _flt, _u64, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                    ctypes.c_uint64, ctypes.c_size_t)

MOE_OK, MOE_EINVAL, MOE_EUNSUPPORTED, MOE_EWORKSPACE, MOE_ECUDA, MOE_EDEVICE = 0, -1, -2, -3, -4, -5


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


class MoeConfig(ctypes.Structure):
    _fields_ = [("hidden", _int), ("inter", _int), ("n_experts", _int), ("n_groups", _int),
                ("topk_groups", _int), ("top_k", _int), ("n_shared", _int),
                ("routed_scaling_factor", _flt), ("wbits", _int), ("expert_topp", _flt)]


class MoeExperts(ctypes.Structure):
    _fields_ = [("w_gate", _vp), ("w_up", _vp), ("w_down", _vp), ("s_gate", _vp), ("s_up", _vp), ("s_down", _vp)]


class MoeWorkspaceLayout(ctypes.Structure):
    _fields_ = [("xq", _vp), ("xd", _vp), ("idx", _vp), ("w", _vp), ("counts", _vp), ("offsets", _vp),
                ("perm", _vp), ("hq", _vp), ("hd", _vp), ("y", _vp), ("error", _vp)]


_SIGS = {
    "moe_quantize_act_q8_0": ([_vp, _i64, _int, _vp, _vp, _vp], _int),
    "moe_pack_weights": ([_vp, _i64, _int, _int, _vp, _vp, _vp], _int),
    "moe_requant_fp8": ([_vp, _vp, _i64, _int, _int, _int, _vp, _vp, _vp], _int),
    "moe_router_workspace_bytes": ([ctypes.POINTER(MoeConfig), _int], _sz),
    "moe_router_select": ([ctypes.POINTER(MoeConfig), _vp, _int, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _int),
    "moe_bucket_tokens": ([ctypes.POINTER(MoeConfig), _vp, _int, _vp, _vp, _vp, _vp], _int),
    "moe_workspace_bytes": ([ctypes.POINTER(MoeConfig), _int], _sz),
    "moe_workspace_init": ([ctypes.POINTER(MoeConfig), _int, _vp, _sz, _vp], _int),
    "moe_layer_forward": ([ctypes.POINTER(MoeConfig), _vp, _int, _vp, _vp, ctypes.POINTER(MoeExperts),
                           ctypes.POINTER(MoeExperts), _vp, _vp, _sz, _vp], _int),
    "moe_layer_forward_partial": ([ctypes.POINTER(MoeConfig), _vp, _int, _vp, _vp, ctypes.POINTER(MoeExperts),
                                   ctypes.POINTER(MoeExperts), _int, _int, _int, _vp, _vp, _sz, _vp], _int),
    "moe_layer_forward_host": ([ctypes.POINTER(MoeConfig), _vp, _int, _vp, _vp, ctypes.POINTER(MoeExperts),
                                ctypes.POINTER(MoeExperts), _vp, _vp, _sz, _vp], _int),
    "moe_layer_forward_noalloc": ([ctypes.POINTER(MoeConfig), _vp, _int, _vp, _vp, ctypes.POINTER(MoeExperts),
                                   ctypes.POINTER(MoeExperts), _vp, _vp], _int),
    "moe_workspace_view": ([ctypes.POINTER(MoeConfig), _int, _vp, _sz, ctypes.POINTER(MoeWorkspaceLayout)], _int),
    "moe_block_dots": ([_vp, _i64, _int, _int, _vp, _int, _vp, _vp], _int),
    "moe_block_dots_routine": ([_vp, _i64, _int, _int, _vp, _int, _int, _vp, _vp], _int),
    "moe_get_device_error": ([_vp, _vp, ctypes.POINTER(ctypes.c_int32)], _int),
    "moe_noalloc_device_error": ([_vp, ctypes.POINTER(ctypes.c_int32)], _int),
    "moe_synth_normal": ([_u64, _u64, _i64, _i64, _flt, _vp, _vp], _int),
    "moe_debug_fault_injection": ([_int, _i64], _int),
    "moe_debug_down_rows": ([ctypes.POINTER(MoeConfig), _int, _int, _int, ctypes.c_void_p, ctypes.POINTER(_int)], _int),
    "moe_profile_events": ([ctypes.POINTER(_vp), _int], _int),
    "moe_forward_launches": ([ctypes.POINTER(MoeConfig), _int], _int),
    "moe_forward_phases": ([ctypes.POINTER(MoeConfig), _int], _int),
    "moe_forward_phase_name": ([ctypes.POINTER(MoeConfig), _int, _int], ctypes.c_char_p),
    "moe_status_string": ([_int], ctypes.c_char_p),
}

PROFILE_MAX_EVENTS = 8
# launches of one forward on each path (moe_forward_launches): fused small
# batch, multi-kernel, batched tensor-core
SMALL_LAUNCHES, MULTI_KERNEL_LAUNCHES, TC_LAUNCHES = 1, 7, 13

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it was not built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m quantized_routed_expert_group_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _LIB = L
    return _LIB


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t: torch.Tensor, dtype: torch.dtype, name: str) -> torch.Tensor:
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor of {dtype}")
    return t


def config(shape: synth.LayerShape) -> MoeConfig:
    return MoeConfig(shape.hidden, shape.inter, shape.n_experts, shape.n_groups, shape.topk_groups,
                     shape.top_k, shape.n_shared, shape.rsf, shape.wbits, shape.topp)


# ----------------------------------------------------------------------------
# Entry points
# ----------------------------------------------------------------------------
def quantize_act_q8_0(x: torch.Tensor, stream=None):
    _cuda(x, torch.float32, "x")
    cols = x.shape[-1]
    rows = x.numel() // cols
    q = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    d = torch.empty(x.shape[:-1] + (cols // 32,), dtype=torch.float32, device=x.device)
    _check(lib().moe_quantize_act_q8_0(_ptr(x), rows, cols, _ptr(q), _ptr(d), _stream(stream)), "quantize_act_q8_0")
    return q, d


def pack_weights(w: torch.Tensor, wbits: int, packed: torch.Tensor | None = None,
                 scales: torch.Tensor | None = None, stream=None):
    _cuda(w, torch.float32, "w")
    rows, cols = w.shape
    if packed is None:
        packed = torch.empty((rows, cols * wbits // 8), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=w.device)
    _check(lib().moe_pack_weights(_ptr(w), rows, cols, wbits, _ptr(packed), _ptr(scales), _stream(stream)),
           "pack_weights")
    return packed, scales


def requant_fp8(w8: torch.Tensor, block_scales: torch.Tensor, block: int, wbits: int,
                packed: torch.Tensor | None = None, scales: torch.Tensor | None = None, stream=None):
    """FP8 E4M3 codes [rows][cols] (uint8) with fp32 block scales -> packed
    codes [rows][cols*wbits/8] and fp32 row scales [rows]."""
    _cuda(w8, torch.uint8, "w8")
    _cuda(block_scales, torch.float32, "block_scales")
    rows, cols = w8.shape
    if packed is None:
        packed = torch.empty((rows, cols * wbits // 8), dtype=torch.uint8, device=w8.device)
    if scales is None:
        scales = torch.empty(rows, dtype=torch.float32, device=w8.device)
    _check(lib().moe_requant_fp8(_ptr(w8), _ptr(block_scales), rows, cols, block, wbits, _ptr(packed), _ptr(scales),
                                 _stream(stream)), "requant_fp8")
    return packed, scales


def router_select(cfg: MoeConfig, x: torch.Tensor, router_w: torch.Tensor, bias: torch.Tensor, stream=None):
    T = x.shape[0]
    ws = torch.empty(max(1, lib().moe_router_workspace_bytes(ctypes.byref(cfg), T)), dtype=torch.uint8,
                     device=x.device)
    idx = torch.empty((T, cfg.top_k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, cfg.top_k), dtype=torch.float32, device=x.device)
    _check(lib().moe_router_select(ctypes.byref(cfg), _ptr(x), T, _ptr(router_w), _ptr(bias), _ptr(idx), _ptr(w),
                                   _ptr(ws), ws.numel(), _stream(stream)), "router_select")
    return idx, w


def bucket_tokens(cfg: MoeConfig, idx: torch.Tensor, stream=None):
    T = idx.shape[0]
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device=idx.device)
    offsets = torch.empty(cfg.n_experts + 1, dtype=torch.int32, device=idx.device)
    perm = torch.empty(max(1, T * cfg.top_k), dtype=torch.int32, device=idx.device)
    _check(lib().moe_bucket_tokens(ctypes.byref(cfg), _ptr(idx), T, _ptr(counts), _ptr(offsets), _ptr(perm),
                                   _stream(stream)), "bucket_tokens")
    return counts, offsets, perm[: T * cfg.top_k]


DOTS_MULTI_KERNEL, DOTS_FUSED, DOTS_TENSOR = 0, 1, 2


def block_dots(packed: torch.Tensor, cols: int, wbits: int, q: torch.Tensor, stream=None, routine: int | None = None):
    """Per-block int32 dots [n][rows][cols/32]; routine None is moe_block_dots,
    otherwise moe_block_dots_routine with that routine (DOTS_*)."""
    rows = packed.shape[0]
    q2 = q.reshape(-1, cols)
    out = torch.empty((q2.shape[0], rows, cols // 32), dtype=torch.int32, device=packed.device)
    if routine is None:
        st = lib().moe_block_dots(_ptr(packed), rows, cols, wbits, _ptr(q2), q2.shape[0], _ptr(out), _stream(stream))
    else:
        st = lib().moe_block_dots_routine(_ptr(packed), rows, cols, wbits, _ptr(q2), q2.shape[0], routine, _ptr(out),
                                          _stream(stream))
    _check(st, "block_dots")
    return out


def debug_down_rows(cfg: MoeConfig, T: int, n_entries: int, grid: int):
    """Test export (see moe_debug_down_rows): the first output row of each CTA of
    the one-token fused forward's down split (grid + 1 values) and its row cap."""
    import numpy as np
    starts = np.zeros(grid + 1, np.int32)
    cap = _int(0)
    _check(lib().moe_debug_down_rows(ctypes.byref(cfg), T, n_entries, grid, starts.ctypes.data, ctypes.byref(cap)),
           "debug_down_rows")
    return starts, cap.value


def debug_fault_injection(withhold_entry: int, wait_budget_ns: int = 0) -> None:
    """Test hook (see moe_debug_fault_injection): -1 switches it off."""
    _check(lib().moe_debug_fault_injection(withhold_entry, wait_budget_ns), "debug_fault_injection")


def synth_normal(seed: int, tid: int, n: int, sigma: float, offset: int = 0, out: torch.Tensor | None = None,
                 device="cuda", stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=device)
    _check(lib().moe_synth_normal(seed, tid, offset, n, sigma, _ptr(out), _stream(stream)), "synth_normal")
    return out


def profile_events(events) -> None:
    """Record torch.cuda.Event objects at the forward's phase boundaries
    (PROFILE_MAX_EVENTS events, created with enable_timing=True), or stop
    when events is None."""
    if events is None:
        _check(lib().moe_profile_events(None, 0), "profile_events")
        return
    for ev in events:
        if ev.cuda_event == 0:  # torch creates the CUDA event lazily, on first record
            ev.record()
    arr = (_vp * len(events))(*[ev.cuda_event for ev in events])
    _check(lib().moe_profile_events(arr, len(events)), "profile_events")


def forward_phases(cfg: MoeConfig, T: int) -> list[str]:
    n = lib().moe_forward_phases(ctypes.byref(cfg), T)
    if n < 0:
        _check(n, "forward_phases")
    return [lib().moe_forward_phase_name(ctypes.byref(cfg), T, i).decode() for i in range(n)]


def forward_launches(cfg: MoeConfig, T: int) -> int:
    n = lib().moe_forward_launches(ctypes.byref(cfg), T)
    if n < 0:
        _check(n, "forward_launches")
    return n


def workspace_bytes(cfg: MoeConfig, T_max: int) -> int:
    n = lib().moe_workspace_bytes(ctypes.byref(cfg), T_max)
    if n == 0:
        raise MoeError(MOE_EINVAL, "workspace_bytes")
    return n


def get_device_error(ws: torch.Tensor, stream=None) -> int:
    code = ctypes.c_int32(0)
    st = lib().moe_get_device_error(_ptr(ws), _stream(stream), ctypes.byref(code))
    if st not in (MOE_OK, MOE_EDEVICE):
        _check(st, "get_device_error")
    return code.value


# ----------------------------------------------------------------------------
# Expert weights resident in HBM
# ----------------------------------------------------------------------------
@dataclass
class ExpertBank:
    """Packed weights and row scales of n experts, expert-major (see moe_experts)."""
    w_gate: torch.Tensor   # [n][inter][hidden*wbits/8] uint8
    w_up: torch.Tensor
    w_down: torch.Tensor   # [n][hidden][inter*wbits/8]
    s_gate: torch.Tensor   # [n][inter] fp32
    s_up: torch.Tensor
    s_down: torch.Tensor   # [n][hidden]

    def struct(self) -> MoeExperts:
        return MoeExperts(self.w_gate.data_ptr(), self.w_up.data_ptr(), self.w_down.data_ptr(),
                          self.s_gate.data_ptr(), self.s_up.data_ptr(), self.s_down.data_ptr())

    @property
    def n(self) -> int:
        return self.w_gate.shape[0]

    def nbytes_expert(self) -> int:
        return sum(t[0].numel() * t.element_size() for t in
                   (self.w_gate, self.w_up, self.w_down, self.s_gate, self.s_up, self.s_down))


def empty_bank(shape: synth.LayerShape, n: int, device) -> ExpertBank:
    H, I, b = shape.hidden, shape.inter, shape.wbits
    u8, f32 = torch.uint8, torch.float32
    return ExpertBank(torch.empty((n, I, H * b // 8), dtype=u8, device=device),
                      torch.empty((n, I, H * b // 8), dtype=u8, device=device),
                      torch.empty((n, H, I * b // 8), dtype=u8, device=device),
                      torch.empty((n, I), dtype=f32, device=device),
                      torch.empty((n, I), dtype=f32, device=device),
                      torch.empty((n, H), dtype=f32, device=device))


def bank_from_host_matrices(shape: synth.LayerShape, mats: list, device) -> ExpertBank:
    """Pack fp32 host matrices [(gate, up, down), ...] on the GPU."""
    bank = empty_bank(shape, len(mats), device)
    for e, (g, u, d) in enumerate(mats):
        for m, (src, dst_w, dst_s) in enumerate(((g, bank.w_gate, bank.s_gate), (u, bank.w_up, bank.s_up),
                                                 (d, bank.w_down, bank.s_down))):
            t = torch.as_tensor(src, dtype=torch.float32).to(device).contiguous()
            pack_weights(t, shape.wbits, dst_w[e], dst_s[e])
    return bank


def synth_bank(wl: synth.Workload, device, shared: bool = False, experts=None) -> ExpertBank:
    """Draw the workload's expert weights in HBM with the device generator and
    pack them on the GPU (all routed experts, or the shared ones)."""
    shape = wl.shape
    ids = list(experts) if experts is not None else list(range(shape.n_shared if shared else shape.n_experts))
    bank = empty_bank(shape, len(ids), device)
    rows_max = max(shape.hidden, shape.inter)
    scratch = torch.empty(rows_max * max(shape.hidden, shape.inter), dtype=torch.float32, device=device)
    for slot, e in enumerate(ids):
        for m, (dst_w, dst_s) in enumerate(((bank.w_gate, bank.s_gate), (bank.w_up, bank.s_up),
                                            (bank.w_down, bank.s_down))):
            rows, cols = synth.matrix_dims(shape, m)
            buf = scratch[: rows * cols]
            synth_normal(wl.seed, synth.expert_tid(shape, e, m, shared), rows * cols, 0.02, out=buf)
            pack_weights(buf.view(rows, cols), shape.wbits, dst_w[slot], dst_s[slot])
    return bank


# ----------------------------------------------------------------------------
# Layer
# ----------------------------------------------------------------------------
class MoeLayer:
    """One quantised MoE layer resident on a device: router weights, routed and
    shared expert banks, and a workspace sized for up to T_max tokens."""

    def __init__(self, shape: synth.LayerShape, router_w: torch.Tensor, bias: torch.Tensor,
                 routed: ExpertBank, shared: ExpertBank | None, T_max: int):
        self.shape = shape
        self.cfg = config(shape)
        self.router_w = _cuda(router_w, torch.float32, "router_w")
        self.bias = _cuda(bias, torch.float32, "bias")
        self.routed = routed
        self.shared = shared
        self._routed_s = routed.struct()
        self._shared_s = shared.struct() if shared is not None else MoeExperts()
        self.T_max = T_max
        self.workspace = torch.empty(workspace_bytes(self.cfg, T_max), dtype=torch.uint8, device=router_w.device)
        _check(lib().moe_workspace_init(ctypes.byref(self.cfg), T_max, _ptr(self.workspace), self.workspace.numel(),
                                        None), "workspace_init")

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        _cuda(x, torch.float32, "x")
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} exceeds the workspace's T_max={self.T_max}")
        if out is None:
            out = torch.empty_like(x)
        _check(lib().moe_layer_forward(ctypes.byref(self.cfg), _ptr(x), T, _ptr(self.router_w), _ptr(self.bias),
                                       ctypes.byref(self._routed_s), ctypes.byref(self._shared_s), _ptr(out),
                                       _ptr(self.workspace), self.workspace.numel(), _stream(stream)),
               "layer_forward")
        return out

    def forward_partial(self, x: torch.Tensor, expert_lo: int, expert_hi: int, with_shared: bool,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """The share of the layer output of the routed experts in
        [expert_lo, expert_hi) (+ the shared expert when with_shared), see
        moe_layer_forward_partial."""
        _cuda(x, torch.float32, "x")
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} exceeds the workspace's T_max={self.T_max}")
        if out is None:
            out = torch.empty_like(x)
        _check(lib().moe_layer_forward_partial(ctypes.byref(self.cfg), _ptr(x), T, _ptr(self.router_w),
                                               _ptr(self.bias), ctypes.byref(self._routed_s),
                                               ctypes.byref(self._shared_s), expert_lo, expert_hi,
                                               1 if with_shared else 0, _ptr(out), _ptr(self.workspace),
                                               self.workspace.numel(), _stream(stream)), "layer_forward_partial")
        return out

    def forward_noalloc(self, x: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
        """The layer through the allocation-free entry point (library-owned
        fixed scratch instead of this object's workspace)."""
        _cuda(x, torch.float32, "x")
        _check(lib().moe_layer_forward_noalloc(ctypes.byref(self.cfg), _ptr(x), x.shape[0], _ptr(self.router_w),
                                               _ptr(self.bias), ctypes.byref(self._routed_s),
                                               ctypes.byref(self._shared_s), _ptr(out), _stream(stream)),
               "layer_forward_noalloc")
        return out

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor, stream=None) -> torch.Tensor:
        """x_host / out_host: CPU fp32 tensors (pinned for asynchronous copies)."""
        if x_host.is_cuda or out_host.is_cuda:
            raise ValueError("forward_host takes host tensors")
        T = x_host.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} exceeds the workspace's T_max={self.T_max}")
        _check(lib().moe_layer_forward_host(ctypes.byref(self.cfg), _ptr(x_host), T, _ptr(self.router_w),
                                            _ptr(self.bias), ctypes.byref(self._routed_s),
                                            ctypes.byref(self._shared_s), _ptr(out_host), _ptr(self.workspace),
                                            self.workspace.numel(), _stream(stream)), "layer_forward_host")
        return out_host

    def view(self, T: int) -> dict:
        """Intermediates of the last forward with T tokens, as torch views."""
        L = MoeWorkspaceLayout()
        _check(lib().moe_workspace_view(ctypes.byref(self.cfg), T, _ptr(self.workspace), self.workspace.numel(),
                                        ctypes.byref(L)), "workspace_view")
        s = self.shape
        slots = T * s.top_k + T * s.n_shared
        base = self.workspace.data_ptr()

        def at(ptr, dtype, shape):
            n = 1
            for d in shape:
                n *= d
            off = ptr - base
            esz = torch.tensor([], dtype=dtype).element_size()
            return self.workspace[off: off + n * esz].view(dtype).view(shape)

        return {
            "xq": at(L.xq, torch.int8, (T, s.hidden)),
            "xd": at(L.xd, torch.float32, (T, s.hidden // 32)),
            "idx": at(L.idx, torch.int32, (T, s.top_k)),
            "w": at(L.w, torch.float32, (T, s.top_k)),
            "counts": at(L.counts, torch.int32, (s.n_experts,)),
            "offsets": at(L.offsets, torch.int32, (s.n_experts + 1,)),
            "perm": at(L.perm, torch.int32, (T * s.top_k,)),
            "hq": at(L.hq, torch.int8, (slots, s.inter)),
            "hd": at(L.hd, torch.float32, (slots, s.inter // 32)),
            "y": at(L.y, torch.float32, (slots, s.hidden)),
            # batched tensor-core path: [x, h] took the fp64-epilogue GEMM
            "fp64_fallback": at(L.error + 32, torch.int32, (2,)),
        }

    def device_error(self, stream=None) -> int:
        return get_device_error(self.workspace, stream)


def synth_layer(wl: synth.Workload, device="cuda", T_max: int | None = None) -> MoeLayer:
    """The workload's layer with seeded synthetic weights (routed experts drawn
    and packed in HBM; router weight and bias from the host generator)."""
    s = wl.shape
    router_w = torch.from_numpy(synth.make_router_w(wl)).to(device)
    bias = torch.from_numpy(synth.make_bias(wl)).to(device)
    routed = synth_bank(wl, device)
    shared = synth_bank(wl, device, shared=True) if s.n_shared else None
    return MoeLayer(s, router_w, bias, routed, shared, T_max or wl.T)
