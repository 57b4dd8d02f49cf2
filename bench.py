#!/usr/bin/env python
"""Benchmark: one GLM-5.2-shape quantised MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward of the whole layer (Q8_0 of x, router, bucketing, expert
gate/up + SiLU + Q8_0 of h, expert down, combine) over one batch of the
workload's tokens, with all weights resident in HBM.  The timed steps cycle
through seeded token batches (64 for decode-sized batches, 8 for larger ones),
so consecutive steps select different experts and every step streams its
experts' weights (170 MB at one token, more at more tokens: more than the
126 MB L2) from HBM.  The JSON line also reports the same batch repeated
(fixed_batch) and the same batch with L2 flushed before every step
(l2_flushed: 2x L2 written; this evicts the kernels' instructions too).  Each
step is timed on the device with CUDA events recorded by the library at its
phase boundaries; the phase events also give the live duration of the
dominant kernel for the roofline (the fused kernel at T <= 4, the gate/up
GEMV at 5 <= T < 64, the gate/up tensor-core GEMM at T >= 64, for which the
int8 tensor utilisation is reported as well).

N > 1: one process per GPU (torchrun); each rank runs an independent replica of
the layer on its own tokens (the layer forward has no exchange step), the
ranks' times are max-reduced and value = tokens of all ranks / that time.

--impl reference times the CPU oracle (plain C, fp64) on the host cores on a
bounded sample of the same workload; on N > 1 only rank 0 runs it.

Other workloads of the same layer: glm52_decode_int4_t1_topp07 (adaptive
expert top-p 0.7), glm52_decode_int2_t1 (packed int2 experts),
glm52_verify_int4_t4, glm52_int8_t16_outliers, glm52_prefill_int4_t512_zipf.
--requant times the FP8 -> int4 requantiser (the converter step) on 16
experts of the GLM-5.2 shape instead, and prints its own JSON line (GB/s).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GLM-5.2-shape MoE layer tokens/s; expert-weight HBM GB/s vs B200 peak"
DEFAULT_WORKLOAD = "glm52_decode_int4_t1"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------
# helpers (host-side logic, covered by CPU tests)
# ----------------------------------------------------------------------------
def measured_peak_hbm() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(tokens_per_rank: int, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job tokens/s: every rank ran `steps` steps of `tokens_per_rank`."""
    return world * tokens_per_rank * steps / (max_total_ms / 1e3)


def expert_bytes(shape) -> int:
    return shape.expert_bytes


def gateup_bytes(shape) -> int:
    """Algorithmic bytes of one expert's gate+up matrices and their row scales."""
    return 2 * shape.matrix_bytes(shape.inter, shape.hidden) + 2 * 4 * shape.inter


# The files each measured kernel's device code is compiled from: a committed
# ncu traffic record of that kernel stays valid while these are unchanged.
KERNEL_SOURCES = {
    "k_moe_small": ["moe_small.cu", "moe_device.cuh", "moe_ptx.cuh"],
    "k_gateup": ["moe_expert.cu", "moe_device.cuh", "moe_ptx.cuh"],
    "k_tc_gemm_dp": ["moe_tc.cu", "moe_tc.cuh", "moe_device.cuh", "moe_ptx.cuh"],
}


def kernel_sources_sha(kernel: str = "k_moe_small") -> str:
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(ROOT, "quantized_routed_expert_group_b200", "csrc", name), "rb") as fh:
            h.update(name.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str) -> float | None:
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken on the current kernel sources; otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            doc = json.load(f)
    except Exception:
        return None
    for row in doc.get("kernels", []):
        if row.get("kernel") == kernel and row.get("workload") == workload and \
                row.get("sources_sha") == kernel_sources_sha(kernel):
            return float(row["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str | None, period_ms: int = 50):
        self.proc = None
        if gpu_id is None:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", str(period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        return parse_clock_samples(out)


def parse_clock_samples(text: str) -> dict | None:
    rows = [r.split(",") for r in text.strip().splitlines() if r.count(",") >= 8]
    if not rows:
        return None
    sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
    mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if "Active" in v and "Not" not in v})
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------
REQUANT_EXPERTS = 16


ROTATIONS_SMALL, ROTATIONS_LARGE = 64, 8  # seeded token batches the timed steps cycle through
TENSOR_I8_NOMINAL_RATIO = 2.0             # dense int8 / dense bf16 tensor throughput (nominal)
FALLBACK_BF16_TFLOPS = 1590.0


def measured_peak_bf16() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["bf16_tflops"])
        return v, "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def rotating_workloads(wl, rank: int, n: int):
    """n seeded token batches of the workload (same shapes and value recipe,
    different seeds); rank r of a multi-GPU run gets its own."""
    from quantized_routed_expert_group_b200 import synth
    return [synth.Workload(wl.name, wl.shape, wl.T, wl.seed + 7919 * rank + 104729 * (i + 1), wl.x_kind,
                           wl.bias_kind) for i in range(n)]


def step_stats(ms: list[float]) -> dict:
    return {"median": round(statistics.median(ms), 5), "mean": round(statistics.mean(ms), 5),
            "min": round(min(ms), 5), "max": round(max(ms), 5)}


def capture_steps(torch, moe, layer, batches, out, flush=None, phase_events=True):
    """One CUDA graph of len(batches) consecutive forwards, each bracketed by
    the library's phase events (moe_profile_events) unless phase_events is
    False, with an L2 flush before each when `flush` is given.  Returns
    (graph, events), or (None, events) if the capture fails (the caller then
    runs the steps eagerly)."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.PROFILE_MAX_EVENTS)] for _ in batches]
    for row in evs:  # torch creates the CUDA event on first record
        for ev in row:
            ev.record()
    torch.cuda.synchronize()
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i, x in enumerate(batches):
                    if flush is not None:
                        flush.fill_(i & 0xFF)
                    if phase_events:
                        moe.profile_events(evs[i])
                    layer.forward(x, out)
                moe.profile_events(None)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        return g, evs
    except Exception as exc:  # noqa: BLE001
        moe.profile_events(None)
        print(f"graph capture unavailable ({exc}); timing eager steps", file=sys.stderr)
        torch.cuda.synchronize()
        return None, evs


def run_steps(torch, moe, layer, batches, out, graph, evs, flush=None):
    """Run the captured steps (or the same steps eagerly)."""
    if graph is not None:
        graph.replay()
        return
    for i, x in enumerate(batches):
        if flush is not None:
            flush.fill_(i & 0xFF)
        moe.profile_events(evs[i])
        layer.forward(x, out)
    moe.profile_events(None)


def run_ours(args) -> dict | None:
    import torch
    import torch.distributed as dist

    from quantized_routed_expert_group_b200 import moe, synth

    rank, world, local = dist_env()
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[args.workload]
    s = wl.shape
    # replicas: same weights, each rank its own tokens; the timed steps cycle
    # through R seeded batches so that no step finds the previous step's
    # experts in L2 (every step streams more weight bytes than L2 holds)
    R = ROTATIONS_SMALL if wl.T <= 16 else ROTATIONS_LARGE
    layer = moe.synth_layer(wl, dev)
    xs = [torch.from_numpy(synth.make_x(w)).to(dev) for w in rotating_workloads(wl, rank, R)]
    out = torch.empty_like(xs[0])
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)

    for i in range(args.warmup):
        layer.forward(xs[i % R], out)
    torch.cuda.synchronize()
    assert layer.device_error() == 0

    K = args.steps
    phases = moe.forward_phases(layer.cfg, wl.T)
    P = len(phases)
    # the K timed steps as one CUDA graph: the device runs them back to back
    # whatever the host's pace; the graph is timed by two events around it
    # (ms_per_step = total / K).  A second graph of the same K steps carries
    # the library's events at each step's phase boundaries (per-step median,
    # phase times); those events cost a little time of their own.
    batches = [xs[i % R] for i in range(K)]
    graph, evs = capture_steps(torch, moe, layer, batches, out)
    graph_plain, _ = capture_steps(torch, moe, layer, batches, out, phase_events=False)
    run_steps(torch, moe, layer, batches[: min(K, args.warmup)], out, None,
              evs[: min(K, args.warmup)])  # untimed eager steps after the capture
    torch.cuda.synchronize()
    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        pass
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_uuid)
    time.sleep(0.15)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph_plain is not None:
        e_start.record()
        graph_plain.replay()
        e_end.record()
    run_steps(torch, moe, layer, batches, out, graph, evs)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    graph_used = graph is not None and graph_plain is not None
    if world > 1:
        dist.barrier()
    step_ms = [evs[i][0].elapsed_time(evs[i][P]) for i in range(K)]
    phase_ms = [[evs[i][p].elapsed_time(evs[i][p + 1]) for i in range(K)] for p in range(P)]
    assert layer.device_error() == 0
    del graph, graph_plain
    total_ms = e_start.elapsed_time(e_end) if graph_used else sum(step_ms)
    max_total = reduce_max(total_ms, dev)
    value = throughput(wl.T, K, world, max_total)
    # active experts of each rotation (the bytes a step streams)
    n_active = []
    tokens_per_entry = []  # of the first batch: routed experts' token counts, then the shared expert's
    for i in range(R):
        layer.forward(xs[i], out)
        cnt = layer.view(wl.T)["counts"]
        n_active.append(int((cnt > 0).sum().item()))
        if i == 0:
            tokens_per_entry = [int(c) for c in cnt.cpu().tolist() if c > 0] + ([wl.T] * s.n_shared)
    torch.cuda.synchronize()

    # variants, reported alongside: the same batch every step (no flush), and
    # the same batch with L2 flushed (2x its size written) before every step
    K_v = min(K, 200)

    def timed(flush_l2: bool) -> list[float]:
        same = [xs[0]] * K_v
        g, ev = capture_steps(torch, moe, layer, same, out, flush if flush_l2 else None)
        run_steps(torch, moe, layer, same, out, g, ev, flush if flush_l2 else None)
        torch.cuda.synchronize()
        return [ev[i][0].elapsed_time(ev[i][P]) for i in range(K_v)]

    fixed_ms = timed(False)
    flushed_ms = timed(True)

    # end to end through the host-buffer entry point (pinned host x / out)
    K_e2e = max(1, min(K, 200))
    xh = [x.cpu().pin_memory() for x in xs]
    oh = torch.empty_like(xh[0]).pin_memory()
    e2e_s = 0.0
    for i in range(K_e2e):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        layer.forward_host(xh[i % R], oh)
        e2e_s += time.perf_counter() - t0
    e2e_max = reduce_max(e2e_s * 1e3, dev)
    e2e_value = throughput(wl.T, K_e2e, world, e2e_max)

    peak, peak_kind = measured_peak_hbm()
    router_bytes = s.n_experts * s.hidden * 4
    mean_active = statistics.mean(n_active)
    layer_bytes = (mean_active + s.n_shared) * expert_bytes(s)
    ms_step = max_total / K
    layer_gbs = layer_bytes / (ms_step * 1e-3) / 1e9
    tensor = None
    if phases == ["fused"]:
        # the fused path: one persistent kernel is the whole step (Q8_0 of x,
        # router logits over the router weights, selection, experts,
        # combine); its bytes are the experts' and the router matrix
        dom_kernel, dom_ms = "k_moe_small", ms_step
        dom_bytes = layer_bytes + router_bytes
    else:
        gu_ms = statistics.mean(phase_ms[phases.index("gate_up")])
        dom_bytes = (mean_active + s.n_shared) * gateup_bytes(s)
        dom_ms = gu_ms
        if moe.forward_launches(layer.cfg, wl.T) == moe.TC_LAUNCHES:
            dom_kernel = "k_tc_gemm_dp"
            # int8 tensor work of the gate/up GEMM: 2 ops per MAC, gate and up
            # (algorithmic: every (token, pick) once; issued: the five digit
            # planes of each token over its 48-token chunk padded to 16)
            ops = 2.0 * 2.0 * (wl.T * s.top_k + wl.T * s.n_shared) * s.hidden * s.inter
            pad_rows = 0
            for n in tokens_per_entry:
                full, rem = divmod(int(n), 48)
                pad_rows += 48 * full + 16 * ((rem + 15) // 16)
            issued = 2.0 * 2.0 * 5 * pad_rows * s.hidden * s.inter
            bf16, bf16_kind = measured_peak_bf16()
            i8_peak = bf16 * TENSOR_I8_NOMINAL_RATIO
            tops = ops / (gu_ms * 1e-3) / 1e12
            itops = issued / (gu_ms * 1e-3) / 1e12
            tensor = {"kernel": "k_tc_gemm_dp (gate/up)", "int8_ops": ops, "achieved_tops": round(tops, 1),
                      "issued_int8_ops": issued, "issued_tops": round(itops, 1),
                      "peak_tops": i8_peak, "peak_kind": f"{bf16_kind} bf16 x {TENSOR_I8_NOMINAL_RATIO:g} (nominal int8/bf16)",
                      "frac": round(tops / i8_peak, 4), "issued_frac": round(itops / i8_peak, 4)}
        else:
            dom_kernel = "k_gateup"
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    if rank != 0:
        return None
    res = {
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded; random-init weights of the layer's shape)",
        "config": {"workload": wl.name, "tokens": wl.T, "hidden": s.hidden, "inter": s.inter,
                   "experts": s.n_experts, "top_k": s.top_k, "shared": s.n_shared, "weights": f"int{s.wbits}",
                   "activations": "Q8_0 int8", "unique_experts_per_step": round(mean_active, 2),
                   "token_batches": f"{R} seeded batches, step i uses batch i mod {R}",
                   "timing": ("the K steps as one CUDA graph timed by two events around it (ms_per_step = total "
                              "/ K); step_ms and phases_ms from a second graph of the same steps with the library's "
                              "events at each step's phase boundaries" if graph_used else
                              "eager steps timed by the library's events (graph capture unavailable)"),
                   "l2": ("not flushed: every step streams its selected experts' weights, more than L2 holds, "
                          "and consecutive steps select different experts"),
                   "parallelism": f"replicas x{world}"},
        "step_ms": step_stats(step_ms),
        "layer_hbm": {"algorithmic_bytes": int(layer_bytes), "gbs": round(layer_gbs, 1),
                      "frac_measured": round(layer_gbs / peak, 4), "frac_spec_8tbs": round(layer_gbs / SPEC_HBM_GBS, 4)},
        "phases_ms": {n: round(statistics.mean(v), 5) for n, v in zip(phases, phase_ms)},
        "fixed_batch": {"steps": K_v, "step_ms": step_stats(fixed_ms)},
        "l2_flushed": {"steps": K_v, "step_ms": step_stats(flushed_ms),
                       "value": round(throughput(wl.T, K_v, 1, sum(flushed_ms)), 3), "unit": "tokens/s"},
        "roofline": {"kernel": dom_kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "algorithmic_bytes_per_launch": int(dom_bytes),
                     "traffic": ncu_traffic(dom_kernel, wl.name)},
        "e2e": {"value": round(e2e_value, 3), "unit": "tokens/s", "h2d_bytes_per_step": xs[0].numel() * 4,
                "d2h_bytes_per_step": out.numel() * 4, "steps": K_e2e},
        "gpu_launches": K * moe.forward_launches(layer.cfg, wl.T),
        "clocks": clocks,
    }
    if tensor is not None:
        res["roofline"]["tensor"] = tensor
    return res


# ----------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline leg)
# ----------------------------------------------------------------------------
def oracle_sample(wl, n_tokens: int):
    """Host inputs for the oracle on the first n_tokens of the workload: router
    weights, and the routed experts those tokens select plus the shared one,
    packed by the oracle's own quantiser (untimed set-up)."""
    from oracle import oracle as orc
    from quantized_routed_expert_group_b200 import synth
    s = wl.shape
    x = synth.make_x(wl)[:n_tokens]
    Wr, bias = synth.make_router_w(wl), synth.make_bias(wl)
    idx, _ = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf, topp=s.topp)
    routed = {}
    for e in sorted(set(idx.reshape(-1).tolist()) - {-1}):  # -1: dropped by the top-p
        routed[e] = orc.pack_expert(*(synth.make_expert_matrix(wl, e, m) for m in range(3)), s.wbits)
    shared = orc.pack_expert(*(synth.make_expert_matrix(wl, 0, m, True) for m in range(3)), s.wbits) \
        if s.n_shared else None
    return x, Wr, bias, routed, shared


def time_oracle(wl, n_tokens: int, budget_s: float, max_steps: int | None = None, warmup: int = 0):
    from oracle import oracle as orc
    x, Wr, bias, routed, shared = oracle_sample(wl, n_tokens)
    for _ in range(warmup):
        orc.layer_forward(wl.shape, x, Wr, bias, routed, shared)
    times = []
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        orc.layer_forward(wl.shape, x, Wr, bias, routed, shared)
        times.append(time.perf_counter() - t0)
        if max_steps is not None and len(times) >= max_steps:
            break
        if time.perf_counter() - t_start >= budget_s:
            break
    return times, orc.num_threads()


def cpu_baseline(wl, budget_s: float = 12.0) -> dict:
    n_tok = 1
    times, cores = time_oracle(wl, n_tok, budget_s)
    tps = n_tok * len(times) / sum(times)
    return {"value": round(tps, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n_tok} token(s) of {wl.name}, {len(times)} forward(s) of the C oracle "
                      f"(plain C, fp64 sums, OpenMP over output rows), {sum(times):.1f} s"}


def run_reference(args) -> dict | None:
    from quantized_routed_expert_group_b200 import synth
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    wl = synth.WORKLOADS[args.workload]
    # each step is the oracle's forward of one token of the workload; the run
    # stops after the requested steps or ~3 minutes, whichever comes first
    times, cores = time_oracle(wl, 1, budget_s=180.0, max_steps=args.steps, warmup=min(args.warmup, 1))
    K = len(times)
    total = sum(times)
    value = K / total
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / K * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.T, "hidden": wl.shape.hidden, "inter": wl.shape.inter,
                   "experts": wl.shape.n_experts, "weights": f"int{wl.shape.wbits}",
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"one token of {wl.name} per step, {K} steps"},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_requant(args) -> dict:
    """The converter step on the GPU: FP8 E4M3 expert weights with 128 x 128
    block scales (seeded, resident in HBM, more than L2) requantised into the
    engine's packed int4 per-row container.  One step = the gate/up rows of
    REQUANT_EXPERTS experts of the GLM-5.2 shape, then their down rows (two
    launches).  Reports the bytes the step must move (FP8 codes and block
    scales in, packed codes and row scales out) per second."""
    import torch
    from quantized_routed_expert_group_b200 import moe, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s, block, wbits, n_exp = synth.GLM_INT4, 128, 4, REQUANT_EXPERTS
    gen = torch.Generator(device=dev).manual_seed(2026)

    def fp8_codes(rows, cols):
        c = torch.randint(0, 256, (rows, cols), dtype=torch.uint8, device=dev, generator=gen)
        c[(c & 0x7F) == 0x7F] = 0x3A  # no NaN codes
        return c

    def block_scales(rows, cols):
        nb = (-(-rows // block), -(-cols // block))
        return torch.rand(nb, device=dev, generator=gen) * 1e-3 + 1e-4

    mats = [(fp8_codes(n_exp * 2 * s.inter, s.hidden), None), (fp8_codes(n_exp * s.hidden, s.inter), None)]
    mats = [(w8, block_scales(*w8.shape)) for w8, _ in mats]
    outs = [(torch.empty((w8.shape[0], w8.shape[1] * wbits // 8), dtype=torch.uint8, device=dev),
             torch.empty(w8.shape[0], dtype=torch.float32, device=dev)) for w8, _ in mats]
    step_bytes = sum(w8.numel() + bs.numel() * 4 + p.numel() + sc.numel() * 4
                     for (w8, bs), (p, sc) in zip(mats, outs))

    def step():
        for (w8, bs), (p, sc) in zip(mats, outs):
            moe.requant_fp8(w8, bs, block, wbits, p, sc)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = min(args.steps, 200)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        pass
    sampler = ClockSampler(gpu_uuid)
    time.sleep(0.15)
    for a, b in ev:
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    gbs = step_bytes / (ms * 1e-3) / 1e9
    peak, peak_kind = measured_peak_hbm()
    res = {
        "metric": "FP8 E4M3 (128x128 block scales) -> packed int4 per-row requantisation, bytes moved per second",
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3 -> int4", "data": "synthetic (seeded FP8 codes and block scales)",
        "config": {"workload": f"requant_fp8_int4_glm52_{n_exp}experts", "experts": n_exp, "hidden": s.hidden,
                   "inter": s.inter, "block": block, "bytes_per_step": step_bytes,
                   "l2": "not flushed: each step moves more than L2"},
        "roofline": {"kernel": "k_pack_rows<4,RowsFp8Block>", "bound": "hbm", "achieved": round(gbs, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(gbs / peak, 4),
                     "algorithmic_bytes_per_launch": step_bytes // 2, "traffic": None},
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        from oracle import oracle as orc
        import numpy as np
        rows = 512
        w8 = mats[0][0][:rows].cpu().numpy()
        bs = mats[0][1][: -(-rows // block)].cpu().numpy()
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < 5.0:
            orc.requant_fp8(w8, bs, block, wbits)
            n += 1
        dt = time.perf_counter() - t0
        moved = n * (w8.size + bs.size * 4 + w8.size * wbits // 8 + rows * 4)
        res["cpu_baseline"] = {"value": round(moved / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                               "sample": f"{n} x {rows} gate rows (6144 FP8 codes each) of the same input, {dt:.1f} s"}
    return res


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--requant", action="store_true",
                    help="time the FP8 -> int4 requantiser (the converter step) instead of the layer")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.requant:
        print(json.dumps(run_requant(args)), flush=True)
        return
    if args.impl == "reference":
        res = run_reference(args)
    else:
        res = run_ours(args)
        if res is not None and res["n_gpus"] == 1 and not args.no_cpu_baseline:
            from quantized_routed_expert_group_b200 import synth
            res["cpu_baseline"] = cpu_baseline(synth.WORKLOADS[args.workload])
    if res is not None:
        print(json.dumps(res), flush=True)
    try:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
