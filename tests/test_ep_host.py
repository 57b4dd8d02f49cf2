"""Expert parallelism, host side (no GPU): the rank partition and the
all-reduce of the ranks' shares, with world_size 2 and 3 gloo groups on CPU.

Each rank's share is computed from the oracle's own trace (its per-slot expert
outputs and routing weights): the routed picks of the rank's expert range,
weighted, plus the shared expert on rank 0, summed in fp64 and rounded to fp32
-- what moe_layer_forward_partial computes on a GPU.  The all-reduced sum must
equal the oracle's layer output to fp32 rounding."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import oracle as orc
from quantized_routed_expert_group_b200 import ep, synth


@pytest.mark.parametrize("E,world", [(16, 1), (16, 2), (16, 3), (256, 8), (7, 3), (5, 5)])
def test_expert_ranges_partition(E, world):
    rs = [ep.expert_range(r, world, E) for r in range(world)]
    assert rs[0][0] == 0 and rs[-1][1] == E
    for (a, b), (c, d) in zip(rs, rs[1:]):
        assert b == c and a <= b
    sizes = [b - a for a, b in rs]
    assert max(sizes) - min(sizes) <= 1
    assert [ep.owns_shared(r) for r in range(world)].count(True) == 1


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_case(T):
    wl = synth.WORKLOADS["tiny_h256_e16_int8_t4"].with_tokens(T)
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    routed = {e: orc.pack_expert(*(synth.make_expert_matrix(wl, e, m) for m in range(3)), s.wbits)
              for e in range(s.n_experts)}
    shared = orc.pack_expert(*(synth.make_expert_matrix(wl, 0, m, True) for m in range(3)), s.wbits)
    return s, x, orc.layer_forward(s, x, Wr, bias, routed, shared)


def _share(s, tr, lo, hi, with_shared):
    """The rank's share from the oracle trace (fp64 sum in pick order, then
    the shared expert; rounded to fp32)."""
    k = s.top_k
    acc = np.zeros((tr.out.shape[0], s.hidden), np.float64)
    for j in range(k):
        m = (tr.idx[:, j] >= lo) & (tr.idx[:, j] < hi)
        acc[m] += tr.w[m, j].astype(np.float64)[:, None] * tr.ys[m, j].astype(np.float64)
    if with_shared:
        acc += tr.ys[:, k].astype(np.float64)
    return torch.from_numpy(acc.astype(np.float32))


def _worker(rank, world, port, T, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s, x, tr = _oracle_case(T)
        seen = []

        def partial(xx, lo, hi, sh):
            seen.append((lo, hi, sh))
            return _share(s, tr, lo, hi, sh)

        out = ep.ep_forward(partial, torch.from_numpy(x), s.n_experts)
        err = float(np.abs(out.numpy().astype(np.float64) - tr.out).max() /
                    np.sqrt(np.mean(tr.out.astype(np.float64) ** 2)))
        q.put((rank, seen, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 4), (3, 17)])
def test_ep_forward_gloo_matches_layer(world, T):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    E = synth.WORKLOADS["tiny_h256_e16_int8_t4"].shape.n_experts
    for r, seen, err in res:
        assert seen == [(*ep.expert_range(r, world, E), r == 0)]
        assert err <= 1e-6, err  # fp32 rounding of the shares and of their sum


def test_ep_forward_without_group_is_the_whole_layer():
    assert not dist.is_initialized()
    s, x, tr = _oracle_case(3)
    out = ep.ep_forward(lambda xx, lo, hi, sh: _share(s, tr, lo, hi, sh), torch.from_numpy(x), s.n_experts)
    np.testing.assert_array_equal(out.numpy(), tr.out)
