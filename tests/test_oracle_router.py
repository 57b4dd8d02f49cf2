"""Pins of the oracle's router and bucketing (CPU only).

Fixed by: hand-worked cases (tests/golden/router_cases.json), the router's
invariants, brute force over every group subset and every expert subset, the
special cases that reduce to a plain sort (one group; zero bias), and numpy's
stable sort / bincount for the bucketing.
"""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.special import expit

from quantized_routed_expert_group_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    with open(os.path.join(GOLDEN, "router_cases.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["note"][:40])
def test_router_golden(orc, case):
    E = len(case["logits"])
    x = np.ones((1, 1), np.float32)
    Wr = np.array(case["logits"], np.float32).reshape(E, 1)
    bias = np.array(case["bias"], np.float32)
    idx, w = orc.router(x, Wr, bias, case["n_groups"], case["topk_groups"], case["top_k"], case["rsf"])
    assert idx[0].tolist() == case["idx"], case["note"]
    np.testing.assert_allclose(w[0], case["w"], rtol=1e-6, err_msg=case["note"])


def _route(orc, wl, T=None):
    if T is not None:
        wl = wl.with_tokens(T)
    s = wl.shape
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    idx, w, c, gs = orc.router(x, Wr, bias, s.n_groups, s.topk_groups, s.top_k, s.rsf, want_scores=True)
    return x, Wr, bias, idx, w, c, gs


def _logits64(x, Wr):
    return x.astype(np.float64) @ Wr.astype(np.float64).T


@pytest.mark.parametrize("name,T", [("tiny_h256_e16_int8_t4", 4), ("tiny_h256_e16_int8_t4", 64),
                                    ("glm52_decode_int4_t1", 8), ("glm52_prefill_int4_t512_zipf", 16)])
def test_router_invariants(orc, name, T):
    wl = synth.WORKLOADS[name]
    s = wl.shape
    x, Wr, bias, idx, w, c, gs = _route(orc, wl, T)
    per = s.n_experts // s.n_groups
    for t in range(T):
        sel = idx[t]
        assert len(set(sel.tolist())) == s.top_k
        groups = set((sel // per).tolist())
        # the kept groups are the topk_groups best by group score
        order = np.argsort(-gs[t], kind="stable")
        kept = set(order[: s.topk_groups].tolist())
        assert groups <= kept
        assert gs[t][list(kept)].min() >= gs[t][[g for g in range(s.n_groups) if g not in kept]].max(initial=-np.inf)
        # selected experts are the best c inside the kept groups, in descending order
        cand = [e for e in range(s.n_experts) if e // per in kept]
        best = sorted(cand, key=lambda e: (-c[t][e], e))[: s.top_k]
        assert sel.tolist() == best
        # weights: non-negative, proportional to the UNBIASED sigmoid, summing to rsf
        assert np.all(w[t] >= 0)
        assert abs(float(w[t].astype(np.float64).sum()) - s.rsf) <= 1e-6 * s.rsf
        sig = expit(_logits64(x[t:t + 1], Wr)[0])[sel]
        np.testing.assert_allclose(w[t], sig / sig.sum() * s.rsf, rtol=2e-6)
        # c = sigmoid(logit) + bias (library sigmoid on a numpy fp64 matmul)
        np.testing.assert_allclose(c[t], expit(_logits64(x[t:t + 1], Wr)[0]) + bias.astype(np.float64),
                                   rtol=0, atol=1e-12)


def test_router_bruteforce_tiny(orc):
    """Enumerate every tg-subset of groups and every k-subset of experts (tiny layer)."""
    wl = synth.WORKLOADS["tiny_h256_e16_int8_t4"]
    s = wl.shape
    x, Wr, bias, idx, w, c, gs = _route(orc, wl, 32)
    per = s.n_experts // s.n_groups
    cc = expit(_logits64(x, Wr)) + bias.astype(np.float64)
    for t in range(x.shape[0]):
        # group score by brute force: the largest sum over any pair of distinct experts
        gscore = [max(cc[t][a] + cc[t][b] for a, b in itertools.combinations(range(g * per, (g + 1) * per), 2))
                  for g in range(s.n_groups)]
        best_groups = max(itertools.combinations(range(s.n_groups), s.topk_groups),
                          key=lambda S: (sum(gscore[g] for g in S), [-g for g in S]))
        cand = [e for e in range(s.n_experts) if e // per in best_groups]
        best_set = max(itertools.combinations(cand, s.top_k),
                       key=lambda S: (sum(cc[t][e] for e in S), [-e for e in S]))
        assert set(idx[t].tolist()) == set(best_set)
        assert set((idx[t] // per).tolist()) <= set(best_groups)


def test_router_one_group_is_plain_topk(orc):
    """G = tg = 1: the router reduces to top-k of sigmoid(logit) + bias."""
    wl = synth.WORKLOADS["glm52_decode_int4_t1"].with_tokens(6)
    x, Wr, bias = synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl)
    idx, w = orc.router(x, Wr, bias, 1, 1, 8, 2.5)
    cc = expit(_logits64(x, Wr)) + bias.astype(np.float64)
    ref = np.argsort(-cc, axis=1, kind="stable")[:, :8]
    np.testing.assert_array_equal(idx, ref)


def test_router_zero_bias_one_group_is_logit_topk(orc):
    """bias = 0 and one group: top-k of the raw logits (sigmoid is monotone)."""
    wl = synth.WORKLOADS["glm52_decode_int4_t1"].with_tokens(6)
    x, Wr = synth.make_x(wl), synth.make_router_w(wl)
    idx, w = orc.router(x, Wr, np.zeros(Wr.shape[0], np.float32), 1, 1, 8, 1.0)
    ref = np.argsort(-_logits64(x, Wr), axis=1, kind="stable")[:, :8]
    np.testing.assert_array_equal(idx, ref)


def test_router_rejects_bad_shapes(orc):
    x = np.zeros((1, 32), np.float32)
    Wr = np.zeros((16, 32), np.float32)
    b = np.zeros(16, np.float32)
    for G, tg, k in ((5, 2, 2), (4, 5, 2), (4, 2, 9), (16, 2, 2)):
        with pytest.raises(ValueError):
            orc.router(x, Wr, b, G, tg, k, 1.0)


@pytest.mark.parametrize("T,k,E", [(1, 8, 256), (4, 2, 16), (37, 8, 256), (512, 8, 256), (0, 8, 256)])
def test_bucket_against_stable_sort(orc, T, k, E):
    rng = np.random.default_rng(T * 1000 + E)
    rows = [rng.choice(E, size=k, replace=False) for _ in range(T)]
    idx = (np.stack(rows) if rows else np.zeros((0, k))).astype(np.int32).reshape(T, k)
    counts, offsets, perm = orc.bucket(idx, E)
    flat = idx.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    assert counts.sum() == T * k
    assert sorted(perm.tolist()) == list(range(T * k))
    for e in range(E):
        toks = perm[offsets[e]:offsets[e + 1]] // k
        assert np.all(np.diff(toks) > 0)
