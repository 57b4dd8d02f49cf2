"""Checks of the seeded input generator (CPU only).

SplitMix64 is checked against its published output sequence, the numpy and C
host paths against each other, and the workload recipes against what they
promise (moments, correlation, outlier channels, Zipf head slope).
"""
import numpy as np
import pytest

from quantized_routed_expert_group_b200 import synth


def test_splitmix64_published_sequence():
    # SplitMix64 seeded with 1234567: the first five outputs as published with the
    # generator (e.g. the Rosetta Code "Pseudo-random numbers/Splitmix64" task).
    ref = [6457827717110365317, 3203168211198807973, 9817491932198370423,
           4593380528125082431, 16408922859458223821]
    assert [synth.stream_key(1234567, n) for n in range(5)] == ref
    key = synth.stream_key(1234567, 0)
    # words(seed, tid, ...) is the stream seeded with key(seed, tid)
    w = synth.words(1234567, 0, 0, 3)
    assert int(w[0]) == synth._mix_int(key + synth.GAMMA)


def test_host_c_matches_numpy():
    a = synth.normal(11, 1007, 9000, 0.02, offset=333, backend="numpy")
    b = synth.normal(11, 1007, 9000, 0.02, offset=333, backend="c")
    np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32))


def test_normal_moments():
    z = synth.normal(5, 77, 200000, 1.0).astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    assert np.abs(z).max() <= 6.0
    u = synth.uniform(5, 78, 100000, -0.1, 0.2).astype(np.float64)
    assert u.min() >= -0.1 and u.max() < 0.1 + 1e-7 and abs(u.mean()) < 0.002


def test_permutation_is_permutation():
    p = synth.permutation(3, 5, 6144)
    assert sorted(p.tolist()) == list(range(6144))


def test_correlated_verify_batch():
    wl = synth.WORKLOADS["glm52_verify_int4_t4"]
    x = synth.make_x(wl).astype(np.float64)
    c = np.corrcoef(x)
    off = c[~np.eye(4, dtype=bool)]
    assert np.all(np.abs(off - 0.8) < 0.03)


def test_outlier_channels():
    wl = synth.WORKLOADS["glm52_int8_t16_outliers"]
    x = synth.make_x(wl)
    ch = synth.outlier_channels(wl)
    assert len(ch) == 61
    big = np.abs(x[:, ch]).mean()
    rest = np.abs(np.delete(x, ch, axis=1)).mean()
    assert 15 < big / rest < 25


@pytest.mark.slow
def test_zipf_head_slope(orc):
    """Prefill workload: the 64 most used experts' token counts fall off with a
    log-log slope near -1.1 (the recipe's calibration of alpha)."""
    wl = synth.WORKLOADS["glm52_prefill_int4_t512_zipf"]
    s = wl.shape
    idx, _ = orc.router(synth.make_x(wl), synth.make_router_w(wl), synth.make_bias(wl),
                        s.n_groups, s.topk_groups, s.top_k, s.rsf)
    cnt = np.sort(np.bincount(idx.reshape(-1), minlength=s.n_experts))[::-1]
    r = np.arange(1, 65)
    slope = np.polyfit(np.log(r), np.log(cnt[:64]), 1)[0]
    assert -1.25 < slope < -0.95, slope
    assert cnt[0] <= wl.T
