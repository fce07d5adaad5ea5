"""The seeded generator: its definition (SplitMix64 counter form, FNV-1a keys,
table inverse of the normal CDF, RNE bfloat16) checked against plain
Python-integer restatements, scipy's normal distribution and torch's own
float32 -> bfloat16 rounding."""
import math

import numpy as np
import torch

from gen import host, workloads

MASK = (1 << 64) - 1


def _splitmix_seq(state, n):
    """SplitMix64 as a sequential generator (Steele, Lea & Flood 2014)."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def test_counter_form_equals_sequential_splitmix():
    key = host.stream_key(20260002, "csa.q")
    seq = _splitmix_seq(key, 40)
    assert [int(v) for v in host.u64(key, 0, 40)] == seq
    assert [int(v) for v in host.u64(key, 17, 5)] == seq[17:22]
    assert [int(v) for v in host.u64_at(key, np.array([3, 0, 39]))] == [seq[3], seq[0], seq[39]]


def test_fnv1a_known_values():
    # FNV-1a 64: the empty string hashes to the offset basis; "a" is the
    # published 0xaf63dc4c8601ec8c.
    assert host.fnv1a64("") == 0xCBF29CE484222325
    assert host.fnv1a64("a") == 0xAF63DC4C8601EC8C


def test_normal_is_standard_normal():
    from scipy import stats

    x = host.normal_f32(1, "moments", (1 << 21,)).astype(np.float64)
    assert abs(x.mean()) < 0.003
    assert abs(x.var() - 1.0) < 0.004
    kurt = np.mean(x ** 4) / np.mean(x ** 2) ** 2
    assert abs(kurt - 3.0) < 0.03, kurt
    # Kolmogorov-Smirnov against N(0, 1): at 2^21 samples the 1% critical
    # value is 1.63 / sqrt(n) = 0.0011
    assert stats.kstest(x, "norm").statistic < 0.0011
    # the tails are there (Irwin-Hall-type sums stop near 3.5)
    for t in (3.0, 4.0):
        want = 2 * stats.norm.sf(t) * x.size
        got = np.count_nonzero(np.abs(x) > t)
        assert abs(got - want) < 5 * math.sqrt(want) + 1, (t, got, want)
    assert np.abs(x).max() > 4.5


def test_normal_table_accuracy():
    """The piecewise-linear inverse CDF stays within 1e-6 (+ float32
    rounding) of the exact quantile at the middle of every segment."""
    from scipy.special import ndtri

    tab = host.normal_table().astype(np.float64)
    e = np.arange(63, dtype=np.float64)[:, None]
    s = np.arange(256, dtype=np.float64)[None, :]
    p_mid = (1.0 + (s + 0.5) / 256) * np.exp2(-(e + 2.0))
    exact = -ndtri(p_mid)
    interp = tab[:, :, 0] + 0.5 * tab[:, :, 1]
    assert np.max(np.abs(interp - exact) / (1.0 + exact)) < 1.5e-6
    assert np.all(tab[:, :, 1] < 0) and np.all(tab[:, :, 0] > 0)


def _normal_by_integers(u: int) -> float:
    """One output of the normal definition, restated with Python integers
    and float32 scalars."""
    tab = host.normal_table()
    v = max(u & ((1 << 63) - 1), 1)
    e = 62 - (v.bit_length() - 1)
    w = v << e
    seg = (w >> 54) & 0xFF
    f = np.float32((w >> 31) & 0x7FFFFF) * np.float32(2.0 ** -23)
    x = np.float32(tab[e, seg, 0] + np.float32(f * tab[e, seg, 1]))
    return float(-x if u >> 63 else x)


def test_normal_definition_bit_by_bit():
    key = host.stream_key(7, "def")
    us = [int(v) for v in host.u64(key, 0, 64)]
    us += [0, 1, (1 << 63) - 1, 1 << 63, (1 << 63) + 1, (1 << 64) - 1, 1 << 40, (1 << 62) + (1 << 61)]
    got = host._normal_from_u64(np.array(us, dtype=np.uint64))
    want = np.array([_normal_by_integers(u) for u in us], dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    # the deepest octave reaches p = 2^-64 and the shallowest starts at 0
    assert 9.0 < float(got[us.index(1)]) < 9.2 and -9.2 < float(got[us.index(1 << 63)]) < -9.0
    assert 0.0 < float(got[us.index((1 << 63) - 1)]) < 1e-3


def test_bf16_rounding_matches_torch():
    x = host.normal_f32(2, "round", (1 << 16,), scale=37.0)
    x = np.concatenate([x, np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.4e38, 1e-40], np.float32)])
    ours = host.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = host.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_random_access_matches_stream():
    spec = workloads.Spec((7, 9, 16), "bf16", 0.5, None)
    w = workloads.WORKLOADS[2]
    full = workloads.host_tensor(w, "csa.pool", spec)
    rows = np.array([0, 5, 62, 13])
    got = workloads.host_rows(w, "csa.pool", rows, spec)
    assert np.array_equal(got, full.reshape(-1, 16)[rows])


def test_offsets_and_scales_are_separate_roundings():
    x = host.normal_f32(3, "g", (1000,))
    g = host.normal_f32(3, "g", (1000,), 0.1, 1.0)
    assert np.array_equal(g, np.float32(1.0) + x * np.float32(0.1))


def test_subset_idx():
    idx = host.random_subset_idx(5, "idx", np.array([0, 3, 100, 4]), 4)
    assert list(idx[0]) == [-1] * 4
    assert list(idx[1]) == [0, 1, 2, -1]
    assert len(set(idx[2])) == 4 and np.all(np.diff(idx[2]) > 0) and idx[2].max() < 100
    assert list(idx[3]) == [0, 1, 2, 3]


def test_workload_shapes():
    w = workloads.WORKLOADS
    assert w[2].n_csa == (w[2].pos + 1) // 4 == 2048
    assert w[3].n_hca == (w[3].pos + 1) // 128 == 1024
    assert w[4].n_csa == 16384 // 4
    assert w[5].n_csa == 262144 and w[5].n_hca == 8192
    toy = workloads.toy_inputs()
    assert toy["csa.q"].shape == (1, 64, 2, 8) and toy["csa.q"].dtype == np.uint16
    assert toy["csa.ix_ca"].shape == (1, 64, 4)
    s = workloads.specs(w[5])
    assert s["csa.ki"].shape == (8, 262144, 128)
