"""The seeded generator: its definition (SplitMix64 counter form, FNV-1a keys,
Irwin-Hall normal approximation, RNE bfloat16) checked against plain
Python-integer restatements and torch's own float32 -> bfloat16 rounding."""
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


def test_normal_moments_and_range():
    x = host.normal_f32(1, "moments", (1 << 20,)).astype(np.float64)
    assert abs(x.mean()) < 0.005
    assert abs(x.var() - 1.0) < 0.01
    assert np.abs(x).max() <= 2 * math.sqrt(3) + 1e-6
    # Irwin-Hall(4) kurtosis is 3 - 1.2/4 = 2.7
    kurt = np.mean(x ** 4) / np.mean(x ** 2) ** 2
    assert abs(kurt - 2.7) < 0.03


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
