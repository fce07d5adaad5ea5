"""Seeded, counter-based input generator (host side, numpy).

This module holds none of the attention method's arithmetic: it only turns
(seed, tensor name, element index) into numbers.  The device generator in
``gen/device.cu`` implements the same definition; a GPU test checks that the
two agree bit for bit, so the oracle and the CUDA path see identical inputs
without either one reading the other's output.

Definition
----------
* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): state advances by the golden gamma
  0x9E3779B97F4A7C15 and each output is the state passed through the
  ``mix64`` finaliser (shifts 30/27/31, multipliers 0xBF58476D1CE4E5B9 and
  0x94D049BB133111EB).  Used counter-style: output ``i`` of the stream with
  key ``K`` is ``mix64(K + (i + 1) * gamma)``.
* Stream key of a tensor: ``K = mix64(mix64(seed + gamma) ^ fnv1a64(name))``
  with the 64-bit FNV-1a string hash (offset 0xcbf29ce484222325, prime
  0x100000001b3).
* Approximate N(0, 1): the four 16-bit fields a_j of one output are summed
  (Irwin-Hall of four discrete uniforms); ``x = float32(S - 131070) *
  float32(sqrt(3) / 65536)``.  The mean is 0 and the variance 1; the tails
  stop at +-2*sqrt(3).  Only integer operations and one correctly rounded
  float32 multiply are involved, so host and device agree exactly.
* Scaling and offsets are single correctly rounded float32 operations
  (``x * s``, then ``o + x``), never fused.
* bfloat16 storage: round-to-nearest-even of the float32 bit pattern.
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)
MASK64 = (1 << 64) - 1

# float32(sqrt(3) / 65536): the unit-variance scale of the Irwin-Hall sum.
NORMAL_SCALE = np.float32(np.sqrt(3.0) / 65536.0)
IH_CENTER = 131070  # 4 * 65535 / 2

_CHUNK = 1 << 22


def _mix64_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (used for keys only)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for byte in name.encode("utf-8"):
        h ^= byte
        h = (h * 0x100000001B3) & MASK64
    return h


def stream_key(seed: int, name: str) -> int:
    """64-bit key of the named tensor's stream."""
    return _mix64_int(_mix64_int((seed + 0x9E3779B97F4A7C15) & MASK64) ^ fnv1a64(name))


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * M1
    z = z ^ (z >> np.uint64(27))
    z = z * M2
    return z ^ (z >> np.uint64(31))


def u64(key: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of the stream with this key."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64_np(np.uint64(key) + idx * GAMMA)


def u64_at(key: int, index: np.ndarray) -> np.ndarray:
    """Outputs at arbitrary element indices (random access)."""
    idx = np.asarray(index, dtype=np.uint64) + np.uint64(1)
    with np.errstate(over="ignore"):
        return _mix64_np(np.uint64(key) + idx * GAMMA)


def _normal_from_u64(u: np.ndarray) -> np.ndarray:
    m16 = np.uint64(0xFFFF)
    s = (u & m16) + ((u >> np.uint64(16)) & m16) + ((u >> np.uint64(32)) & m16) + (u >> np.uint64(48))
    return (s.astype(np.int64) - IH_CENTER).astype(np.float32) * NORMAL_SCALE


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float32 -> bfloat16 bit pattern (uint16)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _transform(x: np.ndarray, scale, offset) -> np.ndarray:
    if scale is not None:
        x = x * np.float32(scale)
    if offset is not None:
        x = np.float32(offset) + x
    return x


def normal_f32(seed: int, name: str, shape, scale=None, offset=None, start: int = 0) -> np.ndarray:
    """float32 tensor: offset + scale * N(0,1)-approx, elements start.. of the stream."""
    n = int(np.prod(shape)) if len(shape) else 1
    key = stream_key(seed, name)
    out = np.empty(n, dtype=np.float32)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        out[c0:c1] = _transform(_normal_from_u64(u64(key, start + c0, c1 - c0)), scale, offset)
    return out.reshape(shape)


def normal_bf16(seed: int, name: str, shape, scale=None, offset=None, start: int = 0) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of the same numbers, rounded RNE."""
    return f32_to_bf16_bits(normal_f32(seed, name, shape, scale, offset, start)).reshape(shape)


def normal_bf16_at(seed: int, name: str, index: np.ndarray, scale=None, offset=None) -> np.ndarray:
    """Random access: bf16 bits of the elements at the given flat indices."""
    key = stream_key(seed, name)
    x = _transform(_normal_from_u64(u64_at(key, np.ravel(index))), scale, offset)
    return f32_to_bf16_bits(x).reshape(np.shape(index))


def random_subset_idx(seed: int, name: str, n_vis: np.ndarray, k: int) -> np.ndarray:
    """Per row r, k distinct entries of 0..n_vis[r]-1 (all of them if fewer),
    sorted ascending and padded with -1.  Row r draws its sort keys from
    elements r * 2**32 + s of the stream.  Returns int32 [rows, k]."""
    key = stream_key(seed, name)
    n_vis = np.asarray(n_vis, dtype=np.int64).ravel()
    out = np.full((n_vis.size, k), -1, dtype=np.int32)
    for r, n in enumerate(n_vis):
        n = int(n)
        if n <= 0:
            continue
        if n <= k:
            out[r, :n] = np.arange(n, dtype=np.int32)
            continue
        keys = u64(key, r << 32, n)
        pick = np.argpartition(keys, k - 1)[:k]
        out[r] = np.sort(pick).astype(np.int32)
    return out
