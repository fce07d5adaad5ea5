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
* N(0, 1) by inverse transform: bit 63 of an output is the sign; the
  other 63 bits v (v = 0 read as 1) give the tail probability p = v / 2^64
  in (0, 1/2).  The leading one of v selects an octave e (p in
  [2^-(e+2), 2^-(e+1)), e = 0 .. 62), the next 8 bits one of 256 segments of
  that octave and the 23 bits after them a fraction f in [0, 1).  |x| =
  T[e][s] + f * D[e][s] with T[e][s] = -ndtri((1 + s/256) 2^-(e+2)) (the
  normal quantile at the segment's start, float32) and D[e][s] =
  T[e][s+1] - T[e][s] (float32 subtraction): a piecewise-linear inverse
  normal CDF whose nodes are exact to float32 and whose interpolation error
  is below 1e-6 everywhere, with tails out to p = 2^-64 (|x| about 9.1).
  The table is computed once on the host (float64 ``scipy.special.ndtri``)
  and handed to the device generator, so both sides read the same numbers;
  the lookup is integer work and the interpolation is one correctly rounded
  float32 multiply and one add, so host and device agree bit for bit.
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

NORMAL_SEGMENTS = 256
NORMAL_OCTAVES = 63
_TABLE = None


def normal_table() -> np.ndarray:
    """float32 [63, 256, 2]: (T, D) of every segment of every octave."""
    global _TABLE
    if _TABLE is None:
        from scipy.special import ndtri

        e = np.arange(NORMAL_OCTAVES, dtype=np.float64)[:, None]
        s = np.arange(NORMAL_SEGMENTS + 1, dtype=np.float64)[None, :]
        p = (1.0 + s / NORMAL_SEGMENTS) * np.exp2(-(e + 2.0))
        t = (-ndtri(p)).astype(np.float32)
        tab = np.empty((NORMAL_OCTAVES, NORMAL_SEGMENTS, 2), np.float32)
        tab[:, :, 0] = t[:, :-1]
        tab[:, :, 1] = t[:, 1:] - t[:, :-1]  # float32 subtraction
        _TABLE = tab
    return _TABLE


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
    u = np.asarray(u, dtype=np.uint64)
    tab = normal_table()
    v = np.maximum(u & np.uint64(0x7FFFFFFFFFFFFFFF), np.uint64(1))
    # floor(log2 v) by integer halving steps (no float rounding)
    bl = np.zeros(v.shape, dtype=np.int64)
    t = v.copy()
    for sh in (32, 16, 8, 4, 2, 1):
        big = t >= np.uint64(1 << sh)
        t = np.where(big, t >> np.uint64(sh), t)
        bl += big.astype(np.int64) * sh
    e = 62 - bl
    w = v << e.astype(np.uint64)
    seg = ((w >> np.uint64(54)) & np.uint64(0xFF)).astype(np.int64)
    f = ((w >> np.uint64(31)) & np.uint64(0x7FFFFF)).astype(np.float32) * np.float32(2.0 ** -23)
    td = tab[e, seg]
    x = td[..., 0] + f * td[..., 1]  # float32 multiply, then float32 add
    return np.where((u >> np.uint64(63)) != 0, -x, x).astype(np.float32)


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
