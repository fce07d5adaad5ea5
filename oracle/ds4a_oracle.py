"""Plain fp64 CPU oracle of the DeepSeek-V4 hybrid (CSA / HCA) attention path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import or run this module.
The CUDA library never calls it and shares no code with it; the two meet
only in the seeded generator (``gen/``), which holds no attention arithmetic.

Everything is float64, computed in the order the pages describe it, with no
tiling, no online softmax and no fusion.  numpy matmul and sort serve as
library steps.  Sources (page title, then section / equation):

[V4-inside]  "DeepSeek V4 Inside: One Token Through Every Block"
             (sections on layer-0 SWA, CSA, HCA, "What is stored").
[beyond]     "DeepSeek-v4 Beyond Basics", sections 3.2.2 (CSA, eqs. 9-17)
             and 3.3 (HCA, eqs. 20-27).
[module1]    "Phase 1 Module 1 - The model & the cost of attention",
             section "The indexer: a learned retrieval mechanism".
[hf-doc]     "DeepSeek-V4" (Transformers documentation), sections on hybrid
             attention and the attention-mask layout.

Readings taken where the pages are silent or garbled (each one is also
listed with its reason in the design notes):
 R1  compressor overlap: stream a covers the entry's own m tokens, stream b
     the previous block's m tokens; per channel one softmax over the 2m
     logits (m for entry 0 and for HCA).           -- parity unpinned
 R2  visibility is applied before top-k: entry s is visible to a query at
     position t iff s < floor((t + 1) / m).
 R3  top-k ties: higher score first, then lower index; the output lists the
     chosen indices ascending and pads with -1.
 R4  the index score has no scale, norm or RoPE: sum_h w_h ReLU(q_h . k).
 R5  softmax scale 1 / sqrt(head_dim).
 R6  RoPE on interleaved pairs (2j, 2j+1) of the last R dims, angle
     pos * base^(-2j/R), base 10000, no YaRN (the pages print only one pair
     at theta_0 = 1; the R = 64 ladder is pinned against an installed
     library's interleaved RoPE).
 R7  compressed entry i carries position i * m.      -- parity unpinned
 R8  RMSNorm eps 1e-6 with a learned gain after normalising; window K=V
     rows arrive in final form.
 R9  window = positions max(0, t - W + 1) .. t inclusive; no dedup with
     compressed entries.
 R10 positions are 0-based.
"""
from __future__ import annotations

import numpy as np


# --------------------------------------------------------------------------
# storage helpers
# --------------------------------------------------------------------------
def store_bf16(x) -> np.ndarray:
    """The ABI stores compressed entries as bfloat16: round (via float32,
    then round-to-nearest-even) and return the bit patterns (uint16).  Used
    by the oracle's own chain when one step's stored output feeds the next."""
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def widen(x) -> np.ndarray:
    """bfloat16 bit patterns (uint16) or float32 -> float64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


# --------------------------------------------------------------------------
# RMSNorm and partial interleaved RoPE
# [beyond] 3.3: RMSNorm on every query head and on the single compressed KV
# head; RoPE on the last 64 dims of each.  [V4-inside] layer-0 SWA: RoPE
# rotates the pair (x, y) at position i into (x cos - y sin, x sin + y cos).
# --------------------------------------------------------------------------
def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis (R8)."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def rope_frequencies(rope_dim: int, base: float) -> np.ndarray:
    """theta_j = base^(-2j/R), j = 0 .. R/2-1 (R6)."""
    j = np.arange(rope_dim // 2, dtype=np.float64)
    return base ** (-2.0 * j / rope_dim)


def rope(x: np.ndarray, pos, rope_dim: int, base: float) -> np.ndarray:
    """Rotate the interleaved pairs of the last ``rope_dim`` dims of x by
    angle pos * theta_j.  ``pos`` may be negative (the output de-rotation of
    [hf-doc] / paper eq. 26 uses position -i).  x: [..., D]; pos broadcasts
    against x[..., 0]."""
    x = np.array(x, dtype=np.float64, copy=True)
    if rope_dim == 0:
        return x
    D = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_frequencies(rope_dim, base)
    c, s = np.cos(ang), np.sin(ang)
    xe = x[..., D - rope_dim::2].copy()  # first of each pair
    xo = x[..., D - rope_dim + 1::2].copy()  # second of each pair
    x[..., D - rope_dim::2] = xe * c - xo * s
    x[..., D - rope_dim + 1::2] = xe * s + xo * c
    return x


# --------------------------------------------------------------------------
# (1) KV compressor
# [beyond] 3.2.2, eqs. 9-12: two token-level streams C^a, C^b with logits
# Z^a, Z^b; position biases B^a, B^b; softmax per channel along the rows
# that gather elements of both Z^a and Z^b; Hadamard-weighted sum; every m
# tokens give one entry.  [V4-inside] CSA: the blocks overlap, 2m weights
# normalised per block.  [beyond] 3.3, eqs. 20-23: HCA is the same with
# m' = 128 and a single stream, no overlap.
# --------------------------------------------------------------------------
def compress_entry(i: int, m: int, tok_begin: int, ca, za, ba, cb=None, zb=None, bb=None) -> np.ndarray:
    """Entry i (unnormalised) from float64 streams [T_tok, c] whose row 0 is
    absolute token ``tok_begin``.  a-half: tokens i*m + r (r < m) with logits
    Z^a + B^a[r]; b-half (CSA, i >= 1): tokens (i-1)*m + r with Z^b + B^b[r]
    (reading R1).  One softmax per channel over all the logits present."""
    logits, values = [], []
    for r in range(m):
        t = i * m + r - tok_begin
        logits.append(za[t] + ba[r])
        values.append(ca[t])
    if cb is not None and i >= 1:
        for r in range(m):
            t = (i - 1) * m + r - tok_begin
            logits.append(zb[t] + bb[r])
            values.append(cb[t])
    L = np.stack(logits)  # [n_terms, c]
    V = np.stack(values)
    L = L - L.max(axis=0, keepdims=True)
    e = np.exp(L)
    wgt = e / e.sum(axis=0, keepdims=True)
    return (wgt * V).sum(axis=0)


def compress(m: int, entry_begin: int, entry_end: int, tok_begin: int,
             ca, za, ba, cb=None, zb=None, bb=None,
             norm_g=None, rope_dim: int = 0, rope_base: float = 10000.0,
             eps: float = 1e-6) -> np.ndarray:
    """Entries entry_begin .. entry_end-1 of one sequence -> float64 [n, c].
    With ``norm_g``: RMSNorm(.) * g, then RoPE of the last ``rope_dim`` dims
    at the entry position i*m (readings R7, R8).  Without it (the indexer-key
    compressor of [beyond] 3.2.2 / [module1] "its own compressed stream"):
    the weighted sum only (reading R4)."""
    ca, za = widen(ca), widen(za)
    ba = widen(ba)
    if cb is not None:
        cb, zb, bb = widen(cb), widen(zb), widen(bb)
    out = []
    for i in range(entry_begin, entry_end):
        e = compress_entry(i, m, tok_begin, ca, za, ba, cb, zb, bb)
        if norm_g is not None:
            e = rms_norm(e, widen(norm_g), eps)
            e = rope(e, i * m, rope_dim, rope_base)
        out.append(e)
    if not out:
        return np.zeros((0, ca.shape[-1]))
    return np.stack(out)


# --------------------------------------------------------------------------
# (2) Lightning indexer and top-k selector
# [beyond] 3.2.2, eqs. 13-17; [module1] section on the indexer (every
# compressed row is scored; the selection prunes only when more than k
# entries are visible);
# [hf-doc] attention-mask layout: -1 sentinels, visibility w < (t+1)//m.
# --------------------------------------------------------------------------
def visible_entries(pos: int, m: int) -> int:
    """Number of compressed entries whose source tokens all lie at or before
    position ``pos``: floor((pos + 1) / m) (reading R2)."""
    return (int(pos) + 1) // int(m)


def index_scores(qi, wi, ki, n_vis: int) -> np.ndarray:
    """I_s = sum_h w_h * ReLU(q_h . K_s) for s < n_vis.
    qi [H_I, D_I], wi [H_I], ki [>= n_vis, D_I] -> float64 [n_vis]."""
    qi, wi, ki = widen(qi), widen(wi), widen(ki)
    dots = ki[:n_vis] @ qi.T  # [n_vis, H_I]
    return np.maximum(dots, 0.0) @ wi


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """Keep the k highest scores (reading R3: ties to the lower index);
    return their indices ascending, padded with -1 to length k.  When there
    are no more than k scores every index is kept."""
    n = scores.shape[0]
    order = np.lexsort((np.arange(n), -scores))  # primary: score desc
    chosen = np.sort(order[:k])
    out = np.full(k, -1, dtype=np.int64)
    out[: chosen.size] = chosen
    return out


def index_topk(qi, wi, ki, pos: int, m: int, k: int, n_c: int):
    """One query: (indices [k], scores of the visible entries)."""
    n_vis = min(visible_entries(pos, m), n_c)
    s = index_scores(qi, wi, ki, n_vis)
    return topk_select(s, k), s


# --------------------------------------------------------------------------
# (3)+(4) shared K=V MQA with sink, merged with the sliding window
# [beyond] 3.2.2 (the selected entries serve as both key and value, eq. 19)
# and 3.3 (eqs. 24-27); [V4-inside] layer-0 SWA sink example and the CSA
# "1 compressed + 2 window keys" example (one normaliser, sink in the
# denominator only); [hf-doc] output de-rotation by -i on the rope slice.
# --------------------------------------------------------------------------
def window_positions(pos: int, window: int) -> np.ndarray:
    """Positions max(0, pos - W + 1) .. pos (reading R9)."""
    return np.arange(max(0, int(pos) - window + 1), int(pos) + 1, dtype=np.int64)


def sink_softmax(z: np.ndarray, sink) -> tuple[np.ndarray, np.ndarray]:
    """p_j = exp(z_j) / (sum_k exp(z_k) + exp(sink)), per row of z [H, n];
    returns (p, sink mass exp(sink) / denominator).  A max shift keeps the
    exponentials finite; it cancels in the ratio."""
    z = np.asarray(z, dtype=np.float64)
    sink = np.asarray(sink, dtype=np.float64).reshape(-1, 1)
    mx = np.maximum(z.max(axis=1, keepdims=True) if z.shape[1] else -np.inf, sink)
    e = np.exp(z - mx)
    es = np.exp(sink - mx)
    den = e.sum(axis=1, keepdims=True) + es
    return e / den, (es / den)[:, 0]


def attend_rows(q, q_norm_g, rows, sink, pos: int, head_dim_scale: float,
                rope_dim: int, rope_base: float, eps: float) -> np.ndarray:
    """Core MQA for one query over explicit K=V rows [n, D]:
    q_hat = RoPE_pos(RMSNorm(q_h) * g); z = q_hat . kv * scale;
    p = sink_softmax(z); o = sum p kv; o = RoPE_{-pos}(o).  -> [H, D]."""
    q = widen(q)
    rows = widen(rows)
    qh = rope(rms_norm(q, widen(q_norm_g), eps), pos, rope_dim, rope_base)
    z = (qh @ rows.T) * head_dim_scale
    p, _ = sink_softmax(z, widen(sink))
    o = p @ rows
    return rope(o, -pos, rope_dim, rope_base)


def window_rows(win, win_cap: int, pos: int, window: int) -> np.ndarray:
    """K=V rows of the window read from a ring: slot = position mod win_cap."""
    return widen(win)[window_positions(pos, window) % win_cap]


def csa_attend(q, q_norm_g, pool, idx, win, win_cap: int, sink, pos: int, cfg) -> np.ndarray:
    """CSA: keys = pool[idx >= 0] followed by the window (one softmax)."""
    sel = np.asarray(idx)
    sel = sel[sel >= 0]
    rows = np.concatenate([widen(pool)[sel], window_rows(win, win_cap, pos, cfg.window)], axis=0)
    return attend_rows(q, q_norm_g, rows, sink, pos, cfg.sm_scale, cfg.rope_dim, cfg.rope_base, cfg.rms_eps)


def hca_attend(q, q_norm_g, pool, n_c: int, win, win_cap: int, sink, pos: int, cfg) -> np.ndarray:
    """HCA: keys = every visible pool entry followed by the window."""
    n_vis = min(visible_entries(pos, cfg.ratio), n_c)
    rows = np.concatenate([widen(pool)[:n_vis], window_rows(win, win_cap, pos, cfg.window)], axis=0)
    return attend_rows(q, q_norm_g, rows, sink, pos, cfg.sm_scale, cfg.rope_dim, cfg.rope_base, cfg.rms_eps)


def attended_key_count(pos: int, cfg, n_c: int, sparse: bool) -> int:
    """Keys one query scores: min(k, visible) + window (CSA) or visible +
    window (HCA); [V4-inside] "What does HCA change?" table."""
    n_vis = min(visible_entries(pos, cfg.ratio), n_c)
    n_win = window_positions(pos, cfg.window).size
    return (min(cfg.topk, n_vis) if sparse else n_vis) + n_win


# --------------------------------------------------------------------------
# (5) grouped low-rank output projection
# [beyond] 3.3 after eq. 26: the head outputs of a token, concatenated, are
# split into g groups of consecutive heads; each group is projected to an
# intermediate of rank r, and the g intermediates side by side are projected
# to the layer's output.  [V4-inside] layer-0 section: grouped W_O (Flash:
# 64 heads in 8 groups); [hf-doc]: grouped o_a projection, then o_b.
# --------------------------------------------------------------------------
def out_proj_mid(o, w_a, n_groups: int) -> np.ndarray:
    """o [M, H, D], w_a [g][r][(H/g) D] -> float64 [M, g r]: group j's
    intermediate is W_a[j] applied to the concatenation of its heads."""
    o = widen(o)
    M = o.shape[0]
    x = o.reshape(M, n_groups, -1)  # [M, g, (H/g) D], heads in order
    wa = widen(w_a)
    return np.concatenate([x[:, j] @ wa[j].T for j in range(n_groups)], axis=1)


def out_proj(o, w_a, w_b, n_groups: int):
    """(intermediate float64 [M, g r], output float64 [M, hidden]).  The
    intermediate goes through the ABI's bf16 storage before the second
    product (reading R12)."""
    mid = out_proj_mid(o, w_a, n_groups)
    y = widen(store_bf16(mid)) @ widen(w_b).T
    return mid, y


# --------------------------------------------------------------------------
# (6) block-scaled low-precision cache storage
# [V4-inside] "What does HCA change?" (paper 2.3.4): the K=V cache keeps its
# RoPE dims in BF16 and the other dims in FP8; the indexer keys are FP4.  The
# element formats and the block scaling follow the OCP Microscaling Formats
# (MX) specification v1.0: 32 consecutive values share one power-of-two
# scale X stored as E8M0 (exponent + 127); each value is V / X rounded to the
# nearest representable element (ties to the even code).  FP8 is E4M3 (bias
# 7, largest 448), FP4 is E2M1 (bias 1, largest 6).  Readings: blocks of 32
# along the channel axis; X is the smallest power of two with max |V| / X
# within the element format's range (the specification's floor rule,
# 2^(floor(log2 max|V|) - emax), would clip a block's largest values by up
# to 12 %), so no element saturates; an all-zero block takes scale code 0.
# --------------------------------------------------------------------------
MX_BLOCK = 32
_FMT = {"e4m3": dict(ebits=4, mbits=3, bias=7, ncodes=127),   # 0x7F is NaN
        "e2m1": dict(ebits=2, mbits=1, bias=1, ncodes=8)}


def format_values(fmt: str) -> np.ndarray:
    """Magnitude of every non-negative code of an element format, by code."""
    f = _FMT[fmt]
    out = []
    for code in range(f["ncodes"]):
        e, m = code >> f["mbits"], code & ((1 << f["mbits"]) - 1)
        if e == 0:  # subnormal
            out.append(m / (1 << f["mbits"]) * 2.0 ** (1 - f["bias"]))
        else:
            out.append((1 + m / (1 << f["mbits"])) * 2.0 ** (e - f["bias"]))
    return np.array(out)


def round_to_format(x, fmt: str) -> np.ndarray:
    """Codes (sign in the bit above the magnitude code) of x rounded to the
    nearest value of the format, ties to the even code, magnitudes clamped
    to the largest normal.  As in IEEE rounding, the sign is kept: a
    negative value that rounds to zero gives negative zero."""
    f = _FMT[fmt]
    grid = format_values(fmt)
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), grid[-1])
    hi = np.clip(np.searchsorted(grid, a), 1, grid.size - 1)
    lo = hi - 1
    dlo, dhi = a - grid[lo], grid[hi] - a
    code = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    sign_bit = 1 << (f["ebits"] + f["mbits"])
    return (code + np.where(np.signbit(x), sign_bit, 0)).astype(np.uint8)


def format_value(codes, fmt: str) -> np.ndarray:
    f = _FMT[fmt]
    sign_bit = 1 << (f["ebits"] + f["mbits"])
    codes = np.asarray(codes).astype(np.int64)
    mag = format_values(fmt)[codes & (sign_bit - 1)]
    return np.where(codes & sign_bit, -mag, mag)


def mx_quantize(x, fmt: str):
    """x [..., n] (n a multiple of 32) -> (element codes uint8 [..., n],
    E8M0 scale codes uint8 [..., n/32])."""
    x = np.asarray(x, dtype=np.float64)
    blocks = x.reshape(*x.shape[:-1], -1, MX_BLOCK)
    amax = np.abs(blocks).max(axis=-1)
    # smallest s with amax <= largest * 2^s, exactly: with amax = f 2^k and
    # largest = g 2^j (f, g in [0.5, 1)), s = k - j, plus one when f > g
    f, k = np.frexp(amax)
    g, j = np.frexp(format_values(fmt)[-1])
    shared = np.clip(k - j + (f > g), -127, 127)
    shared = np.where(amax > 0, shared, -127)
    q = blocks / np.exp2(shared)[..., None]
    codes = round_to_format(q, fmt).reshape(x.shape)
    return codes, (shared + 127).astype(np.uint8)


def mx_dequantize(codes, scales, fmt: str) -> np.ndarray:
    v = format_value(codes, fmt)
    v = v.reshape(*v.shape[:-1], -1, MX_BLOCK)
    return (v * np.exp2(np.asarray(scales, dtype=np.float64) - 127.0)[..., None]).reshape(np.shape(codes))


def kv_fp8_row_bytes(D: int, R: int) -> int:
    """Bytes of one mixed K=V row: D - R FP8 codes, R BF16 values, (D - R)/32
    scales, padded to a multiple of 16."""
    n = D - R
    return (n + 2 * R + n // MX_BLOCK + 15) // 16 * 16


def quantize_kv_fp8(rows, D: int, R: int) -> np.ndarray:
    """bf16 K=V rows (uint16 bits or floats) [..., D] -> byte rows: FP8 codes
    of the first D - R dims, the last R dims as stored bf16 (little endian),
    the E8M0 scales, zero padding."""
    bits = np.asarray(rows)
    if bits.dtype != np.uint16:
        bits = store_bf16(bits)
    n = D - R
    codes, scales = mx_quantize(widen(bits[..., :n]), "e4m3")
    out = np.zeros(bits.shape[:-1] + (kv_fp8_row_bytes(D, R),), np.uint8)
    out[..., :n] = codes
    out[..., n:n + 2 * R] = np.ascontiguousarray(bits[..., n:]).view(np.uint8).reshape(bits.shape[:-1] + (2 * R,))
    out[..., n + 2 * R:n + 2 * R + n // MX_BLOCK] = scales
    return out


def dequantize_kv_fp8(qrows, D: int, R: int) -> np.ndarray:
    q = np.asarray(qrows, dtype=np.uint8)
    n = D - R
    nope = mx_dequantize(q[..., :n], q[..., n + 2 * R:n + 2 * R + n // MX_BLOCK], "e4m3")
    rope_bits = np.ascontiguousarray(q[..., n:n + 2 * R]).view(np.uint16)
    return np.concatenate([nope, widen(rope_bits)], axis=-1)


def quantize_idx_fp4(keys):
    """bf16 indexer keys [..., D] -> (packed E2M1 codes uint8 [..., D/2], even
    element in the low nibble; E8M0 scales uint8 [..., D/32])."""
    bits = np.asarray(keys)
    if bits.dtype != np.uint16:
        bits = store_bf16(bits)
    codes, scales = mx_quantize(widen(bits), "e2m1")
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, scales


def dequantize_idx_fp4(packed, scales) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    codes = np.stack([p & 15, p >> 4], axis=-1).reshape(*p.shape[:-1], 2 * p.shape[-1])
    return mx_dequantize(codes, scales, "e2m1")


# --------------------------------------------------------------------------
# batch drivers (loops over sequences and queries)
# --------------------------------------------------------------------------
def index_topk_batch(qi, wi, ki, q_pos, m: int, k: int, n_c: int, rows=None):
    """qi [B,T,H_I,D_I], wi [B,T,H_I], ki [B,N_c,D_I], q_pos [B,T] ->
    idx int64 [B,T,k] and a dict (b,t) -> scores.  ``rows`` limits the work
    to a list of (b, t)."""
    B, T = np.asarray(q_pos).shape
    idx = np.full((B, T, k), -1, dtype=np.int64)
    scores = {}
    todo = rows if rows is not None else [(b, t) for b in range(B) for t in range(T)]
    for b, t in todo:
        idx[b, t], scores[(b, t)] = index_topk(qi[b, t], wi[b, t], ki[b], int(q_pos[b][t]), m, k, n_c)
    return idx, scores


def csa_attend_batch(q, q_norm_g, pool, idx, win, win_cap, sink, q_pos, cfg, rows=None):
    B, T = np.asarray(q_pos).shape
    out = np.zeros(q.shape, dtype=np.float64)
    todo = rows if rows is not None else [(b, t) for b in range(B) for t in range(T)]
    for b, t in todo:
        out[b, t] = csa_attend(q[b, t], q_norm_g, pool[b], idx[b, t], win[b], win_cap, sink, int(q_pos[b][t]), cfg)
    return out


def hca_attend_batch(q, q_norm_g, pool, n_c, win, win_cap, sink, q_pos, cfg, rows=None):
    B, T = np.asarray(q_pos).shape
    out = np.zeros(q.shape, dtype=np.float64)
    todo = rows if rows is not None else [(b, t) for b in range(B) for t in range(T)]
    for b, t in todo:
        out[b, t] = hca_attend(q[b, t], q_norm_g, pool[b], n_c, win[b], win_cap, sink, int(q_pos[b][t]), cfg)
    return out


def compress_batch(m, entry_begin, entry_end, tok_begin, ca, za, ba, cb=None, zb=None, bb=None,
                   norm_g=None, rope_dim=0, rope_base=10000.0, eps=1e-6) -> np.ndarray:
    """Streams [B, T_tok, c] -> entries float64 [B, n, c]."""
    B = np.asarray(ca).shape[0]
    outs = []
    for b in range(B):
        outs.append(compress(m, entry_begin, entry_end, tok_begin, ca[b], za[b], ba,
                             None if cb is None else cb[b], None if zb is None else zb[b], bb,
                             norm_g, rope_dim, rope_base, eps))
    return np.stack(outs)
