"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each pin takes the oracle module ``O`` as its argument and raises
AssertionError when the oracle disagrees.  ``test_oracle_pins`` runs them on
the oracle; ``test_oracle_mutants`` runs them on copies of the oracle with
planted mistakes and expects at least one to fail for each.

Sources of the fixed values: ``tests/golden/page_numbers.json`` (numbers
printed on the pages, each with its citation), closed forms, invariants, and
library routines (torch's scaled_dot_product_attention and rms_norm, in
float64 on the CPU) for the special cases that reduce to them.
"""
from __future__ import annotations

import dataclasses
import json
import math
import os

import numpy as np
import torch

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")))


@dataclasses.dataclass(frozen=True)
class Cfg:
    n_heads: int = 1
    head_dim: int = 4
    rope_dim: int = 0
    window: int = 2
    idx_heads: int = 1
    idx_dim: int = 4
    topk: int = 4
    ratio: int = 2
    rope_base: float = 10000.0
    rms_eps: float = 1e-6

    @property
    def sm_scale(self):
        return 1.0 / math.sqrt(self.head_dim)


def _close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert a.shape == b.shape and err <= tol, f"{what}: {a} vs {b} (err {err:.3g} > {tol})"


# --------------------------------------------------------------------------
# printed numbers
# --------------------------------------------------------------------------
def pin_swa_sink_example(O):
    g = GOLDEN["swa_sink_example"]
    p, sm = O.sink_softmax(np.array([g["logits"]]), [g["sink"]])
    _close(p[0], g["weights"], 1.5e-4, "SWA sink weights")
    _close(sm[0], g["sink_mass"], 1.5e-4, "SWA sink mass")
    # the logits are q.k times 1/sqrt(head_dim) = 0.5
    _close(np.array(g["qk"]) / math.sqrt(g["head_dim"]), g["logits"], 0.6e-4, "SWA scale")


def _marker_rows(logits, scale):
    """K=V rows whose only non-zero dim j carries 2*z_j, so that with the
    all-ones query (RMS 1, gain 1, head dim 4, scale 1/2) the logit of row j
    is z_j and output dim j is p_j * 2 z_j."""
    rows = np.zeros((len(logits), 4))
    for j, z in enumerate(logits):
        rows[j, j] = z / scale / 1.0
    return rows


def pin_csa_joint_example(O):
    """1 compressed entry + 2 window keys share one normaliser with the sink
    (printed example); checked through the oracle's csa_attend."""
    g = GOLDEN["csa_joint_example"]
    cfg = Cfg(window=2)
    z = g["logits_compressed_then_window"]
    rows = _marker_rows(z, cfg.sm_scale)
    pos, cap = 4, 8
    pool = rows[:1]
    win = np.zeros((cap, 4))
    win[(pos - 1) % cap] = rows[1]
    win[pos % cap] = rows[2]
    q = np.ones((1, 4))
    o = O.csa_attend(q, np.ones(4), pool, np.array([0, -1, -1, -1]), win, cap, [g["sink"]], pos, cfg)
    p = o[0, :3] / (np.array(z) / cfg.sm_scale)
    _close(p, g["weights"], 1.5e-4, "CSA joint weights")
    _close(1.0 - p.sum(), g["sink_mass"], 1.5e-3, "CSA sink mass")  # printed with 3 decimals


def pin_swa_example_through_attend(O):
    """The 2-key SWA example through hca_attend with no compressed entries
    (the window holds the previous token and the query's own token)."""
    g = GOLDEN["swa_sink_example"]
    cfg = Cfg(window=2, ratio=4)
    rows = _marker_rows(g["logits"], cfg.sm_scale)
    pos, cap = 3, 4
    win = np.zeros((cap, 4))
    win[(pos - 1) % cap] = rows[0]
    win[pos % cap] = rows[1]
    o = O.hca_attend(np.ones((1, 4)), np.ones(4), np.zeros((0, 4)), 0, win, cap, [g["sink"]], pos, cfg)
    p = o[0, :2] / (np.array(g["logits"]) / cfg.sm_scale)
    _close(p, g["weights"], 1.5e-4, "SWA weights via attend")


def pin_rope_example(O):
    g = GOLDEN["rope_example"]
    x = np.array(g["q_head1"])
    y = O.rope(x, g["position"], 2, 10000.0)
    _close(y[:2], x[:2], 0.0, "RoPE leaves non-rope dims")
    _close(y[2:], g["rotated_last_pair"], 1e-4, "RoPE rotation at i=3")
    # theta_0 = 1 for the first pair: a unit vector lands on (cos 3, sin 3)
    e = np.zeros(4)
    e[2] = 1.0
    _close(O.rope(e, 3, 2, 10000.0)[2:], [g["cos"], g["sin"]], 1e-4, "RoPE cos/sin at 3")


def pin_rope_dot_at_equal_positions(O):
    """q.k printed for p with itself (0.0749) is unchanged when q and k are
    rotated at the same position."""
    g = GOLDEN["rope_example"]
    q, k = np.array(g["q_head1"]), np.array(g["k_head1"])
    _close(q @ k, g["qk_p_with_itself"], 1e-4, "q.k")
    for pos in (3, 17, -5):
        _close(O.rope(q, pos, 2, 10000.0) @ O.rope(k, pos, 2, 10000.0), g["qk_p_with_itself"], 1e-4,
               "q.k after equal rotations")


def pin_rope_pairs_interleaved(O):
    """Interleaved pairs (2j, 2j+1) of the last R dims rotate together; the
    rotation is norm preserving and RoPE_{-p} undoes RoPE_p."""
    D, R = 12, 8
    for j in range(R // 2):
        e = np.zeros(D)
        e[D - R + 2 * j] = 1.0
        y = O.rope(e, 5, R, 10000.0)
        mask = np.ones(D, bool)
        mask[D - R + 2 * j: D - R + 2 * j + 2] = False
        assert np.all(y[mask] == 0.0), f"pair {j} leaks into other dims: {y}"
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, D))
    y = O.rope(x, np.array([0, 7, -11]), R, 10000.0)
    _close(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), 1e-12, "RoPE norm")
    _close(O.rope(y, -np.array([0, 7, -11]), R, 10000.0), x, 1e-12, "RoPE inverse")
    _close(O.rope(x, 0, R, 10000.0), x, 0.0, "RoPE at 0")


_LIB_ROPE: dict = {}


def _library_rope(x, positions, base):
    """Interleaved-pair RoPE as the installed transformers library computes
    it for DeepSeek-V2 (its rotary embedding's default frequencies and its
    complex-pair rotation), in float32: x [n, d] at positions [n]."""
    key = (x.tobytes(), positions.tobytes(), base)
    if key not in _LIB_ROPE:
        from transformers import DeepseekV2Config
        from transformers.models.deepseek_v2 import modeling_deepseek_v2 as M

        d = x.shape[-1]
        cfg = DeepseekV2Config(qk_rope_head_dim=d, rope_theta=base)
        rot = M.DeepseekV2RotaryEmbedding(cfg)
        xt = torch.from_numpy(x.astype(np.float32))[None, None]  # [1, 1, n, d]
        fc = rot(xt, torch.from_numpy(positions.astype(np.int64))[None])
        y, _ = M.apply_rotary_emb(xt, xt, fc)
        _LIB_ROPE[key] = y[0, 0].double().numpy()
    return _LIB_ROPE[key]


def pin_rope_ladder_library(O):
    """At the Flash rope width (R = 64, base 10000) the oracle's rotation of
    the last R dims matches an installed library's interleaved-pair RoPE
    (transformers, DeepSeek-V2), which fixes every pair's frequency
    (RoFormer, Su et al. 2021, eq. 15: theta_j = base^(-2j/d)); the leading
    D - R dims stay untouched."""
    R, D = 64, 80
    rng = np.random.default_rng(15)
    positions = np.array([0, 1, 3, 17, 100, 1000, 4097])
    x = rng.standard_normal((positions.size, D))
    got = O.rope(x, positions, R, 10000.0)
    _close(got[:, : D - R], x[:, : D - R], 0.0, "RoPE leaves the leading dims")
    _close(got[:, D - R:], _library_rope(x[:, D - R:], positions, 10000.0), 2e-3, "RoPE vs library, R=64")


def pin_store_bf16_library(O):
    """The oracle's bfloat16 storage rounding equals torch's float32 ->
    bfloat16 conversion (round to nearest, ties to even), including exact
    halfway cases and values next to them."""
    rng = np.random.default_rng(16)
    x = (rng.standard_normal(4096) * np.exp2(rng.integers(-20, 20, 4096))).astype(np.float32)
    hi = rng.integers(0, 1 << 15, 512, dtype=np.uint32) << np.uint32(16)
    edge = np.concatenate([hi | np.uint32(0x8000), hi | np.uint32(0x10000 | 0x8000), hi | np.uint32(0x7FFF),
                           hi | np.uint32(0x8001), hi | np.uint32(0x80000000 | 0x8000)]).view(np.float32)
    x = np.concatenate([x, edge, np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.store_bf16(x)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, f"store_bf16 differs from torch at {bad.size} values, e.g. {x[bad[:3]]}"
    _close(O.widen(got), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy(), 0.0,
           "widen of bf16 bits")


def pin_rms_norm_library(O):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 16)) * 3.0
    g = 1.0 + 0.1 * rng.standard_normal(16)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (16,), torch.from_numpy(g), eps=1e-6).numpy()
    _close(O.rms_norm(x, g, 1e-6), ref, 1e-12, "RMSNorm vs torch.rms_norm")


# --------------------------------------------------------------------------
# counts and visibility
# --------------------------------------------------------------------------
def pin_toy_cache_counts(O):
    g = GOLDEN["toy_cache_counts"]
    last = g["tokens"] - 1
    assert O.visible_entries(last, g["csa_m"]) == g["csa_entries"]
    assert O.visible_entries(last, g["hca_m"]) == g["hca_entries"]
    assert O.window_positions(last, g["window"]).size == g["window_entries"]
    # "p sees the previous e and itself": window 2 at position 3 is {2, 3}
    assert list(O.window_positions(3, 2)) == [2, 3]
    assert list(O.window_positions(0, 4)) == [0]


def pin_hca_toy_visibility(O):
    g = GOLDEN["hca_toy_visibility"]
    assert O.visible_entries(g["query_position_0based"], g["hca_m"]) == g["visible_entries"]


def pin_hf_mask_rules(O):
    g = GOLDEN["hf_mask_rules"]
    m = g["hca_m"]
    first0 = min(t for t in range(64) if O.visible_entries(t, m) >= 1)
    first1 = min(t for t in range(64) if O.visible_entries(t, m) >= 2)
    assert (first0, first1) == (g["entry0_first_visible_t"], g["entry1_first_visible_t"]), (first0, first1)
    mc = g["csa_m"]
    firstc = min(t for t in range(64) if O.visible_entries(t, mc) >= 1)
    assert firstc == g["csa_first_query_with_entries"], firstc


def pin_entries_per_query_1m(O):
    g = GOLDEN["entries_per_query_1m"]
    pos = g["context"] - 1
    csa = Cfg(ratio=g["csa_m"], topk=g["topk"], window=g["window"])
    hca = Cfg(ratio=g["hca_m"], topk=g["topk"], window=g["window"])
    n_csa = O.visible_entries(pos, g["csa_m"])
    n_hca = O.visible_entries(pos, g["hca_m"])
    assert O.attended_key_count(pos, csa, n_csa, True) == g["csa"]
    assert O.attended_key_count(pos, hca, n_hca, False) == g["hca"]
    assert O.window_positions(pos, g["window"]).size == g["swa"]
    assert pos + 1 == g["dense"]


# --------------------------------------------------------------------------
# indexer and top-k
# --------------------------------------------------------------------------
def pin_indexer_prunes(O):
    g = GOLDEN["indexer_prunes"]
    rng = np.random.default_rng(3)
    for n, kept in ((g["rows_small"], g["kept_small"]), (g["rows_large"], g["kept_large"])):
        s = rng.standard_normal(n)
        idx = O.topk_select(s, g["topk"])
        sel = idx[idx >= 0]
        assert sel.size == kept
        if n <= g["topk"]:
            assert np.array_equal(sel, np.arange(n))


def pin_topk_definition(O):
    """Every kept score >= every dropped score; output ascending, -1 padded;
    equal scores go to the lower index."""
    rng = np.random.default_rng(4)
    s = np.round(rng.standard_normal(300), 1)  # many ties
    k = 37
    idx = O.topk_select(s, k)
    assert idx.size == k and np.all(np.diff(idx) > 0)
    kept = np.zeros(s.size, bool)
    kept[idx] = True
    assert s[kept].min() >= s[~kept].max()
    thr = s[kept].min()
    ties = np.flatnonzero(s == thr)
    kept_ties = np.flatnonzero(kept & (s == thr))
    assert np.array_equal(kept_ties, ties[: kept_ties.size]), "ties must go to the lower index"
    flat = O.topk_select(np.zeros(10), 4)
    assert list(flat) == [0, 1, 2, 3]
    short = O.topk_select(np.array([0.5, -1.0]), 4)
    assert list(short) == [0, 1, -1, -1]
    assert list(O.topk_select(np.zeros(0), 3)) == [-1, -1, -1]


def pin_index_score_special_cases(O):
    rng = np.random.default_rng(5)
    H, D, N = 3, 6, 40
    k = rng.standard_normal((N, D))
    q = rng.standard_normal((H, D))
    # one-hot head weight: ReLU of that head's dot product
    w = np.array([0.0, 1.0, 0.0])
    _close(O.index_scores(q, w, k, N), np.maximum(k @ q[1], 0.0), 1e-12, "one-hot head")
    # non-negative operands, unit weights: the sum over heads can move inside
    qp, kp = np.abs(q), np.abs(k)
    _close(O.index_scores(qp, np.ones(H), kp, N), kp @ qp.sum(axis=0), 1e-12, "linear case")
    # a negative head weight subtracts; negative dot products contribute 0
    w2 = np.array([-2.0, 0.0, 0.0])
    _close(O.index_scores(-qp, w2, kp, N), np.zeros(N), 0.0, "ReLU kills negative dots")
    _close(O.index_scores(qp, w2, kp, N), -2.0 * (kp @ qp[0]), 1e-12, "negative weight")
    # only visible entries are scored
    assert O.index_scores(q, w, k, 7).shape == (7,)


def pin_index_topk_visibility(O):
    """Entries past the visible count are never selected, whatever their
    scores (selection after masking)."""
    rng = np.random.default_rng(6)
    N, D = 32, 4
    k = rng.standard_normal((N, D))
    k[20:] *= 100.0  # future entries score highest
    q = rng.standard_normal((2, D))
    idx, s = O.index_topk(q, np.ones(2), k, pos=41, m=2, k=8, n_c=N)
    assert s.shape == (21,)
    assert idx.max() <= 20
    idx0, s0 = O.index_topk(q, np.ones(2), k, pos=0, m=2, k=8, n_c=N)
    assert s0.size == 0 and np.all(idx0 == -1)


# --------------------------------------------------------------------------
# attention reductions
# --------------------------------------------------------------------------
def _sdpa_with_sink(qhat, rows, sink, scale):
    """torch SDPA with one extra key whose logit is the sink and value 0."""
    H, D = qhat.shape
    qa = np.concatenate([qhat, np.ones((H, 1))], axis=1)
    outs = []
    for h in range(H):
        ka = np.concatenate([np.concatenate([rows, np.zeros((rows.shape[0], 1))], axis=1),
                             np.concatenate([np.zeros((1, D)), [[sink[h] / scale]]], axis=1)], axis=0)
        va = np.concatenate([rows, np.zeros((1, D))], axis=0)
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qa[h][None, None, None]), torch.from_numpy(ka[None, None]),
            torch.from_numpy(va[None, None]), scale=scale)
        outs.append(o[0, 0, 0].numpy())
    return np.stack(outs)


def pin_attend_vs_library(O):
    """With R = 0, attend_rows equals torch SDPA on the RMS-normalised query
    with the sink as a zero-valued extra key; with sink -> -inf it is plain
    softmax attention."""
    rng = np.random.default_rng(7)
    H, D, n = 3, 16, 11
    q = rng.standard_normal((H, D)) * 2.0
    g = 1.0 + 0.1 * rng.standard_normal(D)
    rows = rng.standard_normal((n, D))
    sink = rng.standard_normal(H)
    scale = 1.0 / math.sqrt(D)
    qhat = torch.nn.functional.rms_norm(torch.from_numpy(q), (D,), torch.from_numpy(g), eps=1e-6).numpy()
    got = O.attend_rows(q, g, rows, sink, 5, scale, 0, 10000.0, 1e-6)
    _close(got, _sdpa_with_sink(qhat, rows, sink, scale), 1e-12, "attend vs SDPA+sink")
    got = O.attend_rows(q, g, rows, np.full(H, -np.inf), 5, scale, 0, 10000.0, 1e-6)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qhat[None, :, None]), torch.from_numpy(np.broadcast_to(rows, (H, n, D))[None].copy()),
        torch.from_numpy(np.broadcast_to(rows, (H, n, D))[None].copy()), scale=scale)[0, :, 0].numpy()
    _close(got, ref, 1e-12, "attend vs SDPA (no sink)")


def pin_attend_relative_positions(O):
    """Keys rotated at their own positions, the query at t, output rotated
    back by -t: the result depends only on relative distances, so shifting
    every position by the same amount leaves it unchanged."""
    rng = np.random.default_rng(8)
    H, D, R, n = 2, 16, 8, 9
    q = rng.standard_normal((H, D))
    g = np.ones(D)
    k = rng.standard_normal((n, D))
    kpos = np.array([0, 4, 8, 12, 16, 30, 31, 32, 33])
    t = 33
    sink = np.array([0.3, -0.7])
    outs = []
    for shift in (0, 57, 1000):
        rows = O.rope(k, kpos + shift, R, 10000.0)
        outs.append(O.attend_rows(q, g, rows, sink, t + shift, 1 / math.sqrt(D), R, 10000.0, 1e-6))
    _close(outs[1], outs[0], 1e-9, "shift 57")
    _close(outs[2], outs[0], 1e-9, "shift 1000")


def _rand_layer(rng, cfg, n_c, cap):
    D = cfg.head_dim
    return (rng.standard_normal((cfg.n_heads, D)), 1 + 0.1 * rng.standard_normal(D),
            rng.standard_normal((n_c, D)), rng.standard_normal((cap, D)), rng.standard_normal(cfg.n_heads))


def pin_hca_equals_csa_all_visible(O):
    rng = np.random.default_rng(9)
    cfg = Cfg(n_heads=2, head_dim=8, rope_dim=4, window=3, ratio=4, topk=64)
    q, g, pool, win, sink = _rand_layer(rng, cfg, 16, 8)
    for pos in (0, 2, 3, 9, 40, 63):
        n_vis = min(O.visible_entries(pos, 4), 16)
        idx = np.full(cfg.topk, -1)
        idx[:n_vis] = np.arange(n_vis)
        a = O.hca_attend(q, g, pool, 16, win, 8, sink, pos, cfg)
        b = O.csa_attend(q, g, pool, idx, win, 8, sink, pos, cfg)
        _close(a, b, 1e-12, f"HCA == CSA(all visible) at {pos}")


def pin_csa_k_ge_nc_is_dense(O):
    """Top-k with k >= entries keeps every visible entry, so CSA equals dense
    attention over the visible pool plus the window."""
    rng = np.random.default_rng(10)
    cfg = Cfg(n_heads=2, head_dim=8, rope_dim=4, window=3, ratio=2, topk=40, idx_heads=3, idx_dim=5)
    q, g, pool, win, sink = _rand_layer(rng, cfg, 20, 64)
    qi, wi, ki = rng.standard_normal((3, 5)), rng.standard_normal(3), rng.standard_normal((20, 5))
    for pos in (1, 5, 30, 39):
        idx, _ = O.index_topk(qi, wi, ki, pos, cfg.ratio, cfg.topk, 20)
        a = O.csa_attend(q, g, pool, idx, win, 64, sink, pos, cfg)
        b = O.hca_attend(q, g, pool, 20, win, 64, sink, pos, cfg)
        _close(a, b, 1e-12, f"CSA(k>=N) == dense at {pos}")


def pin_window_ring_slots(O):
    """The window reads slot pos mod capacity: a ring of capacity W and a
    full token array give the same result."""
    rng = np.random.default_rng(11)
    cfg = Cfg(n_heads=2, head_dim=8, rope_dim=2, window=4, ratio=2)
    q, g, pool, full, sink = _rand_layer(rng, cfg, 8, 40)
    pos = 37
    ring = np.zeros((4, 8))
    for p in range(pos - 3, pos + 1):
        ring[p % 4] = full[p]
    a = O.csa_attend(q, g, pool, np.array([1, 5, -1, -1]), full, 40, sink, pos, cfg)
    b = O.csa_attend(q, g, pool, np.array([1, 5, -1, -1]), ring, 4, sink, pos, cfg)
    _close(a, b, 0.0, "ring vs full")


def pin_csa_gathers_by_index(O):
    """The CSA keys are the pool rows the indices name, wherever they sit:
    moving those rows to the front and renumbering gives the same output."""
    rng = np.random.default_rng(14)
    cfg = Cfg(n_heads=2, head_dim=8, rope_dim=2, window=2, ratio=2, topk=4)
    q, g, pool, win, sink = _rand_layer(rng, cfg, 12, 16)
    pos = 23
    a = O.csa_attend(q, g, pool, np.array([2, 5, 9, -1]), win, 16, sink, pos, cfg)
    moved = np.concatenate([pool[[2, 5, 9]], pool[:9]], axis=0)
    b = O.csa_attend(q, g, moved, np.array([0, 1, 2, -1]), win, 16, sink, pos, cfg)
    _close(a, b, 0.0, "gather by index")
    c = O.csa_attend(q, g, pool, np.array([0, 1, 2, -1]), win, 16, sink, pos, cfg)
    assert np.max(np.abs(a - c)) > 1e-6, "different rows must give a different output"


# --------------------------------------------------------------------------
# compressor
# --------------------------------------------------------------------------
def _token_streams(T, c):
    """Value of token t in every channel is t (stream a) or 1000 + t (b)."""
    ca = np.tile(np.arange(T, dtype=np.float64)[:, None], (1, c))
    return ca, ca + 1000.0


def pin_compress_equal_logits_is_mean(O):
    """With all logits equal every term weighs the same: CSA entry i >= 1 is
    the mean of its own block (stream a) and the previous block (stream b),
    entry 0 the mean of block 0; HCA entry i the mean of block i."""
    T, c, m = 24, 3, 4
    ca, cb = _token_streams(T, c)
    z = np.zeros((T, c))
    b = np.zeros((m, c))
    e = O.compress(m, 0, T // m, 0, ca, z, b, cb, z, b)
    assert e.shape == (T // m, c)
    _close(e[0], np.full(c, (m - 1) / 2), 1e-12, "CSA entry 0")
    for i in range(1, T // m):
        want = (np.mean(np.arange(i * m, (i + 1) * m)) + np.mean(1000 + np.arange((i - 1) * m, i * m))) / 2
        _close(e[i], np.full(c, want), 1e-12, f"CSA entry {i}")
    h = O.compress(m, 0, T // m, 0, ca, z, b)
    for i in range(T // m):
        _close(h[i], np.full(c, i * m + (m - 1) / 2), 1e-12, f"HCA entry {i}")


def pin_compress_dominant_logit_copies(O):
    """A logit far above the others in one channel makes that channel copy
    the matching token of the matching stream; a large position bias does the
    same for its slot in every block."""
    T, c, m = 16, 4, 2
    ca, cb = _token_streams(T, c)
    z = np.zeros((T, c))
    za = z.copy()
    za[5, 2] = 80.0  # token 5, channel 2, stream a -> entry 2 (own block 4..5)
    b0 = np.zeros((m, c))
    e = O.compress(m, 0, T // m, 0, ca, za, b0, cb, z, b0)
    _close(e[2, 2], 5.0, 1e-9, "stream-a dominant logit")
    zb = z.copy()
    zb[5, 1] = 80.0  # token 5 stream b -> entry 3 (previous block 4..5)
    e = O.compress(m, 0, T // m, 0, ca, z, b0, cb, zb, b0)
    _close(e[3, 1], 1005.0, 1e-9, "stream-b dominant logit")
    bb = np.zeros((m, c))
    bb[0, :] = 80.0  # first slot of the previous block
    e = O.compress(m, 1, T // m, 0, ca, z, b0, cb, z, bb)
    for i in range(1, T // m):
        _close(e[i - 1], np.full(c, 1000.0 + (i - 1) * m), 1e-9, f"bias b slot 0, entry {i}")
    ba = np.zeros((m, c))
    ba[1, :] = 80.0
    e = O.compress(m, 0, T // m, 0, ca, z, ba)
    for i in range(T // m):
        _close(e[i], np.full(c, i * m + 1.0), 1e-9, f"bias a slot 1, entry {i}")


def pin_compress_stream_window(O):
    """A stream whose row 0 is token tok_begin gives the same entry as the
    full stream (decode reads only the 2m newest tokens)."""
    rng = np.random.default_rng(12)
    T, c, m = 32, 8, 4
    s = [rng.standard_normal((T, c)) for _ in range(4)]
    ba, bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    g = 1 + 0.1 * rng.standard_normal(c)
    full = O.compress(m, 7, 8, 0, s[0], s[2], ba, s[1], s[3], bb, g, 4)
    tb = T - 2 * m
    part = O.compress(m, 7, 8, tb, s[0][tb:], s[2][tb:], ba, s[1][tb:], s[3][tb:], bb, g, 4)
    _close(part, full, 0.0, "windowed stream")


def pin_compress_norm_and_rope(O):
    """With a unit gain the normalised entry has RMS sqrt(ms/(ms+eps)); RoPE
    at position i*m keeps the norm, and rotating back by -i*m recovers the
    normalised (unrotated) entry, whose first D-R dims are untouched."""
    rng = np.random.default_rng(13)
    T, c, m, R = 16, 8, 2, 4
    s = [rng.standard_normal((T, c)) for _ in range(4)]
    b = np.zeros((m, c))
    raw = O.compress(m, 0, 8, 0, s[0], s[2], b, s[1], s[3], b)
    nrm = O.compress(m, 0, 8, 0, s[0], s[2], b, s[1], s[3], b, np.ones(c), R)
    ms = np.mean(raw ** 2, axis=1)
    _close(np.sqrt(np.mean(nrm ** 2, axis=1)), np.sqrt(ms / (ms + 1e-6)), 1e-12, "RMS after norm")
    unrot = np.stack([O.rope(nrm[i], -i * m, R, 10000.0) for i in range(8)])
    _close(unrot, raw / np.sqrt(ms + 1e-6)[:, None], 1e-12, "norm then RoPE at i*m")


# --------------------------------------------------------------------------
# grouped output projection
# --------------------------------------------------------------------------
def pin_out_proj_block_diagonal(O):
    """The grouped projection equals one dense product with the block-diagonal
    matrix of the group weights (torch.block_diag), applied to the heads in
    order."""
    rng = np.random.default_rng(17)
    M, H, D, g, r = 5, 6, 4, 3, 5
    o = rng.standard_normal((M, H, D))
    wa = rng.standard_normal((g, r, (H // g) * D))
    big = torch.block_diag(*[torch.from_numpy(wa[j]) for j in range(g)]).numpy()  # [g r, H D]
    _close(O.out_proj_mid(o, wa, g), o.reshape(M, -1) @ big.T, 1e-12, "grouped == block-diagonal")


def pin_out_proj_groups_are_separate(O):
    """A token whose only non-zero value sits in head h feeds only the
    intermediate of h's group; with W_b the identity the output is that
    intermediate as stored (bf16)."""
    rng = np.random.default_rng(18)
    M, H, D, g, r = 1, 8, 2, 4, 3
    wa = rng.standard_normal((g, r, (H // g) * D))
    for h in range(H):
        o = np.zeros((M, H, D))
        o[0, h, 1] = 1.0
        mid = O.out_proj_mid(o, wa, g)
        j = h // (H // g)
        mask = np.zeros(g * r, bool)
        mask[j * r:(j + 1) * r] = True
        assert np.all(mid[0, ~mask] == 0.0), f"head {h} leaks outside group {j}"
        _close(mid[0, mask], wa[j][:, (h % (H // g)) * D + 1], 0.0, f"head {h} column")
    o = rng.standard_normal((M, H, D))
    mid, y = O.out_proj(o, wa, np.eye(g * r), g)
    _close(y, O.widen(O.store_bf16(mid)), 0.0, "identity W_b")


# --------------------------------------------------------------------------
# block-scaled FP8 / FP4 storage
# --------------------------------------------------------------------------
def pin_e4m3_rounding_vs_torch(O):
    """E4M3 round-to-nearest-even (subnormals, ties, the top of the range)
    equals torch's float32 -> float8_e4m3fn conversion for every value torch
    keeps finite."""
    rng = np.random.default_rng(19)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-14, 9, 20000))).astype(np.float32)
    grid = np.concatenate([O.format_values("e4m3"), -O.format_values("e4m3")])
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)  # exact ties between neighbours
    x = np.concatenate([x, grid.astype(np.float32), mids, np.float32([448.0, 460.0, 464.0, -464.0])])
    x = x[np.abs(x) <= 464.0]
    ours = O.format_value(O.round_to_format(x, "e4m3"), "e4m3")
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    bad = np.flatnonzero(ours != ref)
    assert bad.size == 0, f"e4m3 differs from torch at {x[bad[:4]]}: {ours[bad[:4]]} vs {ref[bad[:4]]}"
    # the codes themselves, the sign of a value that rounds to zero included
    codes = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.round_to_format(x, "e4m3"), codes), "e4m3 codes differ from torch's"
    assert O.format_value(O.round_to_format(np.array([1e6, -1e6]), "e4m3"), "e4m3").tolist() == [448.0, -448.0]


def pin_e2m1_table(O):
    """E2M1: the eight magnitudes, nearest-even rounding at the midpoints
    (OCP MX specification's element format) and clamping at 6."""
    assert O.format_values("e2m1").tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.2, 0.3, 5.1, 7.0, -1.25, -5.0])
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 0.0, 0.5, 6.0, 6.0, -1.0, -4.0]
    assert O.format_value(O.round_to_format(x, "e2m1"), "e2m1").tolist() == want
    # codes: sign in bit 3, kept for a negative value that rounds to zero
    assert O.round_to_format(np.array([-0.1, 0.1, -6.0, -0.0]), "e2m1").tolist() == [8, 0, 15, 8]


def pin_mx_block_scale(O):
    """The block scale is the smallest power of two that keeps the block's
    largest magnitude in range: on-grid blocks survive a round trip exactly,
    a block max just above the largest element doubles the scale, and every
    value lands within half a step of itself."""
    for fmt, top in (("e4m3", 448.0), ("e2m1", 6.0)):
        grid = O.format_values(fmt)
        for s in (-20, -3, 0, 5):
            blk = np.resize(grid, 32) * 2.0 ** s
            blk[7] = top * 2.0 ** s
            codes, sc = O.mx_quantize(blk, fmt)
            assert int(sc[0]) == 127 + s, (fmt, s, sc)
            _close(O.mx_dequantize(codes, sc, fmt), blk, 0.0, f"{fmt} on-grid round trip")
            nxt = np.nextafter(top, np.inf) * 2.0 ** s
            _, sc2 = O.mx_quantize(np.concatenate([[nxt], np.zeros(31)]), fmt)
            assert int(sc2[0]) == 128 + s
        rng = np.random.default_rng(20)
        x = rng.standard_normal((50, 64)) * np.exp2(rng.integers(-6, 6, (50, 1)))
        codes, sc = O.mx_quantize(x, fmt)
        d = O.mx_dequantize(codes, sc, fmt)
        step = np.exp2(sc.astype(np.float64) - 127.0).repeat(32, axis=-1)
        # half of the largest gap of the format (1 for E4M3 near 448 is 16, scaled)
        half_gap = {"e4m3": 16.0, "e2m1": 1.0}[fmt]
        assert np.all(np.abs(d - x) <= half_gap * step + 1e-300)
    codes, sc = O.mx_quantize(np.zeros(32), "e4m3")
    assert int(sc[0]) == 0 and not codes.any()


def pin_kv_fp8_row_layout(O):
    """A mixed K=V row: FP8 codes of the first D - R dims, the last R dims as
    the stored bf16 bits, the scales, zero padding to 16 bytes; 592 bytes at
    the Flash shape; FP4 indexer keys pack the even element in the low
    nibble."""
    assert O.kv_fp8_row_bytes(512, 64) == 592
    rng = np.random.default_rng(21)
    rows = O.store_bf16(rng.standard_normal((4, 512)))
    q = O.quantize_kv_fp8(rows, 512, 64)
    assert q.shape == (4, 592) and not q[:, 590:].any()
    assert np.array_equal(q[:, 448:576].view(np.uint16), rows[:, 448:])
    d = O.dequantize_kv_fp8(q, 512, 64)
    assert np.array_equal(d[:, 448:], O.widen(rows[:, 448:]))
    codes, sc = O.mx_quantize(O.widen(rows[:, :448]), "e4m3")
    assert np.array_equal(q[:, :448], codes) and np.array_equal(q[:, 576:590], sc)
    keys = O.store_bf16(rng.standard_normal((3, 128)))
    packed, scales = O.quantize_idx_fp4(keys)
    c4, s4 = O.mx_quantize(O.widen(keys), "e2m1")
    assert np.array_equal(packed & 15, c4[:, 0::2]) and np.array_equal(packed >> 4, c4[:, 1::2])
    assert np.array_equal(scales, s4)
    _close(O.dequantize_idx_fp4(packed, scales), O.mx_dequantize(c4, s4, "e2m1"), 0.0, "fp4 unpack")


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
