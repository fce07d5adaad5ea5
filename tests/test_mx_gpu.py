"""Block-scaled cache storage on the GPU against the fp64 oracle: the FP8 /
FP4 quantisers bit for bit on identical bf16 inputs; the compressor writing
FP8 K=V entries and FP4 indexer keys during a token-by-token decode; the
indexer over FP4 keys and the attention over FP8 pools (checked like their
bf16 forms: top-k sets identical outside the tie zone, outputs within
max-abs-relative 1e-2); and the 1M-context decode mix in bench.py's launch
configuration with sampled sequences."""
import math

import numpy as np
import pytest
import torch

import long_context_hybrid_kv_b200 as L
from gen import host
from gen import workloads as W
from gpu_util import bf, check_ok, f32, f64, i32, ws_f32
from oracle import compare as C
from oracle import ds4a_oracle as O

pytestmark = pytest.mark.gpu
SEED = 5150
FLASH = W.FLASH_CSA
HCA = W.FLASH_HCA


def _u8(t):
    return t.cpu().numpy().astype(np.uint8)


def _spread_rows(name, n, D):
    """bf16 rows with blocks of widely different magnitudes, exact zeros,
    and values at the top of a block."""
    x = host.normal_f32(SEED, name, (n, D)).astype(np.float64)
    mag = np.exp2(host.normal_f32(SEED, name + ".m", (n, D // 32)).astype(np.float64) * 6.0)
    x = x * np.repeat(mag, 32, axis=1)
    x[0, :32] = 0.0
    x[1, :] = 0.0
    x[2, 5] = 448.0 * 4
    return O.store_bf16(x)


def test_quantize_kv_fp8_bit_exact():
    rows = _spread_rows("q8", 333, 512)
    out = torch.full((333, 592), 0xAB, dtype=torch.uint8, device="cuda")
    L.ds4a_quantize_kv_fp8(bf(rows), 64, out)
    check_ok()
    assert L.ds4a_kv_fp8_row_bytes(512, 64) == 592
    want = O.quantize_kv_fp8(rows, 512, 64)
    got = _u8(out)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:4].tolist()}"


def test_quantize_idx_fp4_bit_exact():
    keys = _spread_rows("q4", 517, 128)
    codes = torch.empty((517, 64), dtype=torch.uint8, device="cuda")
    scales = torch.empty((517, 4), dtype=torch.uint8, device="cuda")
    L.ds4a_quantize_idx_fp4(bf(keys), codes, scales)
    check_ok()
    wc, ws = O.quantize_idx_fp4(keys)
    assert np.array_equal(_u8(codes), wc) and np.array_equal(_u8(scales), ws)


def _fp8_pool(rows_bf16, B, n_c):
    """GPU FP8 pool made by the library's quantiser from bf16 rows (the
    oracle quantises the same bf16 rows itself)."""
    pool8 = torch.empty((B, n_c, 592), dtype=torch.uint8, device="cuda")
    L.ds4a_quantize_kv_fp8(bf(rows_bf16).reshape(B * n_c, 512), 64, pool8.view(B * n_c, 592))
    return pool8


def _fp4_keys(keys_bf16, B, n_c):
    codes = torch.empty((B, n_c, 64), dtype=torch.uint8, device="cuda")
    scales = torch.empty((B, n_c, 4), dtype=torch.uint8, device="cuda")
    L.ds4a_quantize_idx_fp4(bf(keys_bf16).reshape(B * n_c, 128), codes.view(B * n_c, 64), scales.view(B * n_c, 4))
    return codes, scales


@pytest.mark.parametrize("n_c,positions", [(1300, [2, 3, 2047, 2051, 2055, 3999, 9999]),
                                           (50000, [4 * 50000 - 1, 4 * 20000 - 1, 4 * 12289 - 1])])
def test_index_topk_fp4(n_c, positions):
    B, Tq = 2, len(positions)
    qi = host.normal_bf16(SEED, f"i4.{n_c}.qi", (B, Tq, 64, 128))
    wi = host.normal_bf16(SEED, f"i4.{n_c}.wi", (B, Tq, 64))
    ki = host.normal_bf16(SEED, f"i4.{n_c}.ki", (B, n_c, 128))
    codes, scales = _fp4_keys(ki, B, n_c)
    cfg = L.layer_cfg(FLASH)
    qpos = np.tile(np.asarray(positions, np.int32), (B, 1))
    idx = torch.empty((B, Tq, 512), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, Tq, 512), dtype=torch.float32, device="cuda")
    ws = ws_f32(L.ds4a_index_topk_workspace(cfg, B, Tq, n_c))
    L.ds4a_index_topk_fp4(cfg, i32(qpos), bf(qi), bf(wi), codes, scales, n_c, idx, ws, score_out=sc)
    check_ok()
    gidx, gsc = idx.cpu().numpy(), sc.cpu().numpy()
    for b in range(B):
        kdq = O.dequantize_idx_fp4(*O.quantize_idx_fp4(ki[b]))
        for t in range(Tq):
            ridx, rs = O.index_topk(qi[b, t], wi[b, t], kdq, int(qpos[b, t]), 4, 512, n_c)
            msg = C.check_topk_row(gidx[b, t], rs, 512)
            assert msg is None, f"row {(b, t)}: {msg}"
            sel = gidx[b, t][gidx[b, t] >= 0]
            if sel.size:
                den = np.abs(rs[sel]) + max(1e-3 * np.abs(rs).max(), 1e-12)
                assert np.max(np.abs(gsc[b, t, :sel.size] - rs[sel]) / den) < 1e-4


def _attend_fp8_case(name, cfg_py, B, positions, n_c, sparse, win_cap):
    Tq = len(positions)
    H, D = cfg_py.n_heads, cfg_py.head_dim
    q = host.normal_bf16(SEED, f"{name}.q", (B, Tq, H, D))
    g = host.normal_f32(SEED, f"{name}.g", (D,), 0.1, 1.0)
    pool = host.normal_bf16(SEED, f"{name}.pool", (B, n_c, D))
    win = host.normal_bf16(SEED, f"{name}.win", (B, win_cap, D))
    sink = host.normal_f32(SEED, f"{name}.sink", (H,))
    qpos = np.tile(np.asarray(positions, np.int32), (B, 1))
    cfg = L.layer_cfg(cfg_py)
    pool8 = _fp8_pool(pool, B, n_c)
    out = torch.empty((B, Tq, H, D), dtype=torch.bfloat16, device="cuda")
    ws = ws_f32(L.ds4a_attend_workspace(cfg, B, Tq, n_c, sparse))
    dq = np.stack([O.dequantize_kv_fp8(O.quantize_kv_fp8(pool[b], 512, 64), 512, 64) for b in range(B)])
    if sparse:
        n_vis = np.minimum((qpos + 1) // cfg_py.ratio, n_c)
        idx = host.random_subset_idx(SEED, f"{name}.idx", n_vis.ravel(), cfg_py.topk).reshape(B, Tq, -1)
        L.ds4a_sparse_attend_fp8(cfg, i32(qpos), bf(q), f32(g), pool8, n_c, i32(idx), bf(win), win_cap, f32(sink),
                                 out, ws)
        ref = O.csa_attend_batch(q, g, dq, idx, win, win_cap, sink, qpos, cfg_py)
    else:
        L.ds4a_hca_attend_fp8(cfg, i32(qpos), bf(q), f32(g), pool8, n_c, bf(win), win_cap, f32(sink), out, ws)
        ref = O.hca_attend_batch(q, g, dq, n_c, win, win_cap, sink, qpos, cfg_py)
    check_ok()
    got = f64(out)
    for b in range(B):
        for t in range(Tq):
            err = C.max_abs_rel(got[b, t], ref[b, t])
            assert err < C.OUT_TOL, f"{name} query {(b, t)} pos {positions[t]}: err {err}"


def test_sparse_attend_fp8_decode():
    _attend_fp8_case("a8d", FLASH, 2, [0, 5, 127, 300, 3999], 1000, True, 128)


def test_sparse_attend_fp8_prefill_sized():
    pos = sorted(set([0, 1, 2, 3, 5, 126, 127, 128, 131] + list(range(200, 3999, 23))))
    _attend_fp8_case("a8p", FLASH, 1, pos, 1000, True, 4096)


def test_hca_attend_fp8():
    _attend_fp8_case("h8", HCA, 2, [126, 127, 5119, 140000], 1100, False, 128)


def test_compress_append_mx():
    # a decode of 1024 tokens writing FP8 K=V entries (CSA, m=4) and FP4
    # indexer keys: the rounding of the entry to bf16 may differ by an ulp
    # between fp32 and fp64, so a code may move to its neighbour where that
    # decides it; every code equal or adjacent, almost all equal
    T, B = 1024, 2
    cfg = L.LayerCfg(64, 512, 64, 128, 64, 128, 512, 4, 512 ** -0.5, 10000.0, 1e-6)
    res = {}
    for name, c, fmt, norm in (("kv", 512, L.DS4A_MX_KV_FP8, True), ("ix", 128, L.DS4A_MX_IDX_FP4, False)):
        st = {s: host.normal_bf16(SEED, f"cm.{name}.{s}", (B, T, c)) for s in ("ca", "cb", "za", "zb")}
        ba = host.normal_f32(SEED, f"cm.{name}.ba", (4, c), 0.5)
        bb = host.normal_f32(SEED, f"cm.{name}.bb", (4, c), 0.5)
        g = host.normal_f32(SEED, f"cm.{name}.g", (c,), 0.1, 1.0) if norm else None
        n = T // 4
        state = torch.zeros(L.ds4a_compress_state_bytes(cfg, B, c, True) // 2, dtype=torch.bfloat16, device="cuda")
        if fmt == L.DS4A_MX_KV_FP8:
            pool, scales = torch.zeros((B, n, 592), dtype=torch.uint8, device="cuda"), None
        else:
            pool = torch.zeros((B, n, c // 2), dtype=torch.uint8, device="cuda")
            scales = torch.zeros((B, n, c // 32), dtype=torch.uint8, device="cuda")
        dev = {k: bf(v) for k, v in st.items()}
        for t in range(T):
            pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
            rows = {k: v[:, t].contiguous() for k, v in dev.items()}
            L.ds4a_compress_append_mx(cfg, pos, rows["ca"], rows["za"], f32(ba), state, fmt, pool, scales=scales,
                                      cb=rows["cb"], zb=rows["zb"], bias_b=f32(bb), norm_g=f32(g) if norm else None)
        check_ok()
        for b in range(B):
            ent = O.compress(4, 0, n, 0, st["ca"][b], st["za"][b], ba, st["cb"][b], st["zb"][b], bb, g,
                             64 if norm else 0)
            if fmt == L.DS4A_MX_KV_FP8:
                want = O.quantize_kv_fp8(O.store_bf16(ent), 512, 64)
                got = _u8(pool[b])
                gc, wc = got[:, :448], want[:, :448]
                vg, vw = O.format_value(gc, "e4m3"), O.format_value(wc, "e4m3")
                gs, wsc = got[:, 576:590], want[:, 576:590]
                # RoPE dims: bf16 as stored, within the bf16 tolerance
                rg = got[:, 448:576].copy().view(np.uint16)
                rw = want[:, 448:576].copy().view(np.uint16)
                assert C.max_abs_rel(O.widen(rg), O.widen(rw)) < C.OUT_TOL
                assert not got[:, 590:].any()
                grid = O.format_values("e4m3")
            else:
                wc4, wsc = O.quantize_idx_fp4(O.store_bf16(ent))
                gc = np.stack([_u8(pool[b]) & 15, _u8(pool[b]) >> 4], -1).reshape(n, c)
                wc = np.stack([wc4 & 15, wc4 >> 4], -1).reshape(n, c)
                vg, vw = O.format_value(gc, "e2m1"), O.format_value(wc, "e2m1")
                gs = _u8(scales[b])
                grid = O.format_values("e2m1")
            same_scale = gs == wsc
            assert same_scale.mean() > 0.99, f"{name} seq {b}: scales {same_scale.mean()}"
            blk = np.repeat(same_scale, 32, axis=1)
            eq = (gc == wc)[blk]
            assert eq.mean() > 0.98, f"{name} seq {b}: {eq.mean()} of codes equal"
            # differing codes are neighbours on the format's grid
            rank_g = np.searchsorted(grid, np.abs(vg[blk])) * np.sign(vg[blk])
            rank_w = np.searchsorted(grid, np.abs(vw[blk])) * np.sign(vw[blk])
            assert np.all(np.abs(rank_g - rank_w) <= 1), f"{name} seq {b}: a code moved by more than one step"
            res[(name, b)] = eq.mean()


def test_workload_mix_decode_mx():
    import bench
    st = bench.State(11)
    st.step()
    check_ok()
    w = st.w
    c, h = w.csa, w.hca
    for ly in st.layers:
        if ly.kind == "csa":
            _check_csa_mx(st, ly, w, [0, 5])
        else:
            _check_hca_mx(st, ly, w, [0, 1, 7])


def _check_csa_mx(st, ly, w, bsel):
    c = w.csa
    n_c, pos, m = w.n_csa, w.pos, c.ratio
    e, tb = n_c - 1, pos - 2 * m + 1
    H = {n: W.host_tensor(w, f"csa.{n}") for n in ("kv_ca", "kv_cb", "kv_za", "kv_zb", "ix_ca", "ix_cb", "ix_za",
                                                  "ix_zb", "kv_ba", "kv_bb", "ix_ba", "ix_bb", "kv_g", "q", "qi",
                                                  "wi", "q_norm_g", "sink", "win")}
    gidx = ly.idx.cpu().numpy()
    gout = f64(ly.out)
    for b in bsel:
        ent = O.compress(m, e, e + 1, tb, H["kv_ca"][b], H["kv_za"][b], H["kv_ba"], H["kv_cb"][b], H["kv_zb"][b],
                         H["kv_bb"], H["kv_g"], c.rope_dim)[0]
        kent = O.compress(m, e, e + 1, tb, H["ix_ca"][b], H["ix_za"][b], H["ix_ba"], H["ix_cb"][b], H["ix_zb"][b],
                          H["ix_bb"])[0]
        ki = W.host_rows(w, "csa.ki", b * n_c + np.arange(n_c))
        ki[e] = O.store_bf16(kent)
        kdq = O.dequantize_idx_fp4(*O.quantize_idx_fp4(ki))
        idx, scores = O.index_topk(H["qi"][b, 0], H["wi"][b, 0], kdq, pos, m, c.topk, n_c)
        msg = C.check_topk_row(gidx[b, 0], scores, c.topk)
        assert msg is None, f"seq {b}: {msg}"
        sel = idx[idx >= 0]
        rows = W.host_rows(w, "csa.pool", b * n_c + sel)
        rows[sel == e] = O.store_bf16(ent)
        pool = np.zeros((n_c, c.head_dim))
        pool[sel] = O.dequantize_kv_fp8(O.quantize_kv_fp8(rows, 512, 64), 512, 64)
        out = O.csa_attend(H["q"][b, 0], H["q_norm_g"], pool, idx, H["win"][b], c.window, H["sink"], pos, c)
        if np.array_equal(gidx[b, 0], idx):
            got = gout[b, 0]
        else:  # tie-zone difference: the oracle's set, attended on the GPU too
            idx2 = ly.idx.clone()
            idx2[b, 0] = torch.from_numpy(idx.astype(np.int32)).to(idx2.device)
            out2 = torch.empty_like(ly.out)
            L.ds4a_sparse_attend_fp8(ly.cfg, ly.q_pos, ly.t["q"], ly.t["q_norm_g"], ly.kv8, n_c, idx2, ly.t["win"],
                                     c.window, ly.t["sink"], out2, ly.ws_att)
            check_ok()
            got = f64(out2)[b, 0]
        err = C.max_abs_rel(got, out)
        assert err < C.OUT_TOL, f"seq {b}: attend err {err}"


def _check_hca_mx(st, ly, w, bsel):
    h = w.hca
    n_c, pos, m = w.n_hca, w.pos, h.ratio
    e, tb = n_c - 1, pos - m + 1
    Hh = {n: W.host_tensor(w, f"hca.{n}") for n in ("kv_c", "kv_z", "kv_b", "kv_g", "q", "q_norm_g", "sink", "win")}
    gout = f64(ly.out)
    for b in bsel:
        ent = O.compress(m, e, e + 1, tb, Hh["kv_c"][b], Hh["kv_z"][b], Hh["kv_b"], norm_g=Hh["kv_g"],
                         rope_dim=h.rope_dim)[0]
        rows = W.host_rows(w, "hca.pool", b * n_c + np.arange(n_c))
        rows[e] = O.store_bf16(ent)
        pool = O.dequantize_kv_fp8(O.quantize_kv_fp8(rows, 512, 64), 512, 64)
        out = O.hca_attend(Hh["q"][b, 0], Hh["q_norm_g"], pool, n_c, Hh["win"][b], h.window, Hh["sink"], pos, h)
        err = C.max_abs_rel(gout[b, 0], out)
        assert err < C.OUT_TOL, f"seq {b}: err {err}"
