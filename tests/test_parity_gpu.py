"""GPU parity: each ABI call against the fp64 oracle on the same seeded
inputs (element by element at sizes spanning several tiles and a ragged
tail), the edge cases, the device error word, and the full-size workloads in
the launch configuration bench.py times (sampled where the oracle would take
too long).  Tolerances: max-abs-relative 1e-2 for bf16 outputs; top-k sets
identical outside the 1e-4 relative tie zone (oracle/compare.py)."""
import math

import numpy as np
import pytest
import torch

import long_context_hybrid_kv_b200 as L
from gen import device as gd
from gen import host
from gen import workloads as W
from gpu_util import bf, bits, check_ok, f32, f64, i32, kernels_used, ws_f32
from oracle import compare as C
from oracle import ds4a_oracle as O

pytestmark = pytest.mark.gpu

FLASH = W.FLASH_CSA
HCA = W.FLASH_HCA
SEED = 4242


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need cuda:0"
    torch.cuda.set_device(0)
    L.lib()
    gd.lib()
    yield
    torch.cuda.synchronize()


def nb(name, shape, scale=None, offset=None):
    return host.normal_bf16(SEED, name, shape, scale, offset)


def nf(name, shape, scale=None, offset=None):
    return host.normal_f32(SEED, name, shape, scale, offset)


# ---------------------------------------------------------------------------
# generator
# ---------------------------------------------------------------------------
def test_device_generator_matches_host():
    for name, shape, sc, off, dt in [("a", (1000,), None, None, "bf16"), ("b", (77, 33), 0.25, None, "bf16"),
                                     ("g", (512,), 0.1, 1.0, "f32"), ("s", (64,), None, None, "f32"),
                                     ("w", (3, 5), 1 / math.sqrt(16), None, "f32")]:
        t = torch.empty(shape, dtype=torch.bfloat16 if dt == "bf16" else torch.float32, device="cuda")
        gd.fill(t, SEED, name, sc, off)
        if dt == "bf16":
            assert np.array_equal(bits(t), host.normal_bf16(SEED, name, shape, sc, off)), name
        else:
            assert np.array_equal(t.cpu().numpy(), host.normal_f32(SEED, name, shape, sc, off)), name
    big = torch.empty((3, 1 << 20), dtype=torch.bfloat16, device="cuda")
    gd.fill(big, SEED, "big")
    rows = np.array([0, 1, 2])
    idx = np.array([0, 12345, (1 << 20) - 1])
    flat = (rows[:, None] * (1 << 20) + idx[None, :]).ravel()
    assert np.array_equal(bits(big).ravel()[flat], host.normal_bf16_at(SEED, "big", flat))


# ---------------------------------------------------------------------------
# compressor
# ---------------------------------------------------------------------------
COMPRESS_CASES = {
    # name: (c, m, overlap, norm, rope, B, tok_begin, T_tok, entry range)
    "csa_kv_prefill": (512, 4, True, True, 64, 2, 0, 520, (0, 130)),
    "csa_kv_decode_pos1m": (512, 4, True, True, 64, 2, 1048568, 8, (262143, 262144)),
    "csa_ix_prefill": (128, 4, True, False, 0, 2, 0, 516, (0, 129)),
    "hca_kv": (512, 128, False, True, 64, 2, 0, 640, (0, 5)),
    "hca_kv_decode": (512, 128, False, True, 64, 3, 130944, 128, (1023, 1024)),
    # many long entries: one block per entry, not the channel-split cluster
    "hca_kv_many": (512, 128, False, True, 64, 2, 0, 5120, (0, 40)),
    # long entries of another width: the term-split cluster kernel
    "hca_256_split": (256, 128, False, True, 32, 2, 0, 640, (0, 5)),
    "toy_kv": (8, 2, True, True, 2, 1, 0, 64, (0, 32)),
    "toy_ix": (4, 2, True, False, 0, 1, 0, 64, (0, 32)),
    "mid_entries": (256, 4, True, True, 32, 1, 40, 60, (11, 25)),
}


@pytest.mark.parametrize("case", sorted(COMPRESS_CASES))
def test_compress(case):
    c, m, overlap, norm, R, B, tb, T, (e0, e1) = COMPRESS_CASES[case]
    cfg = L.LayerCfg(64, 512, R, 128, 64, 128, 512, m, 512 ** -0.5, 10000.0, 1e-6)
    ca, za = nb(f"{case}.ca", (B, T, c)), nb(f"{case}.za", (B, T, c))
    ba = nf(f"{case}.ba", (m, c), 1 / math.sqrt(m))
    cb = zb = bb = None
    if overlap:
        cb, zb = nb(f"{case}.cb", (B, T, c)), nb(f"{case}.zb", (B, T, c))
        bb = nf(f"{case}.bb", (m, c), 1 / math.sqrt(m))
    g = nf(f"{case}.g", (c,), 0.1, 1.0) if norm else None
    pool = torch.full((B, e1 + 3, c), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.ds4a_compress(cfg, bf(ca), bf(za), f32(ba), pool, cb=None if cb is None else bf(cb),
                    zb=None if zb is None else bf(zb), bias_b=None if bb is None else f32(bb),
                    norm_g=None if g is None else f32(g), tok_begin=tb, entry_begin=e0, entry_end=e1)
    check_ok()
    got = f64(pool)
    ref = O.compress_batch(m, e0, e1, tb, ca, za, ba, cb, zb, bb, g, R)
    err = C.max_abs_rel(got[:, e0:e1], ref)
    assert err < C.OUT_TOL, err
    # untouched rows stay untouched
    assert np.isnan(got[:, :e0]).all() and np.isnan(got[:, e1:]).all()


# ---------------------------------------------------------------------------
# indexer + top-k
# ---------------------------------------------------------------------------
def _index_case(B, positions, n_c, cfg_py, name, ki=None):
    Tq = len(positions)
    qi = nb(f"{name}.qi", (B, Tq, cfg_py.idx_heads, cfg_py.idx_dim))
    wi = nb(f"{name}.wi", (B, Tq, cfg_py.idx_heads))
    if ki is None:
        ki = nb(f"{name}.ki", (B, max(n_c, 1), cfg_py.idx_dim))
    qpos = np.tile(np.asarray(positions, np.int32), (B, 1))
    cfg = L.layer_cfg(cfg_py)
    idx = torch.empty((B, Tq, cfg_py.topk), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, Tq, cfg_py.topk), dtype=torch.float32, device="cuda")
    ws = ws_f32(L.ds4a_index_topk_workspace(cfg, B, Tq, n_c))
    L.ds4a_index_topk(cfg, i32(qpos), bf(qi), bf(wi), bf(ki), n_c, idx, ws, score_out=sc)
    check_ok()
    return qi, wi, ki, qpos, idx.cpu().numpy(), sc.cpu().numpy()


def _check_index(qi, wi, ki, qpos, gidx, gsc, cfg_py, n_c, rows=None):
    B, Tq = qpos.shape
    todo = rows if rows is not None else [(b, t) for b in range(B) for t in range(Tq)]
    for b, t in todo:
        ridx, rs = O.index_topk(qi[b, t], wi[b, t], ki[b], int(qpos[b, t]), cfg_py.ratio, cfg_py.topk, n_c)
        msg = C.check_topk_row(gidx[b, t], rs, cfg_py.topk)
        assert msg is None, f"row {(b, t)}: {msg}"
        sel = gidx[b, t][gidx[b, t] >= 0]
        if sel.size:
            den = np.abs(rs[sel]) + max(1e-3 * np.abs(rs).max(), 1e-12)
            err = np.max(np.abs(gsc[b, t, : sel.size] - rs[sel]) / den)
            assert err < 1e-4, f"row {(b, t)} score error {err}"
        assert np.all(np.isneginf(gsc[b, t, sel.size:]))


def test_index_topk_flash_ragged():
    # N_c = 1300 (not a tile multiple); visible counts 0, 1, 511, 512, 513, 1000, 1300
    pos = [2, 3, 2047, 2051, 2055, 3999, 9999]
    qi, wi, ki, qpos, gidx, gsc = _index_case(2, pos, 1300, FLASH, "ragged")
    _check_index(qi, wi, ki, qpos, gidx, gsc, FLASH, 1300)
    assert np.all(gidx[:, 0] == -1)


def test_index_topk_no_entries():
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, [5, 100], 0, FLASH, "none")
    assert np.all(gidx == -1)


def test_index_topk_ties_take_lower_index():
    # every key equal -> every score equal -> the k lowest indices
    n_c = 2000
    row = nb("tie.row", (1, 1, FLASH.idx_dim))
    ki = np.repeat(row, n_c, axis=1)
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, [4 * n_c - 1], n_c, FLASH, "tie", ki=ki)
    assert np.array_equal(gidx[0, 0], np.arange(FLASH.topk))


def test_index_topk_large_rows_cluster_path():
    # rows above the shared-memory size take the 8-block cluster selector:
    # random keys (checked against the oracle) and all-equal keys (ties)
    n_c = 50000
    pos = [4 * n_c - 1, 4 * 20000 - 1, 4 * 12289 - 1]
    qi, wi, ki, qpos, gidx, gsc = _index_case(2, pos, n_c, FLASH, "clus")
    _check_index(qi, wi, ki, qpos, gidx, gsc, FLASH, n_c)
    row = nb("clus.tie", (1, 1, FLASH.idx_dim))
    ki = np.repeat(row, n_c, axis=1)
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, [4 * n_c - 1], n_c, FLASH, "clustie", ki=ki)
    assert np.array_equal(gidx[0, 0], np.arange(FLASH.topk))


def test_index_topk_cluster_crowded_scores():
    # keys within ~2 % of one row: the scores are distinct but crowd into one
    # or two histogram bins of the cluster selector, whose floor then leaves
    # more candidates than a block keeps, so every block selects its own k
    # best before block 0 merges (the selector's second path)
    n_c = 40000
    row = nf("crowd.row", (1, 1, FLASH.idx_dim))
    noise = nf("crowd.noise", (1, n_c, FLASH.idx_dim))
    ki = host.f32_to_bf16_bits((row * (1.0 + 0.02 * noise)).astype(np.float32)).reshape(1, n_c, FLASH.idx_dim)
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, [4 * n_c - 1, 4 * 30000 - 1], n_c, FLASH, "crowd", ki=ki)
    _check_index(qi, wi, ki, qpos, gidx, gsc, FLASH, n_c)


@pytest.mark.parametrize("k", [1500, 2048, 3000])
def test_index_topk_cluster_large_k(k):
    # k above the block's 1024 threads (no per-block floor in the second
    # path), at the local-candidate kernel's limit (2048), and above it (the
    # multi-pass cluster kernel)
    import dataclasses

    cfg_py = dataclasses.replace(FLASH, topk=k)
    n_c = 30000
    pos = [4 * n_c - 1, 4 * (k + 700) - 1]
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, pos, n_c, cfg_py, f"bigk{k}")
    _check_index(qi, wi, ki, qpos, gidx, gsc, cfg_py, n_c)


def test_index_topk_beyond_cluster_rows():
    # longer than the cluster selector's 262144: the global-memory selector
    n_c = 262144 + 1000
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, [4 * n_c - 1], n_c, FLASH, "huge")
    _check_index(qi, wi, ki, qpos, gidx, gsc, FLASH, n_c)


def test_index_topk_prefill_rows():
    # causal prefill over 4096 tokens (1024 entries), sampled rows
    T = 4096
    pos = list(range(T))
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, pos, T // 4, FLASH, "pref")
    rng = np.random.default_rng(1)
    rows = sorted(set([0, 1, 2, 3, 4, 7, 2046, 2047, 2048, 2051, 2052, 4095] +
                      list(rng.integers(0, T, 40))))
    _check_index(qi, wi, ki, qpos, gidx, gsc, FLASH, T // 4, [(0, t) for t in rows])


def test_index_topk_toy():
    c = W.TOY_CSA
    pos = list(range(64))
    qi, wi, ki, qpos, gidx, gsc = _index_case(1, pos, 32, c, "toyidx")
    _check_index(qi, wi, ki, qpos, gidx, gsc, c, 32)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def _attend_case(name, cfg_py, B, positions, n_c, sparse, win_cap, use_ws=True, idx=None, ws_bytes=None,
                 pool_pad=0):
    """One attend call against the oracle.  pool_pad > 0 lays the pool's
    sequences out pool_pad elements further apart than [N_c, D] rows."""
    Tq = len(positions)
    H, D = cfg_py.n_heads, cfg_py.head_dim
    q = nb(f"{name}.q", (B, Tq, H, D))
    g = nf(f"{name}.g", (D,), 0.1, 1.0)
    pool = nb(f"{name}.pool", (B, max(n_c, 1), D))
    win = nb(f"{name}.win", (B, win_cap, D))
    sink = nf(f"{name}.sink", (H,))
    qpos = np.tile(np.asarray(positions, np.int32), (B, 1))
    cfg = L.layer_cfg(cfg_py)
    out = torch.empty((B, Tq, H, D), dtype=torch.bfloat16, device="cuda")
    if ws_bytes is not None:
        ws = ws_f32(ws_bytes)
    else:
        ws = ws_f32(L.ds4a_attend_workspace(cfg, B, Tq, n_c, sparse)) if use_ws else None
    pool_d = bf(pool)
    if pool_pad:
        rows = pool.shape[1] * D
        flat = torch.zeros(B * (rows + pool_pad), dtype=torch.bfloat16, device="cuda")
        pool_d = flat.as_strided(tuple(pool.shape), (rows + pool_pad, D, 1))
        pool_d.copy_(bf(pool))
    if sparse:
        if idx is None:
            n_vis = np.minimum((qpos + 1) // cfg_py.ratio, n_c)
            idx = host.random_subset_idx(SEED, f"{name}.idx", n_vis.ravel(), cfg_py.topk).reshape(B, Tq, -1)
        L.ds4a_sparse_attend(cfg, i32(qpos), bf(q), f32(g), pool_d, n_c, i32(idx), bf(win), win_cap, f32(sink),
                             out, ws)
        ref = O.csa_attend_batch(q, g, pool, idx, win, win_cap, sink, qpos, cfg_py)
    else:
        L.ds4a_hca_attend(cfg, i32(qpos), bf(q), f32(g), pool_d, n_c, bf(win), win_cap, f32(sink), out, ws)
        ref = O.hca_attend_batch(q, g, pool, n_c, win, win_cap, sink, qpos, cfg_py)
    check_ok()
    got = f64(out)
    for b in range(B):
        for t in range(Tq):
            err = C.max_abs_rel(got[b, t], ref[b, t])
            assert err < C.OUT_TOL, f"query {(b, t)} pos {positions[t]}: err {err}"
    return got, ref


@pytest.mark.parametrize("split", [True, False], ids=["split", "nosplit"])
def test_sparse_attend_flash(split):
    # positions: inside the first window, exactly W, few entries, many entries
    _attend_case("sp", FLASH, 2, [0, 5, 127, 300, 3999], 1000, True, 128,
                 ws_bytes=None if split else 2 * 5 * 65536)


@pytest.mark.parametrize("split", [True, False], ids=["split", "nosplit"])
def test_hca_attend_flash(split):
    _attend_case("hc", HCA, 2, [126, 127, 5119, 6000], 40, False, 128,
                 ws_bytes=None if split else 2 * 4 * 65536)


def test_attend_tensor_core_without_splits():
    # a workspace too small for split partials: the tensor-core path with
    # one split per query (final output written by the attention kernel)
    pos = [0, 5, 127, 300, 3999]
    names = kernels_used(lambda: _attend_case("tc1", FLASH, 2, pos, 1000, True, 128, ws_bytes=2 * 5 * 65536))
    assert "attend_tc" in names and "attend_combine" not in names, names
    names = kernels_used(lambda: _attend_case("tc1h", HCA, 2, [126, 5119], 40, False, 128, ws_bytes=2 * 2 * 65536))
    assert "attend_tc" in names and "attend_combine" not in names, names


def test_attend_paths_used():
    # Flash shapes take the tensor-core kernel whatever the workspace (with
    # none, one split per query and no combine); other head shapes run on
    # CUDA cores
    names = kernels_used(lambda: _attend_case("path", FLASH, 1, [3999], 1000, True, 128))
    assert names == ["attend_tc", "attend_combine"], names  # decode-sized: q^ inside the kernel
    names = kernels_used(lambda: _attend_case("path0", FLASH, 1, [3999], 1000, True, 128, use_ws=False))
    assert names == ["attend_tc"], names
    names = kernels_used(lambda: _attend_case("pathtoy", W.TOY_CSA, 1, [63], 32, True, 4, use_ws=False))
    assert names == ["attend_generic"], names


def test_attend_many_splits_and_empty_splits():
    # 1093 visible HCA entries + 128 window keys = 10 tiles, split ten ways;
    # beside it a query whose keys fill two tiles leaves eight splits empty
    names = kernels_used(lambda: _attend_case("many", HCA, 1, [140000], 1100, False, 128))
    assert names == ["attend_tc", "attend_combine"], names
    _attend_case("two", HCA, 1, [130, 140000], 1100, False, 128)
    # a pool whose sequences are not a whole number of rows apart (gathered
    # rows; the dense HCA tile loads need whole rows)
    _attend_case("pad", FLASH, 2, [0, 5, 127, 300, 3999], 1000, True, 128, pool_pad=8)
    _attend_case("padh", HCA, 2, [5119, 6000], 40, False, 128, pool_pad=8)


def test_attend_prefill_sized_launches():
    # more than 148 queries: the prefill form of the kernel (work items
    # round-robin over the blocks, q-hat loaded by TMA and prepared in place
    # by the producers, the next item built during the last tile); positions
    # cover empty, partial
    # and full windows, selected counts that are not multiples of four and
    # ragged last tiles
    pos = sorted(set([0, 1, 2, 3, 5, 6, 7, 126, 127, 128, 129, 130, 131] + list(range(200, 3999, 23))))
    assert len(pos) > 148
    _attend_case("pf", FLASH, 1, pos, 1000, True, 4096)
    # HCA over consecutive pool entries (whole tiles by TMA tile loads) in
    # the prefill form
    hpos = list(range(16383, 16383 + 160 * 131, 131))
    _attend_case("pfh", HCA, 1, hpos, 300, False, 512)


def test_swa_only_layer():
    # the sliding-window-only layer is HCA attention with no pool entries
    _attend_case("swa", HCA, 1, [0, 3, 200], 0, False, 128)


def test_no_window():
    import dataclasses
    cfg = dataclasses.replace(FLASH, window=0)
    got, ref = _attend_case("nowin", cfg, 1, [40, 4000], 700, True, 1)
    # a query with neither entries nor window gives 0 (all mass on the sink)
    cfg0 = dataclasses.replace(FLASH, window=0)
    q = torch.ones((1, 1, 64, 512), dtype=torch.bfloat16, device="cuda")
    out = torch.full((1, 1, 64, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    z = torch.zeros(512, dtype=torch.float32, device="cuda")
    idx = torch.full((1, 1, 512), -1, dtype=torch.int32, device="cuda")
    ws = ws_f32(L.ds4a_attend_workspace(L.layer_cfg(cfg0), 1, 1, 0, True))
    L.ds4a_sparse_attend(L.layer_cfg(cfg0), i32([[2]]), q, z + 1, None, 0, idx, None, 0, z[:64], out, ws)
    check_ok()
    assert float(out.float().abs().max()) == 0.0


def test_sparse_attend_toy_prefill_and_decode():
    c = W.TOY_CSA
    _attend_case("toyp", c, 1, list(range(64)), 32, True, 64)
    _attend_case("toyd", c, 1, [63], 32, True, 4)


def test_attend_full_selection_equals_hca():
    # CSA with every visible entry selected equals HCA over the same pool
    B, n_c, pos = 1, 300, [1199, 700]
    n_vis = np.minimum((np.array(pos) + 1) // 4, n_c)
    idx = np.full((B, len(pos), 512), -1, np.int32)
    for t, n in enumerate(n_vis):
        idx[0, t, :n] = np.arange(n)
    g1, _ = _attend_case("eq", FLASH, B, pos, n_c, True, 128, idx=idx)
    g2, _ = _attend_case("eq", FLASH, B, pos, n_c, False, 128)
    assert C.max_abs_rel(g1, g2) < 1e-2


# ---------------------------------------------------------------------------
# device error word
# ---------------------------------------------------------------------------
def test_bad_index_sets_error_word():
    cfg = L.layer_cfg(FLASH)
    q = gd.tensor(W.WORKLOADS[2], "csa.q")
    pool = gd.tensor(W.WORKLOADS[2], "csa.pool")
    win = gd.tensor(W.WORKLOADS[2], "csa.win")
    g = torch.ones(512, device="cuda")
    sink = torch.zeros(64, device="cuda")
    idx = torch.arange(512, dtype=torch.int32, device="cuda").reshape(1, 1, 512)
    idx[0, 0, 100] = 5000  # beyond N_c = 2048
    out = torch.empty((1, 1, 64, 512), dtype=torch.bfloat16, device="cuda")
    ws = ws_f32(L.ds4a_attend_workspace(cfg, 1, 1, 2048, True))
    L.ds4a_sparse_attend(cfg, i32([[8191]]), q, g, pool, 2048, idx, win, 128, sink, out, ws)
    rc, b = L.ds4a_check()
    assert rc == L.DS4A_EDEVICE and (b & 1)
    assert torch.isfinite(out.float()).all()
    assert L.ds4a_check() == (0, 0)  # cleared
    L.ds4a_sparse_attend(cfg, i32([[-4]]), q, g, pool, 2048, idx, win, 128, sink, out, ws)
    rc, b = L.ds4a_check()
    assert rc == L.DS4A_EDEVICE and (b & 2)


def test_bounded_wait_runs_out_and_reports():
    # a kernel waits on an mbarrier nothing arrives at, with a ~1 ms bound:
    # it records the timeout, exits, and the host reads DS4A_ETIMEOUT; the
    # context stays usable for the next call
    assert L.ds4a_check() == (0, 0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.ds4a_selftest_wait_timeout(2_000_000, status)
    rc, b = L.ds4a_check()
    assert rc == L.DS4A_ETIMEOUT and (b & 4), (rc, b)
    assert int(status.item()) == 2
    assert L.ds4a_check() == (0, 0)  # cleared
    _attend_case("after_timeout", FLASH, 1, [3999], 1000, True, 128)


# ---------------------------------------------------------------------------
# full-size workloads, in bench.py's launch configuration
# ---------------------------------------------------------------------------
def _state(wid):
    import bench
    st = bench.State(wid)
    st.step()
    check_ok()
    return st


def _decode_csa_ref(w, ly, bsel):
    """Oracle chain of one CSA decode layer for the sequences bsel."""
    c = w.csa
    n_c, pos, m = w.n_csa, w.pos, c.ratio
    e = n_c - 1
    tb = pos - 2 * m + 1
    pre = ly.prefix + "csa."
    H = {n: W.host_tensor(w, pre + n) for n in ("kv_ca", "kv_cb", "kv_za", "kv_zb", "ix_ca", "ix_cb",
                                               "ix_za", "ix_zb", "kv_ba", "kv_bb", "ix_ba", "ix_bb",
                                               "kv_g", "q", "qi", "wi", "q_norm_g", "sink", "win")}
    res = {}
    for b in bsel:
        ent = O.compress(m, e, e + 1, tb, H["kv_ca"][b], H["kv_za"][b], H["kv_ba"], H["kv_cb"][b],
                         H["kv_zb"][b], H["kv_bb"], H["kv_g"], c.rope_dim)[0]
        kent = O.compress(m, e, e + 1, tb, H["ix_ca"][b], H["ix_za"][b], H["ix_ba"], H["ix_cb"][b],
                          H["ix_zb"][b], H["ix_bb"])[0]
        ki = W.host_rows(w, pre + "ki", b * n_c + np.arange(n_c))
        ki[e] = O.store_bf16(kent)
        idx, scores = O.index_topk(H["qi"][b, 0], H["wi"][b, 0], ki, pos, m, c.topk, n_c)
        sel = idx[idx >= 0]
        pool = np.zeros((n_c, c.head_dim), np.uint16)
        pool[sel] = W.host_rows(w, pre + "pool", b * n_c + sel)
        pool[e] = O.store_bf16(ent)
        out = O.csa_attend(H["q"][b, 0], H["q_norm_g"], pool, idx, H["win"][b], c.window, H["sink"], pos, c)
        res[b] = (ent, kent, idx, scores, out)
    return res


def _reattend_with(ly, pool, n_c, win, win_cap, oracle_idx: dict):
    """The layer's attention rerun on the GPU, in the same launch
    configuration, with the oracle's index set substituted for the rows in
    ``oracle_idx`` ((b, t) -> int indices).  Rows whose GPU set differs from
    the oracle's only inside the tie zone are checked this way: the input
    flows from the oracle to the GPU, never back."""
    idx2 = ly.idx.clone()
    for (b, t), ix in oracle_idx.items():
        idx2[b, t] = torch.from_numpy(np.asarray(ix, np.int32)).to(idx2.device)
    out2 = torch.empty_like(ly.out)
    t_ = ly.t
    L.ds4a_sparse_attend(ly.cfg, ly.q_pos, t_["q"], t_["q_norm_g"], pool, n_c, idx2, win, win_cap,
                         t_["sink"], out2, ly.ws_att)
    check_ok()
    return f64(out2)


def _check_csa_decode(st, ly, w, bsel):
    """Every sampled sequence: compressed entries, the top-k set (tie rule)
    and the attention output, each against the oracle's own chain."""
    ref = _decode_csa_ref(w, ly, bsel)
    gpool = ly.t["pool"]
    gki = ly.t["ki"]
    gidx = ly.idx.cpu().numpy()
    gout = f64(ly.out)
    e = w.n_csa - 1
    redo = {}
    for b, (ent, kent, idx, scores, out) in ref.items():
        assert C.max_abs_rel(f64(gpool[b, e]), ent) < C.OUT_TOL
        assert C.max_abs_rel(f64(gki[b, e]), kent) < C.OUT_TOL
        msg = C.check_topk_row(gidx[b, 0], scores, w.csa.topk)
        assert msg is None, f"seq {b}: {msg}"
        if not np.array_equal(gidx[b, 0], idx):
            redo[(b, 0)] = idx
    gout2 = _reattend_with(ly, gpool, ly.n_c, ly.t["win"], ly.t["win"].shape[1], redo) if redo else None
    compared = 0
    for b, (ent, kent, idx, scores, out) in ref.items():
        got = gout2[b, 0] if (b, 0) in redo else gout[b, 0]
        err = C.max_abs_rel(got, out)
        assert err < C.OUT_TOL, f"seq {b}: attend err {err} (oracle index set: {(b, 0) in redo})"
        compared += 1
    assert compared == len(bsel)


def _check_hca_decode(st, ly, w, bsel):
    h = w.hca
    n_c, pos, m = w.n_hca, w.pos, h.ratio
    e = n_c - 1
    tb = pos - m + 1
    pre = ly.prefix + "hca."
    Hh = {n: W.host_tensor(w, pre + n) for n in ("kv_c", "kv_z", "kv_b", "kv_g", "q", "q_norm_g", "sink", "win")}
    gout = f64(ly.out)
    for b in bsel:
        ent = O.compress(m, e, e + 1, tb, Hh["kv_c"][b], Hh["kv_z"][b], Hh["kv_b"], norm_g=Hh["kv_g"],
                         rope_dim=h.rope_dim)[0]
        assert C.max_abs_rel(f64(ly.t["pool"][b, e]), ent) < C.OUT_TOL
        pool = W.host_rows(w, pre + "pool", b * n_c + np.arange(n_c))
        pool[e] = O.store_bf16(ent)
        out = O.hca_attend(Hh["q"][b, 0], Hh["q_norm_g"], pool, n_c, Hh["win"][b], h.window, Hh["sink"], pos, h)
        err = C.max_abs_rel(gout[b, 0], out)
        assert err < C.OUT_TOL, f"seq {b}: err {err}"


def _check_swa_decode(st, ly, w, bsel):
    h = w.hca
    pre = ly.prefix + "swa."
    Hs = {n: W.host_tensor(w, pre + n) for n in ("q", "q_norm_g", "sink", "win")}
    gout = f64(ly.out)
    for b in bsel:
        out = O.hca_attend(Hs["q"][b, 0], Hs["q_norm_g"], np.zeros((0, h.head_dim)), 0, Hs["win"][b], h.window,
                           Hs["sink"], w.pos, h)
        err = C.max_abs_rel(gout[b, 0], out)
        assert err < C.OUT_TOL, f"{ly.prefix} seq {b}: err {err}"


def test_workload_schedule43_decode():
    # one decode step through the 43 layers of the Flash schedule (two
    # window-only layers, then CSA and HCA alternating): every layer's output
    # against the oracle, both sequences
    st = _state(8)
    w = st.w
    kinds = [ly.kind for ly in st.layers]
    assert kinds[:4] == ["swa", "swa", "csa", "hca"] and len(kinds) == 43
    assert kinds.count("csa") == 21 and kinds.count("hca") == 20
    for ly in st.layers:
        if ly.kind == "csa":
            _check_csa_decode(st, ly, w, [0, 1])
        elif ly.kind == "hca":
            _check_hca_decode(st, ly, w, [0, 1])
        else:
            _check_swa_decode(st, ly, w, [0, 1])


def test_workload_toy_csa_prefill():
    st = _state(1)
    w = st.w
    c = w.csa
    ly = st.layers[0]
    x = W.toy_inputs(w)
    qp = W.query_positions(w)
    n = ly.n_c
    pool = O.compress_batch(c.ratio, 0, n, 0, x["csa.kv_ca"], x["csa.kv_za"], x["csa.kv_ba"], x["csa.kv_cb"],
                            x["csa.kv_zb"], x["csa.kv_bb"], x["csa.kv_g"], c.rope_dim)
    ki = O.compress_batch(c.ratio, 0, n, 0, x["csa.ix_ca"], x["csa.ix_za"], x["csa.ix_ba"], x["csa.ix_cb"],
                          x["csa.ix_zb"], x["csa.ix_bb"])
    assert C.max_abs_rel(f64(ly.pool), pool) < C.OUT_TOL
    assert C.max_abs_rel(f64(ly.ki), ki) < C.OUT_TOL
    idx, scores = O.index_topk_batch(x["csa.qi"], x["csa.wi"], O.store_bf16(ki), qp, c.ratio, c.topk, n)
    gidx = ly.idx.cpu().numpy()
    for t in range(64):
        assert C.check_topk_row(gidx[0, t], scores[(0, t)], c.topk) is None
    out = O.csa_attend_batch(x["csa.q"], x["csa.q_norm_g"], O.store_bf16(pool), idx, x["csa.win"], 64,
                             x["csa.sink"], qp, c)
    redo = {(0, t): idx[0, t] for t in range(64) if not np.array_equal(gidx[0, t], idx[0, t])}
    got = f64(ly.out)
    if redo:
        got2 = _reattend_with(ly, ly.pool, n, ly.t["win"], ly.T, redo)
        for (_, t) in redo:
            got[0, t] = got2[0, t]
    # every one of the 64 rows is compared
    assert C.max_abs_rel(got[0], out[0]) < C.OUT_TOL


def test_workload_csa_decode_b1_8k():
    st = _state(2)
    _check_csa_decode(st, st.layers[0], st.w, [0])


def test_workload_hca_decode_b32_128k():
    st = _state(3)
    _check_hca_decode(st, st.layers[0], st.w, list(range(32)))


def test_workload_mix_decode_b8_1m():
    st = _state(5)
    _check_csa_decode(st, st.layers[0], st.w, [0, 3, 7])
    _check_hca_decode(st, st.layers[1], st.w, list(range(8)))


def _tensor_core_path_active():
    cfg = L.layer_cfg(FLASH)
    q = torch.zeros((1, 1, 64, 512), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    z = torch.ones(512, device="cuda")
    idx = torch.full((1, 1, 512), -1, dtype=torch.int32, device="cuda")
    win = torch.zeros((1, 128, 512), dtype=torch.bfloat16, device="cuda")
    ws = ws_f32(L.ds4a_attend_workspace(cfg, 1, 1, 0, True))
    names = kernels_used(lambda: L.ds4a_sparse_attend(cfg, i32([[10]]), q, z, None, 0, idx, win, 128,
                                                      z[:64], out, ws))
    return any("tc" in n for n in names)


def test_workload_csa_prefill_16k_sampled():
    if not _tensor_core_path_active():
        pytest.skip("full 16k prefill runs only on the tensor-core path (the CUDA-core path takes minutes)")
    st = _state(4)
    w = st.w
    c = w.csa
    ly = st.layers[0]
    n = ly.n_c
    Hs = {n_: W.host_tensor(w, f"csa.{n_}") for n_ in ("kv_ca", "kv_cb", "kv_za", "kv_zb", "ix_ca", "ix_cb",
                                                       "ix_za", "ix_zb", "kv_ba", "kv_bb", "ix_ba", "ix_bb",
                                                       "kv_g", "q_norm_g", "sink", "win")}
    pool = O.compress(c.ratio, 0, n, 0, Hs["kv_ca"][0], Hs["kv_za"][0], Hs["kv_ba"], Hs["kv_cb"][0],
                      Hs["kv_zb"][0], Hs["kv_bb"], Hs["kv_g"], c.rope_dim)
    ki = O.compress(c.ratio, 0, n, 0, Hs["ix_ca"][0], Hs["ix_za"][0], Hs["ix_ba"], Hs["ix_cb"][0],
                    Hs["ix_zb"][0], Hs["ix_bb"])
    assert C.max_abs_rel(f64(ly.pool)[0], pool) < C.OUT_TOL
    assert C.max_abs_rel(f64(ly.ki)[0], ki) < C.OUT_TOL
    rng = np.random.default_rng(3)
    rows = sorted(set([0, 1, 3, 127, 128, 2047, 2051, 8191, 16383] + list(rng.integers(0, 16384, 15))))
    gidx = ly.idx.cpu().numpy()
    gout = ly.out
    pb, kb = O.store_bf16(pool), O.store_bf16(ki)
    refs, redo = {}, {}
    for t in rows:
        qi = W.host_rows(w, "csa.qi", t * c.idx_heads + np.arange(c.idx_heads))
        wi = W.host_rows(w, "csa.wi", np.array([t]))[0]
        q = W.host_rows(w, "csa.q", t * c.n_heads + np.arange(c.n_heads))
        idx, scores = O.index_topk(qi, wi, kb, t, c.ratio, c.topk, n)
        msg = C.check_topk_row(gidx[0, t], scores, c.topk)
        assert msg is None, f"row {t}: {msg}"
        refs[t] = O.csa_attend(q, Hs["q_norm_g"], pb, idx, Hs["win"][0], 16384, Hs["sink"], t, c)
        if not np.array_equal(gidx[0, t], idx):
            redo[(0, t)] = idx
    got2 = _reattend_with(ly, ly.pool, n, ly.t["win"], ly.T, redo) if redo else None
    compared = 0
    for t in rows:
        got = got2[0, t] if (0, t) in redo else f64(gout[0, t])
        err = C.max_abs_rel(got, refs[t])
        assert err < C.OUT_TOL, f"row {t}: err {err} (oracle index set: {(0, t) in redo})"
        compared += 1
    assert compared == len(rows)
