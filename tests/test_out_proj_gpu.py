"""The grouped low-rank output projection (ds4a_out_proj) against the fp64
oracle: a small shape spanning several row tiles with a ragged last one,
and the Flash shape (64 heads x 512 in 8 groups, rank 1024, hidden 4096) at
decode size (split-K path) and at prefill size on sampled rows.  Tolerance:
max-abs-relative 1e-2 per row (bf16 storage, float32 accumulation)."""
import math

import numpy as np
import pytest
import torch

import long_context_hybrid_kv_b200 as L
from gen import host
from gpu_util import bf, bits, check_ok, f64, ws_f32
from oracle import compare as C
from oracle import ds4a_oracle as O

pytestmark = pytest.mark.gpu
SEED = 909


def _inputs(name, M, H, D, g, r, hidden):
    k1 = (H // g) * D
    o = host.normal_bf16(SEED, f"{name}.o", (M, H, D))
    wa = host.normal_bf16(SEED, f"{name}.wa", (g, r, k1), 1 / math.sqrt(k1))
    wb = host.normal_bf16(SEED, f"{name}.wb", (hidden, g * r), 1 / math.sqrt(g * r))
    return o, wa, wb


def _run(name, M, H, D, g, r, hidden):
    cfg = L.OprojCfg(H, D, g, r, hidden)
    o, wa, wb = _inputs(name, M, H, D, g, r, hidden)
    mid = torch.empty((M, g * r), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, hidden), dtype=torch.bfloat16, device="cuda")
    ws = ws_f32(L.ds4a_out_proj_workspace(cfg, M))
    L.ds4a_out_proj(cfg, bf(o), bf(wa), bf(wb), mid, y, ws)
    check_ok()
    return o, wa, wb, mid, y


def _check_rows(o, wa, wb, mid, y, g, rows):
    ref_mid, ref_y = O.out_proj(o[rows], wa, wb, g)
    gm, gy = f64(mid)[rows], f64(y)[rows]
    for i, t in enumerate(rows):
        e1 = C.max_abs_rel(gm[i], ref_mid[i])
        assert e1 < C.OUT_TOL, f"row {t}: intermediate err {e1}"
    # the second product from the oracle's own stored intermediate
    for i, t in enumerate(rows):
        e2 = C.max_abs_rel(gy[i], ref_y[i])
        assert e2 < C.OUT_TOL, f"row {t}: output err {e2}"


@pytest.mark.parametrize("M", [1, 5, 130, 300])
def test_out_proj_small(M):
    # 8 heads x 64 in 2 groups (K 256 per group), rank 256, hidden 512
    H, D, g, r, hidden = 8, 64, 2, 256, 512
    o, wa, wb, mid, y = _run(f"small{M}", M, H, D, g, r, hidden)
    _check_rows(o, wa, wb, mid, y, g, list(range(M)))


def test_out_proj_flash_decode():
    # 8 tokens: the weights stream through split-K partial sums
    o, wa, wb, mid, y = _run("fdec", 8, 64, 512, 8, 1024, 4096)
    _check_rows(o, wa, wb, mid, y, 8, list(range(8)))


def test_out_proj_flash_prefill_sampled():
    M = 4096 + 77
    o, wa, wb, mid, y = _run("fpre", M, 64, 512, 8, 1024, 4096)
    rng = np.random.default_rng(5)
    rows = sorted(set([0, 1, 127, 128, 2047, M - 78, M - 1] + list(rng.integers(0, M, 9))))
    _check_rows(o, wa, wb, mid, y, 8, rows)


def test_out_proj_two_calls_and_bad_shapes():
    # the split-K workspace is cleared by every call: a second call gives the
    # same bits
    cfg = L.OprojCfg(64, 512, 8, 1024, 4096)
    o, wa, wb = _inputs("twice", 8, 64, 512, 8, 1024, 4096)
    ws = ws_f32(L.ds4a_out_proj_workspace(cfg, 8))
    outs = []
    for _ in range(2):
        mid = torch.empty((8, 8192), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((8, 4096), dtype=torch.bfloat16, device="cuda")
        L.ds4a_out_proj(cfg, bf(o), bf(wa), bf(wb), mid, y, ws)
        check_ok()
        outs.append(bits(y))
    assert np.array_equal(outs[0], outs[1])
    with pytest.raises(L.Ds4aError) as ex:
        L.ds4a_out_proj(L.OprojCfg(64, 512, 8, 1000, 4096), bf(o), bf(wa), bf(wb), mid, y, ws)
    assert ex.value.code == L.DS4A_EUNSUPPORTED
