"""The compressor's decode-time cache (ds4a_compress_append): a decode that
appends 4096 tokens one call at a time, for two sequences at different
positions, must leave in the pool exactly the entries the oracle's batch
compressor makes from the full streams (CSA K=V with RMSNorm and RoPE, CSA
indexer keys, HCA K=V).  Tolerance: max-abs-relative 1e-2 (bf16 storage,
float32 arithmetic)."""
import math

import numpy as np
import pytest
import torch

import long_context_hybrid_kv_b200 as L
from gen import host
from gen import workloads as W
from gpu_util import bf, check_ok, f32, f64
from oracle import compare as C
from oracle import ds4a_oracle as O

pytestmark = pytest.mark.gpu

SEED = 777
T = 4096
LAG = 2  # sequence 1 runs LAG positions ahead of sequence 0


def _case(name, c, m, overlap, norm, R):
    B = 2
    n_tok = T + LAG
    streams = {s: host.normal_bf16(SEED, f"{name}.{s}", (B, n_tok, c)) for s in (["ca", "cb", "za", "zb"]
                                                                                 if overlap else ["ca", "za"])}
    # sequence 0 starts at position 0 and never sees tokens T .. T+LAG-1;
    # sequence 1 starts at position LAG: its first LAG tokens were never
    # appended and read as the zeroed state
    for s in streams.values():
        s[1, :LAG] = 0
    ba = host.normal_f32(SEED, f"{name}.ba", (m, c), 1 / math.sqrt(m))
    bb = host.normal_f32(SEED, f"{name}.bb", (m, c), 1 / math.sqrt(m)) if overlap else None
    g = host.normal_f32(SEED, f"{name}.g", (c,), 0.1, 1.0) if norm else None
    cfg = L.LayerCfg(64, 512, R, 128, 64, 128, 512, m, 512 ** -0.5, 10000.0, 1e-6)
    n_cap = n_tok // m
    pool = torch.full((B, n_cap, c), float("nan"), dtype=torch.bfloat16, device="cuda")
    state = torch.zeros(L.ds4a_compress_state_bytes(cfg, B, c, overlap) // 2, dtype=torch.bfloat16, device="cuda")
    dev = {k: bf(v) for k, v in streams.items()}
    ba_d, bb_d = f32(ba), (f32(bb) if overlap else None)
    g_d = f32(g) if norm else None
    steps = torch.arange(T, dtype=torch.int32, device="cuda")
    for t in range(T):
        pos = torch.stack([steps[t], steps[t] + LAG])
        rows = {k: torch.stack([v[0, t], v[1, t + LAG]]) for k, v in dev.items()}
        L.ds4a_compress_append(cfg, pos, rows["ca"], rows["za"], ba_d, state, pool,
                               cb=rows.get("cb"), zb=rows.get("zb"), bias_b=bb_d, norm_g=g_d)
    check_ok()
    got = f64(pool)
    for b, last in ((0, T - 1), (1, T - 1 + LAG)):
        n = (last + 1) // m
        ref = O.compress(m, 0, n, 0, streams["ca"][b], streams["za"][b], ba, streams.get("cb", [None] * 2)[b],
                         streams.get("zb", [None] * 2)[b], bb, g, R)
        err = C.max_abs_rel(got[b, :n], ref)
        assert err < C.OUT_TOL, f"{name} seq {b}: err {err}"
        assert np.isnan(got[b, n:]).all(), f"{name} seq {b}: entries past the last closed one were written"
    return cfg, state, pool


def test_append_csa_kv():
    _case("ap_kv", 512, 4, True, True, 64)


def test_append_csa_index_keys():
    _case("ap_ix", 128, 4, True, False, 0)


def test_append_hca_kv():
    _case("ap_hca", 512, 128, False, True, 64)


def test_append_reports_full_pool_and_bad_position():
    cfg = L.LayerCfg(64, 512, 0, 128, 64, 128, 512, 4, 512 ** -0.5, 10000.0, 1e-6)
    c = 128
    rows = torch.zeros((1, c), dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros((4, c), dtype=torch.float32, device="cuda")
    state = torch.zeros(L.ds4a_compress_state_bytes(cfg, 1, c, True) // 2, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((1, 2, c), dtype=torch.bfloat16, device="cuda")
    # position 11 closes entry 2, beyond a pool of 2 entries
    L.ds4a_compress_append(cfg, torch.tensor([11], dtype=torch.int32, device="cuda"), rows, rows, bias, state, pool,
                           cb=rows, zb=rows, bias_b=bias)
    rc, b = L.ds4a_check()
    assert rc == L.DS4A_EDEVICE and (b & 1), (rc, b)
    L.ds4a_compress_append(cfg, torch.tensor([-1], dtype=torch.int32, device="cuda"), rows, rows, bias, state, pool,
                           cb=rows, zb=rows, bias_b=bias)
    rc, b = L.ds4a_check()
    assert rc == L.DS4A_EDEVICE and (b & 2), (rc, b)
    assert float(pool.float().abs().max()) == 0.0


def test_append_jobs_equal_separate_calls():
    # a CSA layer's two compressors in one ds4a_compress_append_jobs launch
    # give the same bits as two ds4a_compress_append calls
    B, T = 3, 96
    cfg = L.LayerCfg(64, 512, 64, 128, 64, 128, 512, 4, 512 ** -0.5, 10000.0, 1e-6)
    outs = []
    for mode in ("jobs", "separate"):
        pools, states, args = [], [], []
        for name, c, norm in (("jkv", 512, True), ("jix", 128, False)):
            st = {s: bf(host.normal_bf16(SEED, f"{name}.{s}", (B, T, c))) for s in ("ca", "cb", "za", "zb")}
            ba = f32(host.normal_f32(SEED, f"{name}.ba", (4, c), 0.5))
            bb = f32(host.normal_f32(SEED, f"{name}.bb", (4, c), 0.5))
            g = f32(host.normal_f32(SEED, f"{name}.g", (c,), 0.1, 1.0)) if norm else None
            state = torch.zeros(L.ds4a_compress_state_bytes(cfg, B, c, True) // 2, dtype=torch.bfloat16,
                                device="cuda")
            pool = torch.zeros((B, T // 4, c), dtype=torch.bfloat16, device="cuda")
            pools.append(pool)
            args.append((st, ba, bb, g, state, pool))
        for t in range(T):
            pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
            rows = [{k: v[:, t].contiguous() for k, v in a[0].items()} for a in args]
            if mode == "jobs":
                jobs = [L.append_job(r["ca"], r["za"], a[1], a[4], a[5], cb=r["cb"], zb=r["zb"], bias_b=a[2],
                                     norm_g=a[3]) for r, a in zip(rows, args)]
                L.ds4a_compress_append_jobs(cfg, pos, T // 4, jobs)
            else:
                for r, a in zip(rows, args):
                    L.ds4a_compress_append(cfg, pos, r["ca"], r["za"], a[1], a[4], a[5], cb=r["cb"], zb=r["zb"],
                                           bias_b=a[2], norm_g=a[3])
        check_ok()
        outs.append([p.view(torch.int16).cpu().numpy() for p in pools])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)
