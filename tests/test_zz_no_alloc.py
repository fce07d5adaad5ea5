"""ds4a_index_topk_noalloc, the entry point for callers that cannot allocate
device memory (it uses the library's own fixed scratch instead of a caller
workspace), against ds4a_index_topk with a workspace on the same inputs,
for two calls in a row.  Kept in a file of its own that runs last."""
import ctypes

import numpy as np
import pytest
import torch

import long_context_hybrid_kv_b200 as L
from gen import host
from gen import workloads as W

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Tq, n_c, positions):
    c = W.FLASH_CSA
    dev = torch.device("cuda:0")

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    qi = bf(host.normal_bf16(seed, "na.qi", (B, Tq, c.idx_heads, c.idx_dim)))
    wi = bf(host.normal_bf16(seed, "na.wi", (B, Tq, c.idx_heads)))
    ki = bf(host.normal_bf16(seed, "na.ki", (B, n_c, c.idx_dim)))
    pos = torch.tensor(np.tile(np.asarray(positions, np.int32), (B, 1)), device=dev)
    return pos, qi, wi, ki


@pytest.mark.parametrize("shape", [(1, 1, 2048, [8191]), (2, 3, 5000, [3, 4095, 19999])])
def test_noalloc_matches_workspace_call(shape):
    torch.cuda.set_device(0)
    B, Tq, n_c, positions = shape
    cfg = L.layer_cfg(W.FLASH_CSA)
    k = W.FLASH_CSA.topk
    for call, seed in enumerate((11, 12)):  # two calls in a row, different inputs
        pos, qi, wi, ki = _inputs(seed, B, Tq, n_c, positions)
        idx_ref = torch.empty((B, Tq, k), dtype=torch.int32, device="cuda")
        sc_ref = torch.empty((B, Tq, k), dtype=torch.float32, device="cuda")
        ws = torch.empty(L.ds4a_index_topk_workspace(cfg, B, Tq, n_c) // 4, dtype=torch.float32, device="cuda")
        L.ds4a_index_topk(cfg, pos, qi, wi, ki, n_c, idx_ref, ws, score_out=sc_ref)
        idx = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
        sc = torch.full((B, Tq, k), 7.0, dtype=torch.float32, device="cuda")
        L.ds4a_index_topk_noalloc(cfg, pos, qi, wi, ki, n_c, idx, score_out=sc)
        rc, bits = L.ds4a_check()
        assert rc == 0, (rc, bits)
        assert torch.equal(idx, idx_ref), f"call {call}: indices differ"
        a, b = sc.cpu().numpy(), sc_ref.cpu().numpy()
        fin = np.isfinite(b)
        assert np.array_equal(np.isfinite(a), fin)
        assert np.max(np.abs(a[fin] - b[fin]) / (np.abs(b[fin]) + 1e-6)) <= 1e-6, f"call {call}: scores differ"


def test_noalloc_fills_the_whole_scratch():
    # exactly 2^21 scores (B * T_q * N_c = 1 * 16 * 131072) on the
    # tensor-core scorer: accepted, and equal to the workspace call; one
    # more entry is rejected
    torch.cuda.set_device(0)
    B, Tq, n_c = 1, 16, 131072
    positions = [4 * n_c - 1 - 37 * i for i in range(Tq)]
    cfg = L.layer_cfg(W.FLASH_CSA)
    k = W.FLASH_CSA.topk
    for call, seed in enumerate((21, 22)):
        pos, qi, wi, ki = _inputs(seed, B, Tq, n_c, positions)
        idx_ref = torch.empty((B, Tq, k), dtype=torch.int32, device="cuda")
        ws = torch.empty(L.ds4a_index_topk_workspace(cfg, B, Tq, n_c) // 4, dtype=torch.float32, device="cuda")
        L.ds4a_index_topk(cfg, pos, qi, wi, ki, n_c, idx_ref, ws)
        idx = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
        L.ds4a_index_topk_noalloc(cfg, pos, qi, wi, ki, n_c, idx)
        rc, bits = L.ds4a_check()
        assert rc == 0, (rc, bits)
        assert torch.equal(idx, idx_ref), f"call {call}: indices differ"
    kbig = torch.empty((B, n_c + 1, W.FLASH_CSA.idx_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.Ds4aError) as ex:
        L.ds4a_index_topk_noalloc(cfg, pos, qi, wi, kbig, n_c + 1, idx)
    assert ex.value.code == L.DS4A_ENOSPACE


def test_noalloc_rejects_sizes_beyond_its_scratch():
    cfg = L.layer_cfg(W.FLASH_CSA)
    A = ctypes.c_void_p(1 << 20)
    rc = L.lib().ds4a_index_topk_noalloc(ctypes.byref(cfg), 9, 1, A, A, A, A, 262144 * 128, 262144, A, None, None)
    assert rc == L.DS4A_ENOSPACE
