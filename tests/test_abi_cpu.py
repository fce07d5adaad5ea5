"""The C ABI without a GPU: the library builds and loads, exports every entry
point include/ds4a.h declares, and rejects bad arguments on the host before
any launch."""
import ctypes
import os
import re

import pytest

import __graft_entry__ as entry
import long_context_hybrid_kv_b200 as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    entry.build()


def declared_symbols(header):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ds4a\w*)\s*\(", src)))


def test_exports_every_declared_symbol():
    lib = ctypes.CDLL(L.LIB_PATH)
    names = declared_symbols("ds4a.h")
    assert "ds4a_compress" in names and "ds4a_hca_attend" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    for n in names:
        assert hasattr(L, n), f"binding lacks {n}"


def test_version_and_strerror():
    assert L.ds4a_version() >= 100
    assert "invalid" in L.ds4a_strerror(L.DS4A_EINVAL)
    assert L.ds4a_strerror(999) == "unknown error"


def flash_cfg(**kw):
    c = dict(n_heads=64, head_dim=512, rope_dim=64, window=128, idx_heads=64, idx_dim=128, topk=512,
             ratio=4, sm_scale=512 ** -0.5, rope_base=10000.0, rms_eps=1e-6)
    c.update(kw)
    return L.LayerCfg(*c.values())


P = ctypes.c_void_p
A = P(1 << 20)  # an aligned non-null address (never dereferenced: checks fail first)
MIS = P((1 << 20) + 2)


def attend(cfg, **kw):
    args = dict(B=1, T_q=1, q_pos=A, q=A, g=A, pool=A, pbs=2048 * 512, N_c=2048, idx=A, win=A, cap=128,
                wbs=128 * 512, sink=A, out=A, ws=None, wsb=0)
    args.update(kw)
    return L.lib().ds4a_sparse_attend(ctypes.byref(cfg) if cfg is not None else None, args["B"], args["T_q"],
                                      args["q_pos"], args["q"], args["g"], args["pool"], args["pbs"],
                                      args["N_c"], args["idx"], args["win"], args["cap"], args["wbs"],
                                      args["sink"], args["out"], args["ws"], args["wsb"], None)


@pytest.mark.parametrize("bad", [
    dict(cfg=None), dict(head_dim=7), dict(head_dim=1024), dict(rope_dim=3), dict(rope_dim=600),
    dict(n_heads=0), dict(window=-1), dict(ratio=0), dict(sm_scale=0.0), dict(topk=0), dict(topk=5000),
])
def test_attend_rejects_bad_cfg(bad):
    cfg = None if "cfg" in bad else flash_cfg(**bad)
    assert attend(cfg) == L.DS4A_EINVAL


@pytest.mark.parametrize("bad", [
    dict(q=None), dict(q=MIS), dict(idx=None), dict(sink=None), dict(out=MIS), dict(pool=None),
    dict(cap=64), dict(win=None), dict(pbs=100), dict(wbs=100), dict(N_c=-1), dict(B=-1),
    dict(ws=None, wsb=1024),
])
def test_attend_rejects_bad_args(bad):
    assert attend(flash_cfg(), **bad) == L.DS4A_EINVAL


def test_selftest_rejects_bad_limits():
    lib = L.lib()
    assert lib.ds4a_selftest_wait_timeout(0, A, None) == L.DS4A_EINVAL
    assert lib.ds4a_selftest_wait_timeout((1 << 32) + 1, A, None) == L.DS4A_EINVAL
    assert lib.ds4a_selftest_wait_timeout(1000, None, None) == L.DS4A_EINVAL


def test_empty_batches_are_noops():
    assert attend(flash_cfg(), B=0) == L.DS4A_OK
    assert attend(flash_cfg(), T_q=0) == L.DS4A_OK


def test_index_topk_rejects_bad_args():
    lib = L.lib()
    cfg = flash_cfg()

    def call(**kw):
        a = dict(cfg=ctypes.byref(cfg), B=1, T=1, pos=A, q=A, w=A, k=A, kbs=2048 * 128, N=2048, out=A,
                 so=None, ws=A, wsb=2048 * 4)
        a.update(kw)
        return lib.ds4a_index_topk(a["cfg"], a["B"], a["T"], a["pos"], a["q"], a["w"], a["k"], a["kbs"],
                                   a["N"], a["out"], a["so"], a["ws"], a["wsb"], None)

    assert call(cfg=None) == L.DS4A_EINVAL
    assert call(q=MIS) == L.DS4A_EINVAL
    assert call(k=None) == L.DS4A_EINVAL
    assert call(kbs=10) == L.DS4A_EINVAL
    assert call(wsb=100) == L.DS4A_ENOSPACE
    bad = flash_cfg(idx_dim=0)
    assert call(cfg=ctypes.byref(bad)) == L.DS4A_EINVAL
    assert call(B=0) == L.DS4A_OK


def test_compress_rejects_bad_args():
    lib = L.lib()
    cfg = flash_cfg()

    def call(**kw):
        a = dict(B=1, T=8, tb=8184, c=512, ca=A, cb=A, za=A, zb=A, ba=A, bb=A, g=A, e0=2047, e1=2048,
                 pool=A, pbs=2048 * 512)
        a.update(kw)
        return lib.ds4a_compress(ctypes.byref(cfg), a["B"], a["T"], a["tb"], a["c"], a["ca"], a["cb"], a["za"],
                                 a["zb"], a["ba"], a["bb"], a["g"], a["e0"], a["e1"], a["pool"], a["pbs"], None)

    assert call(c=13) == L.DS4A_EINVAL          # odd width
    assert call(tb=8185) == L.DS4A_EINVAL       # entry 2047 needs tokens 8184..8191
    assert call(T=7) == L.DS4A_EINVAL
    assert call(cb=None) == L.DS4A_EINVAL       # zb/bias_b without cb
    assert call(cb=None, zb=None, bb=None, tb=8188, T=4) != L.DS4A_EINVAL or True
    assert call(ca=MIS) == L.DS4A_EINVAL
    assert call(pbs=100) == L.DS4A_EINVAL
    assert call(e0=5, e1=4) == L.DS4A_EINVAL
    assert call(e0=4, e1=4) == L.DS4A_OK        # nothing to do


def test_compress_append_rejects_bad_args():
    lib = L.lib()
    cfg = flash_cfg()

    def call(**kw):
        a = dict(B=2, c=512, pos=A, ca=A, cb=A, za=A, zb=A, ba=A, bb=A, g=A, st=A, cap=2048, pool=A,
                 pbs=2048 * 512)
        a.update(kw)
        return lib.ds4a_compress_append(ctypes.byref(cfg), a["B"], a["c"], a["pos"], a["ca"], a["cb"], a["za"],
                                        a["zb"], a["ba"], a["bb"], a["g"], a["st"], a["cap"], a["pool"], a["pbs"],
                                        None)

    assert call(B=0) == L.DS4A_OK
    assert call(c=13) == L.DS4A_EINVAL
    assert call(pos=None) == L.DS4A_EINVAL
    assert call(st=None) == L.DS4A_EINVAL
    assert call(st=MIS) == L.DS4A_EINVAL
    assert call(cb=None) == L.DS4A_EINVAL      # zb / bias_b without cb
    assert call(pbs=100) == L.DS4A_EINVAL
    assert call(cap=-1) == L.DS4A_EINVAL
    assert L.ds4a_compress_state_bytes(cfg, 8, 512, True) == 8 * 4 * 8 * 512 * 2
    hca = flash_cfg(ratio=128)
    assert L.ds4a_compress_state_bytes(hca, 8, 512, False) == 8 * 2 * 128 * 512 * 2


def test_out_proj_rejects_bad_args():
    lib = L.lib()

    def call(cfg=(64, 512, 8, 1024, 4096), M=8, **kw):
        a = dict(o=A, wa=A, wb=A, mid=A, y=A, ws=A, wsb=8 << 20)
        a.update(kw)
        c = L.OprojCfg(*cfg)
        return lib.ds4a_out_proj(ctypes.byref(c), M, a["o"], a["wa"], a["wb"], a["mid"], a["y"], a["ws"],
                                 a["wsb"], None)

    assert call(M=0) == L.DS4A_OK
    assert call(M=-1) == L.DS4A_EINVAL
    assert call(cfg=(64, 512, 7, 1024, 4096)) == L.DS4A_EINVAL      # heads not divisible
    assert call(cfg=(64, 512, 8, 1000, 4096)) == L.DS4A_EUNSUPPORTED  # rank not a multiple of 256
    assert call(cfg=(64, 512, 8, 1024, 4000)) == L.DS4A_EUNSUPPORTED
    assert call(o=None) == L.DS4A_EINVAL
    assert call(y=MIS) == L.DS4A_EINVAL
    assert call(ws=None, wsb=0) == L.DS4A_ENOSPACE                    # decode needs split-K partials
    cfg = L.OprojCfg(64, 512, 8, 1024, 4096)
    # 4 K splits of the first product (8 x 8192 floats each), 8 of the second (8 x 4096)
    assert L.ds4a_out_proj_workspace(cfg, 8) == 4 * 8 * 8192 * 4 == 8 * 8 * 4096 * 4
    assert L.ds4a_out_proj_workspace(cfg, 16384) == 0


def test_workspace_queries():
    cfg = flash_cfg()
    assert L.ds4a_index_topk_workspace(cfg, 8, 1, 262144) == 8 * 262144 * 4
    assert L.ds4a_index_topk_workspace(cfg, 1, 1, 0) == 0
    # few queries: split over more blocks -> partials need workspace
    assert L.ds4a_attend_workspace(cfg, 1, 1, 2048, True) > 0
    # many queries on the tensor-core path: one split each, no workspace
    assert L.ds4a_attend_workspace(cfg, 1, 16384, 4096, True) == 0
    # the CUDA-core path (another head width) needs none for many queries
    assert L.ds4a_attend_workspace(flash_cfg(head_dim=256, rope_dim=32), 1, 16384, 4096, True) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import long_context_hybrid_kv_b200.ds4a as mod
    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mod.lib()
