"""Thin ctypes binding of libds4a (include/ds4a.h): argument marshalling only.

Every function has the name of its C entry point and takes torch tensors
(device memory) where the C call takes device pointers; every step of the
path runs in the library's CUDA kernels.  A missing library raises; there is
no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "DS4A_OK", "DS4A_EINVAL", "DS4A_EUNSUPPORTED", "DS4A_ECUDA", "DS4A_EDEVICE", "DS4A_ETIMEOUT",
    "DS4A_ENOSPACE", "Ds4aError", "LayerCfg", "layer_cfg", "lib", "LIB_PATH", "ds4a_compress",
    "ds4a_compress_state_bytes", "ds4a_compress_append", "ds4a_index_topk_workspace", "ds4a_index_topk", "ds4a_index_topk_noalloc", "ds4a_attend_workspace", "ds4a_sparse_attend",
    "ds4a_hca_attend", "ds4a_check", "ds4a_strerror", "ds4a_trace_enable", "ds4a_trace_read",
    "ds4a_version", "ds4a_selftest_wait_timeout", "OprojCfg", "ds4a_out_proj_workspace", "ds4a_out_proj",
    "DS4A_MX_KV_FP8", "DS4A_MX_IDX_FP4", "ds4a_kv_fp8_row_bytes", "ds4a_quantize_kv_fp8", "ds4a_quantize_idx_fp4",
    "ds4a_compress_append_mx", "ds4a_index_topk_fp4", "ds4a_sparse_attend_fp8", "ds4a_hca_attend_fp8",
    "AppendJob", "append_job", "ds4a_compress_append_jobs",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libds4a.so")

DS4A_OK, DS4A_EINVAL, DS4A_EUNSUPPORTED, DS4A_ECUDA, DS4A_EDEVICE, DS4A_ETIMEOUT, DS4A_ENOSPACE = range(7)
DS4A_MX_KV_FP8, DS4A_MX_IDX_FP4 = 1, 2


class Ds4aError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {ds4a_strerror(code)} (code {code})")


class LayerCfg(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("window", ctypes.c_int32),
                ("idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("ratio", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("rope_base", ctypes.c_float),
                ("rms_eps", ctypes.c_float)]


class OprojCfg(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("group_rank", ctypes.c_int32), ("hidden", ctypes.c_int32)]


class AppendJob(ctypes.Structure):
    _fields_ = [("c", ctypes.c_int32), ("format", ctypes.c_int32),
                ("ca", ctypes.c_void_p), ("cb", ctypes.c_void_p), ("za", ctypes.c_void_p), ("zb", ctypes.c_void_p),
                ("bias_a", ctypes.c_void_p), ("bias_b", ctypes.c_void_p), ("norm_g", ctypes.c_void_p),
                ("state", ctypes.c_void_p), ("pool", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("pool_bstride", ctypes.c_int64)]


def layer_cfg(c) -> LayerCfg:
    """LayerCfg from any object with the fields of ds4a_layer_cfg
    (sm_scale defaults to 1/sqrt(head_dim))."""
    scale = getattr(c, "sm_scale", None) or 1.0 / math.sqrt(c.head_dim)
    return LayerCfg(c.n_heads, c.head_dim, c.rope_dim, c.window, c.idx_heads, c.idx_dim, c.topk,
                    c.ratio, scale, getattr(c, "rope_base", 10000.0), getattr(c, "rms_eps", 1e-6))


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_CFG = ctypes.POINTER(LayerCfg)

_SIGS = {
    "ds4a_compress": (_I, [_CFG, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _I64, _P]),
    "ds4a_compress_state_bytes": (_SZ, [_CFG, _I, _I, _I]),
    "ds4a_compress_append": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _I64, _P]),
    "ds4a_index_topk_workspace": (_SZ, [_CFG, _I, _I, _I]),
    "ds4a_compress_append_jobs": (_I, [_CFG, _I, _P, _I, ctypes.POINTER(AppendJob), _I, _P]),
    "ds4a_kv_fp8_row_bytes": (_SZ, [_I, _I]),
    "ds4a_quantize_kv_fp8": (_I, [_I, _I, _I, _P, _I64, _P, _I64, _P]),
    "ds4a_quantize_idx_fp4": (_I, [_I, _I, _P, _I64, _P, _P, _P]),
    "ds4a_compress_append_mx": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _I64, _P]),
    "ds4a_index_topk_fp4": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _P, _I64, _I, _P, _P, _P, _SZ, _P]),
    "ds4a_sparse_attend_fp8": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _I64, _I, _P, _P, _I, _I64, _P, _P, _P, _SZ, _P]),
    "ds4a_hca_attend_fp8": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _I64, _I, _P, _I, _I64, _P, _P, _P, _SZ, _P]),
    "ds4a_index_topk": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _I64, _I, _P, _P, _P, _SZ, _P]),
    "ds4a_index_topk_noalloc": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _I64, _I, _P, _P, _P]),
    "ds4a_attend_workspace": (_SZ, [_CFG, _I, _I, _I, _I]),
    "ds4a_sparse_attend": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _I64, _I, _P, _P, _I, _I64, _P, _P, _P, _SZ, _P]),
    "ds4a_hca_attend": (_I, [_CFG, _I, _I, _P, _P, _P, _P, _I64, _I, _P, _I, _I64, _P, _P, _P, _SZ, _P]),
    "ds4a_check": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "ds4a_out_proj_workspace": (_SZ, [ctypes.POINTER(OprojCfg), _I]),
    "ds4a_out_proj": (_I, [ctypes.POINTER(OprojCfg), _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "ds4a_selftest_wait_timeout": (_I, [_I64, _P, _P]),
    "ds4a_strerror": (ctypes.c_char_p, [_I]),
    "ds4a_trace_enable": (_I, [_I]),
    "ds4a_trace_read": (_I, [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float), _I]),
    "ds4a_version": (_I, []),
}


def lib():
    """The loaded libds4a (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


# plain ints (or None) for pointer arguments: ctypes converts them through
# the c_void_p argtypes without a wrapper object per argument
def _ptr(t):
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ok(rc: int, where: str):
    if rc != DS4A_OK:
        raise Ds4aError(rc, where)


def _bf16(t, name):
    import torch
    if t is not None:
        if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
            raise TypeError(f"{name} must hold bfloat16 storage, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    return t


def ds4a_strerror(code: int) -> str:
    return lib().ds4a_strerror(code).decode()


def ds4a_version() -> int:
    return lib().ds4a_version()


def ds4a_compress(cfg: LayerCfg, ca, za, bias_a, pool, *, entry_begin: int, entry_end: int,
                  cb=None, zb=None, bias_b=None, norm_g=None, tok_begin: int = 0, stream=None):
    """Streams [B, T_tok, c] (row r = token tok_begin + r) -> pool[b, i, :] for
    entry_begin <= i < entry_end.  cb None selects the single-stream HCA form;
    norm_g None stores the raw weighted sum (indexer keys)."""
    _bf16(ca, "ca"), _bf16(za, "za"), _bf16(cb, "cb"), _bf16(zb, "zb")
    B, T_tok, c = ca.shape
    rc = lib().ds4a_compress(ctypes.byref(cfg), B, T_tok, tok_begin, c, _ptr(ca), _ptr(cb), _ptr(za),
                             _ptr(zb), _ptr(bias_a), _ptr(bias_b), _ptr(norm_g), entry_begin,
                             entry_end, _ptr(pool), pool.stride(0), _stream(stream))
    _ok(rc, "ds4a_compress")


def ds4a_compress_state_bytes(cfg: LayerCfg, B: int, c: int, overlap: bool) -> int:
    return lib().ds4a_compress_state_bytes(ctypes.byref(cfg), B, c, int(bool(overlap)))


def ds4a_compress_append(cfg: LayerCfg, pos, ca, za, bias_a, state, pool, *, cb=None, zb=None, bias_b=None,
                         norm_g=None, stream=None):
    """New token rows ca/za (cb/zb) [B, c] at positions pos [B] into the
    ring state; entries that close go to pool [B, N_cap, c]."""
    _bf16(ca, "ca"), _bf16(za, "za"), _bf16(cb, "cb"), _bf16(zb, "zb")
    B, c = ca.shape
    rc = lib().ds4a_compress_append(ctypes.byref(cfg), B, c, _ptr(pos), _ptr(ca), _ptr(cb), _ptr(za), _ptr(zb),
                                    _ptr(bias_a), _ptr(bias_b), _ptr(norm_g), _ptr(state), pool.shape[1],
                                    _ptr(pool), pool.stride(0), _stream(stream))
    _ok(rc, "ds4a_compress_append")


def ds4a_kv_fp8_row_bytes(D: int, R: int) -> int:
    return lib().ds4a_kv_fp8_row_bytes(D, R)


def ds4a_quantize_kv_fp8(rows, R: int, out, *, stream=None):
    """bf16 K=V rows [n, D] -> FP8 / BF16 rows out [n, row_bytes] (uint8)."""
    _bf16(rows, "rows")
    n, D = rows.reshape(-1, rows.shape[-1]).shape
    rc = lib().ds4a_quantize_kv_fp8(n, D, R, _ptr(rows), D, _ptr(out), out.shape[-1], _stream(stream))
    _ok(rc, "ds4a_quantize_kv_fp8")


def ds4a_quantize_idx_fp4(keys, codes, scales, *, stream=None):
    """bf16 indexer keys [n, D] -> E2M1 codes [n, D/2] and E8M0 scales [n, D/32] (uint8)."""
    _bf16(keys, "keys")
    n, D = keys.reshape(-1, keys.shape[-1]).shape
    rc = lib().ds4a_quantize_idx_fp4(n, D, _ptr(keys), D, _ptr(codes), _ptr(scales), _stream(stream))
    _ok(rc, "ds4a_quantize_idx_fp4")


def ds4a_compress_append_mx(cfg: LayerCfg, pos, ca, za, bias_a, state, fmt: int, pool, *, scales=None, cb=None,
                            zb=None, bias_b=None, norm_g=None, stream=None):
    """ds4a_compress_append writing block-scaled entries: pool is uint8
    [B, N_cap, row_bytes] (FP8 K=V) or [B, N_cap, c/2] (FP4 keys, with
    scales [B, N_cap, c/32])."""
    _bf16(ca, "ca"), _bf16(za, "za"), _bf16(cb, "cb"), _bf16(zb, "zb")
    B, c = ca.shape
    rc = lib().ds4a_compress_append_mx(ctypes.byref(cfg), B, c, _ptr(pos), _ptr(ca), _ptr(cb), _ptr(za), _ptr(zb),
                                       _ptr(bias_a), _ptr(bias_b), _ptr(norm_g), _ptr(state), pool.shape[1], fmt,
                                       _ptr(pool), _ptr(scales), pool.shape[1], _stream(stream))
    _ok(rc, "ds4a_compress_append_mx")


def ds4a_index_topk_fp4(cfg: LayerCfg, q_pos, q_idx, w_idx, k_codes, k_scales, N_c: int, idx_out, ws, *,
                        score_out=None, stream=None):
    """ds4a_index_topk over FP4 keys: k_codes [B, >=N_c, D/2], k_scales [B, >=N_c, D/32]."""
    _bf16(q_idx, "q_idx"), _bf16(w_idx, "w_idx")
    B, T_q = q_pos.shape
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().ds4a_index_topk_fp4(ctypes.byref(cfg), B, T_q, _ptr(q_pos), _ptr(q_idx), _ptr(w_idx), _ptr(k_codes),
                                   _ptr(k_scales), 0 if k_codes is None else k_codes.shape[1], N_c, _ptr(idx_out),
                                   _ptr(score_out), _ptr(ws), ws_bytes, _stream(stream))
    _ok(rc, "ds4a_index_topk_fp4")


def ds4a_sparse_attend_fp8(cfg: LayerCfg, q_pos, q, q_norm_g, pool, N_c: int, idx, win, win_cap: int, sink, out,
                           ws=None, *, stream=None):
    """ds4a_sparse_attend over an FP8 / BF16 pool: uint8 [B, >=N_c, row_bytes]."""
    _bf16(q, "q")
    B, T_q = q_pos.shape
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().ds4a_sparse_attend_fp8(ctypes.byref(cfg), B, T_q, _ptr(q_pos), _ptr(q), _ptr(q_norm_g), _ptr(pool),
                                      0 if pool is None else pool.shape[1], N_c, _ptr(idx), _ptr(win), win_cap,
                                      0 if win is None else win.stride(0), _ptr(sink), _ptr(out), _ptr(ws), ws_bytes,
                                      _stream(stream))
    _ok(rc, "ds4a_sparse_attend_fp8")


def ds4a_hca_attend_fp8(cfg: LayerCfg, q_pos, q, q_norm_g, pool, N_c: int, win, win_cap: int, sink, out, ws=None,
                        *, stream=None):
    """ds4a_hca_attend over an FP8 / BF16 pool: uint8 [B, >=N_c, row_bytes]."""
    _bf16(q, "q")
    B, T_q = q_pos.shape
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().ds4a_hca_attend_fp8(ctypes.byref(cfg), B, T_q, _ptr(q_pos), _ptr(q), _ptr(q_norm_g), _ptr(pool),
                                   0 if pool is None else pool.shape[1], N_c, _ptr(win), win_cap,
                                   0 if win is None else win.stride(0), _ptr(sink), _ptr(out), _ptr(ws), ws_bytes,
                                   _stream(stream))
    _ok(rc, "ds4a_hca_attend_fp8")


def append_job(ca, za, bias_a, state, pool, *, cb=None, zb=None, bias_b=None, norm_g=None, fmt: int = 0,
               scales=None) -> AppendJob:
    """One job of ds4a_compress_append_jobs (pool: bf16 [B, N_cap, c], or the
    block-scaled uint8 rows of fmt)."""
    _bf16(ca, "ca"), _bf16(za, "za"), _bf16(cb, "cb"), _bf16(zb, "zb")
    bstride = pool.stride(0) if fmt == 0 else pool.shape[1]
    return AppendJob(ca.shape[1], fmt, _ptr(ca), _ptr(cb), _ptr(za), _ptr(zb), _ptr(bias_a), _ptr(bias_b),
                     _ptr(norm_g), _ptr(state), _ptr(pool), _ptr(scales), bstride)


def ds4a_compress_append_jobs(cfg: LayerCfg, pos, N_cap: int, jobs, *, stream=None):
    """Up to two compressors of one layer, one decode step, one launch when both are CSA-shaped."""
    arr = (AppendJob * len(jobs))(*jobs)
    rc = lib().ds4a_compress_append_jobs(ctypes.byref(cfg), pos.shape[0], _ptr(pos), N_cap, arr, len(jobs),
                                         _stream(stream))
    _ok(rc, "ds4a_compress_append_jobs")


def ds4a_index_topk_workspace(cfg: LayerCfg, B: int, T_q: int, N_c: int) -> int:
    return lib().ds4a_index_topk_workspace(ctypes.byref(cfg), B, T_q, N_c)


def ds4a_index_topk(cfg: LayerCfg, q_pos, q_idx, w_idx, k_idx, N_c: int, idx_out, ws, *,
                    score_out=None, stream=None):
    """q_idx [B,T_q,H_I,D_I], w_idx [B,T_q,H_I], k_idx [B,>=N_c,D_I] ->
    idx_out int32 [B,T_q,k] (ascending, -1 padded)."""
    _bf16(q_idx, "q_idx"), _bf16(w_idx, "w_idx")
    B, T_q = q_pos.shape
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().ds4a_index_topk(ctypes.byref(cfg), B, T_q, _ptr(q_pos), _ptr(q_idx), _ptr(w_idx),
                               _ptr(k_idx), 0 if k_idx is None else k_idx.stride(0), N_c,
                               _ptr(idx_out), _ptr(score_out), _ptr(ws), ws_bytes, _stream(stream))
    _ok(rc, "ds4a_index_topk")


def ds4a_index_topk_noalloc(cfg: LayerCfg, q_pos, q_idx, w_idx, k_idx, N_c: int, idx_out, *,
                            score_out=None, stream=None):
    """ds4a_index_topk without a workspace argument: the library's own
    fixed device scratch (up to 2**21 scores) serves every call, for
    callers that cannot allocate device memory."""
    _bf16(q_idx, "q_idx"), _bf16(w_idx, "w_idx")
    B, T_q = q_pos.shape
    rc = lib().ds4a_index_topk_noalloc(ctypes.byref(cfg), B, T_q, _ptr(q_pos), _ptr(q_idx), _ptr(w_idx),
                                       _ptr(k_idx), 0 if k_idx is None else k_idx.stride(0), N_c,
                                       _ptr(idx_out), _ptr(score_out), _stream(stream))
    _ok(rc, "ds4a_index_topk_noalloc")


def ds4a_attend_workspace(cfg: LayerCfg, B: int, T_q: int, N_c: int, sparse: bool) -> int:
    return lib().ds4a_attend_workspace(ctypes.byref(cfg), B, T_q, N_c, int(bool(sparse)))


def ds4a_sparse_attend(cfg: LayerCfg, q_pos, q, q_norm_g, pool, N_c: int, idx, win, win_cap: int,
                       sink, out, ws=None, *, stream=None):
    _bf16(q, "q")
    B, T_q = q_pos.shape
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().ds4a_sparse_attend(ctypes.byref(cfg), B, T_q, _ptr(q_pos), _ptr(q), _ptr(q_norm_g),
                                  _ptr(pool), 0 if pool is None else pool.stride(0), N_c, _ptr(idx),
                                  _ptr(win), win_cap, 0 if win is None else win.stride(0), _ptr(sink),
                                  _ptr(out), _ptr(ws), ws_bytes, _stream(stream))
    _ok(rc, "ds4a_sparse_attend")


def ds4a_hca_attend(cfg: LayerCfg, q_pos, q, q_norm_g, pool, N_c: int, win, win_cap: int, sink, out,
                    ws=None, *, stream=None):
    _bf16(q, "q")
    B, T_q = q_pos.shape
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().ds4a_hca_attend(ctypes.byref(cfg), B, T_q, _ptr(q_pos), _ptr(q), _ptr(q_norm_g),
                               _ptr(pool), 0 if pool is None else pool.stride(0), N_c, _ptr(win),
                               win_cap, 0 if win is None else win.stride(0), _ptr(sink), _ptr(out),
                               _ptr(ws), ws_bytes, _stream(stream))
    _ok(rc, "ds4a_hca_attend")


def ds4a_out_proj_workspace(cfg: OprojCfg, M: int) -> int:
    return lib().ds4a_out_proj_workspace(ctypes.byref(cfg), M)


def ds4a_out_proj(cfg: OprojCfg, o, w_a, w_b, mid, y, ws=None, *, stream=None):
    """o [M, H, D] -> mid [M, g*r] and y [M, hidden] (grouped projection)."""
    _bf16(o, "o"), _bf16(w_a, "w_a"), _bf16(w_b, "w_b")
    M = o.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = lib().ds4a_out_proj(ctypes.byref(cfg), M, _ptr(o), _ptr(w_a), _ptr(w_b), _ptr(mid), _ptr(y), _ptr(ws),
                             ws_bytes, _stream(stream))
    _ok(rc, "ds4a_out_proj")


def ds4a_check(stream=None) -> tuple[int, int]:
    """Synchronise and read/clear the device error word -> (code, bits)."""
    bits = ctypes.c_uint32(0)
    rc = lib().ds4a_check(_stream(stream), ctypes.byref(bits))
    return rc, bits.value


def ds4a_selftest_wait_timeout(limit_cycles: int, status_out, *, stream=None):
    """One block waits on a barrier nothing arrives at, with a bound of
    limit_cycles SM cycles; status_out (int32 device tensor) gets 2 when the
    bound ran out.  ds4a_check then reports DS4A_ETIMEOUT."""
    rc = lib().ds4a_selftest_wait_timeout(int(limit_cycles), _ptr(status_out), _stream(stream))
    _ok(rc, "ds4a_selftest_wait_timeout")


def ds4a_trace_enable(on: bool = True):
    lib().ds4a_trace_enable(int(bool(on)))


def ds4a_trace_read(cap: int = 65536) -> list[tuple[str, float]]:
    names = (ctypes.c_char_p * cap)()
    ms = (ctypes.c_float * cap)()
    n = lib().ds4a_trace_read(names, ms, cap)
    if n < 0:
        raise Ds4aError(-n, "ds4a_trace_read")
    return [(names[i].decode(), ms[i]) for i in range(min(n, cap))]
