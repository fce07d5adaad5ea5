"""Planted mistakes: each mutant is a copy of the oracle source with one
plausible error; at least one pin must reject every mutant."""
import importlib.util
import os
import types

import pytest

from pins import PINS

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "ds4a_oracle.py")

# name -> list of (old, new) source replacements (each old must occur once,
# unless the name ends in "*": then every occurrence is replaced)
MUTANTS = {
    "sink dropped from denominator": [("den = e.sum(axis=1, keepdims=True) + es", "den = e.sum(axis=1, keepdims=True)")],
    "no output de-rotation": [("return rope(o, -pos, rope_dim, rope_base)", "return o")],
    "de-rotation with +pos": [("return rope(o, -pos, rope_dim, rope_base)", "return rope(o, pos, rope_dim, rope_base)")],
    "rope angle sign": [("ang = np.asarray(pos, dtype=np.float64)[..., None]", "ang = -np.asarray(pos, dtype=np.float64)[..., None]")],
    "rope half-split pairs*": [("D - rope_dim::2]", "D - rope_dim:D - rope_dim // 2]"),
                               ("D - rope_dim + 1::2]", "D - rope_dim // 2:]")],
    "rope non-rotation": [("x[..., D - rope_dim::2] = xe * c - xo * s", "x[..., D - rope_dim::2] = xe * c + xo * s")],
    "visibility off by one": [("return (int(pos) + 1) // int(m)", "return int(pos) // int(m)")],
    "window off by one": [("np.arange(max(0, int(pos) - window + 1), int(pos) + 1,", "np.arange(max(0, int(pos) - window), int(pos),")],
    "missing ReLU": [("return np.maximum(dots, 0.0) @ wi", "return dots @ wi")],
    "ReLU after head sum": [("return np.maximum(dots, 0.0) @ wi", "return np.maximum(dots @ wi, 0.0)")],
    "top-k keeps lowest": [("order = np.lexsort((np.arange(n), -scores))", "order = np.lexsort((np.arange(n), scores))")],
    "ties to higher index": [("order = np.lexsort((np.arange(n), -scores))", "order = np.lexsort((-np.arange(n), -scores))")],
    "scale 1/D": [("z = (qh @ rows.T) * head_dim_scale", "z = (qh @ rows.T) * head_dim_scale ** 2")],
    "query not normalised": [("qh = rope(rms_norm(q, widen(q_norm_g), eps), pos, rope_dim, rope_base)",
                              "qh = rope(q * widen(q_norm_g), pos, rope_dim, rope_base)")],
    "query not rotated": [("qh = rope(rms_norm(q, widen(q_norm_g), eps), pos, rope_dim, rope_base)",
                           "qh = rms_norm(q, widen(q_norm_g), eps)")],
    "rmsnorm without eps": [("return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)",
                             "return x / np.sqrt(ms) * np.asarray(g, dtype=np.float64)")],
    "rmsnorm without gain": [("return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)",
                              "return x / np.sqrt(ms + eps)")],
    "overlap forward": [("t = (i - 1) * m + r - tok_begin", "t = (i + 1) * m + r - tok_begin")],
    "softmax over channels": [("wgt = e / e.sum(axis=0, keepdims=True)", "wgt = e / e.sum(axis=1, keepdims=True)")],
    "biases swapped": [("logits.append(za[t] + ba[r])", "logits.append(za[t] + (bb[r] if bb is not None else ba[r]))")],
    "entry position (i+1)m-1": [("e = rope(e, i * m, rope_dim, rope_base)", "e = rope(e, (i + 1) * m - 1, rope_dim, rope_base)")],
    "HCA ignores visibility": [('"""HCA: keys = every visible pool entry followed by the window."""\n    n_vis = min(visible_entries(pos, cfg.ratio), n_c)',
                                '"""HCA: keys = every visible pool entry followed by the window."""\n    n_vis = n_c')],
    "window ring slot": [("return widen(win)[window_positions(pos, window) % win_cap]",
                          "return widen(win)[window_positions(pos, window) % win.shape[0] if False else window_positions(pos, window) - window_positions(pos, window)[0]]")],
    "rope exponent -j/R": [("return base ** (-2.0 * j / rope_dim)", "return base ** (-1.0 * j / rope_dim)")],
    "store_bf16 truncates": [("return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)",
                              "return (b >> np.uint32(16)).astype(np.uint16)")],
    "store_bf16 ties away from zero": [("return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)",
                                        "return ((b + np.uint32(0x8000)) >> np.uint32(16)).astype(np.uint16)")],
    "out_proj heads strided across groups": [("x = o.reshape(M, n_groups, -1)  # [M, g, (H/g) D], heads in order",
                                              "x = o.reshape(M, -1, n_groups).transpose(0, 2, 1)")],
    "out_proj weight transposed per group": [("np.concatenate([x[:, j] @ wa[j].T for j in range(n_groups)], axis=1)",
                                              "np.concatenate([x[:, j] @ wa[j].reshape(-1, wa.shape[1]) for j in range(n_groups)], axis=1)")],
    "out_proj second product unrounded": [("y = widen(store_bf16(mid)) @ widen(w_b).T", "y = mid @ widen(w_b).T")],
    "mx rounding ties away from zero": [("code = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))",
                                         "code = np.where(dlo < dhi, lo, hi)")],
    "mx scale floor rule (clips)": [("shared = np.clip(k - j + (f > g), -127, 127)", "shared = np.clip(k - j, -127, 127)")],
    "fp4 nibbles swapped": [("packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)",
                             "packed = (codes[..., 1::2] | (codes[..., 0::2] << 4)).astype(np.uint8)")],
    "fp8 rope dims quantised too": [("out[..., n:n + 2 * R] = np.ascontiguousarray(bits[..., n:]).view(np.uint8).reshape(bits.shape[:-1] + (2 * R,))",
                                     "out[..., n:n + 2 * R] = np.ascontiguousarray(store_bf16(np.round(widen(bits[..., n:])))).view(np.uint8).reshape(bits.shape[:-1] + (2 * R,))")],
    "e4m3 subnormal exponent off by one": [("out.append(m / (1 << f[\"mbits\"]) * 2.0 ** (1 - f[\"bias\"]))",
                                            "out.append(m / (1 << f[\"mbits\"]) * 2.0 ** (0 - f[\"bias\"]))")],
    "mx drops the sign of zero": [("return (code + np.where(np.signbit(x), sign_bit, 0)).astype(np.uint8)",
                                   "return (code + np.where(np.signbit(x) & (code > 0), sign_bit, 0)).astype(np.uint8)")],
    "pool row ignores idx": [("rows = np.concatenate([widen(pool)[sel], window_rows",
                              "rows = np.concatenate([widen(pool)[: sel.size], window_rows")],
}


def _load(name, edits, replace_all):
    src = open(SRC).read()
    for old, new in edits:
        n = src.count(old)
        assert n >= 1, f"mutant {name!r}: {old!r} not found"
        if not replace_all:
            assert n == 1, f"mutant {name!r}: {old!r} found {n} times"
        src = src.replace(old, new)
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    exec(compile(src, SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = _load(name, MUTANTS[name], name.endswith("*"))
    failed = []
    for pin in PINS:
        try:
            pin(mod)
        except Exception as e:  # AssertionError or a crash both reject it
            failed.append(pin.__name__)
    assert failed, f"no pin rejects the mutant {name!r}"
