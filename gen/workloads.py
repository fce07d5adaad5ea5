"""The five synthetic workloads and their tensor recipes.

Shapes follow the Flash-0731 attention sizes printed in "DeepSeek V4 Inside:
One Token Through Every Block" (config JSON and the toy-vs-Flash knob table)
and the toy width of the same page.  Every tensor is named; its numbers come
from ``gen.host`` (numpy) or ``gen.device`` (CUDA) under the same recipe.

Value distributions:
* activations / projected tensors / caches: N(0, 1) approximation;
* toy projection weights: N(0, 1/fan_in);
* compressor position biases B^a, B^b: N(0, 1/m), float32;
* RMSNorm gains: 1 + 0.1 N(0, 1), float32;
* attention sinks: N(0, 1), float32.
Seeds: workload id -> 20260000 + id.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

from . import host


@dataclasses.dataclass(frozen=True)
class LayerCfg:
    n_heads: int
    head_dim: int
    rope_dim: int
    window: int
    idx_heads: int
    idx_dim: int
    topk: int
    ratio: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-6

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


@dataclasses.dataclass(frozen=True)
class Spec:
    shape: tuple
    dtype: str  # "bf16" | "f32"
    scale: float | None = None
    offset: float | None = None


@dataclasses.dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    kind: str  # "toy" | "csa_decode" | "hca_decode" | "csa_prefill" | "mix_decode" | "schedule_decode"
    B: int
    pos: int  # decode: position of the query token; prefill: T - 1
    csa: LayerCfg | None
    hca: LayerCfg | None
    n_csa: int  # compressed entries in the CSA pool
    n_hca: int
    n_layers: int = 0  # schedule_decode: layers of the Flash schedule
    storage: str = "bf16"  # "mx": FP8 / BF16 K=V pools and FP4 indexer keys

    @property
    def seed(self) -> int:
        return 20260000 + self.wid


def layer_ratio(layer: int) -> int:
    """Compression ratio of a Flash layer ("Phase 1 Module 1", section on the
    per-layer pattern; "DeepSeek V4 Inside", compress_ratios of the config):
    layers 0 and 1 keep only the sliding window (0), then even layers are
    CSA (4) and odd layers HCA (128)."""
    if layer < 2:
        return 0
    return 4 if layer % 2 == 0 else 128


def schedule_layers(w: Workload) -> list[tuple[str, str]]:
    """(tensor-name prefix, kind) of every layer of a schedule workload, kind
    in "swa" | "csa" | "hca"."""
    kinds = {0: "swa", 4: "csa", 128: "hca"}
    return [(f"L{l:02d}.", kinds[layer_ratio(l)]) for l in range(w.n_layers)]


FLASH_CSA = LayerCfg(n_heads=64, head_dim=512, rope_dim=64, window=128,
                     idx_heads=64, idx_dim=128, topk=512, ratio=4)
FLASH_HCA = dataclasses.replace(FLASH_CSA, ratio=128)
TOY_CSA = LayerCfg(n_heads=2, head_dim=8, rope_dim=2, window=4,
                   idx_heads=2, idx_dim=4, topk=4, ratio=2)
TOY_HIDDEN = 16
TOY_T = 64

WORKLOADS = {
    1: Workload(1, "toy_csa_prefill_t64", "toy", 1, TOY_T - 1, TOY_CSA, None, TOY_T // 2, 0),
    2: Workload(2, "csa_decode_b1_ctx8k", "csa_decode", 1, 8191, FLASH_CSA, None, 2048, 0),
    3: Workload(3, "hca_decode_b32_ctx128k", "hca_decode", 32, 131071, None, FLASH_HCA, 0, 1024),
    4: Workload(4, "csa_prefill_b1_t16k", "csa_prefill", 1, 16383, FLASH_CSA, None, 4096, 0),
    5: Workload(5, "mix_decode_b8_ctx1m", "mix_decode", 8, 1048575, FLASH_CSA, FLASH_HCA, 262144, 8192),
    # a 4096-token prefill, small enough for multi-pass profiler captures
    6: Workload(6, "csa_prefill_b1_t4k", "csa_prefill", 1, 4095, FLASH_CSA, None, 1024, 0),
    # one decode step through the 43 attention layers of the Flash schedule
    7: Workload(7, "schedule43_decode_b8_ctx128k", "schedule_decode", 8, 131071, FLASH_CSA, FLASH_HCA,
                32768, 1024, n_layers=43),
    # the same schedule at a size the oracle checks layer by layer quickly
    8: Workload(8, "schedule43_decode_b2_ctx16k", "schedule_decode", 2, 16383, FLASH_CSA, FLASH_HCA,
                4096, 128, n_layers=43),
    # grouped output projection of a Flash layer (64 heads x 512 in 8 groups,
    # rank 1024, hidden 4096) for a decode batch and for a prefill
    9: Workload(9, "outproj_decode_b8", "out_proj", 8, 0, FLASH_CSA, None, 0, 0),
    10: Workload(10, "outproj_prefill_t16k", "out_proj", 16384, 0, FLASH_CSA, None, 0, 0),
    # the 1M mix with block-scaled caches: FP8 K=V pools (RoPE dims BF16) and
    # FP4 indexer keys; the same generated values, quantised on the device
    11: Workload(11, "mix_decode_b8_ctx1m_mx", "mix_decode", 8, 1048575, FLASH_CSA, FLASH_HCA, 262144, 8192,
                 storage="mx"),
    # the mix at a 128K context: a few hundred MB on the device, still far
    # above L2 -- the size for multi-pass profiler captures (not bench lines)
    12: Workload(12, "mix_decode_b8_ctx128k", "mix_decode", 8, 131071, FLASH_CSA, FLASH_HCA, 32768, 1024),
    13: Workload(13, "mix_decode_b8_ctx128k_mx", "mix_decode", 8, 131071, FLASH_CSA, FLASH_HCA, 32768, 1024,
                 storage="mx"),
}

# Flash grouped output projection: groups of heads, rank per group, hidden
OPROJ_GROUPS, OPROJ_RANK, OPROJ_HIDDEN = 8, 1024, 4096


def _gain(shape):
    return Spec(shape, "f32", 0.1, 1.0)


def _csa_decode_specs(s: dict, pre: str, B: int, c: LayerCfg, n_csa: int):
    m = c.ratio
    s[pre + "csa.q"] = Spec((B, 1, c.n_heads, c.head_dim), "bf16")
    s[pre + "csa.q_norm_g"] = _gain((c.head_dim,))
    s[pre + "csa.sink"] = Spec((c.n_heads,), "f32")
    s[pre + "csa.qi"] = Spec((B, 1, c.idx_heads, c.idx_dim), "bf16")
    s[pre + "csa.wi"] = Spec((B, 1, c.idx_heads), "bf16")
    s[pre + "csa.ki"] = Spec((B, n_csa, c.idx_dim), "bf16")
    s[pre + "csa.pool"] = Spec((B, n_csa, c.head_dim), "bf16")
    s[pre + "csa.win"] = Spec((B, c.window, c.head_dim), "bf16")
    # compressor streams of the 2m newest tokens (the entry that closes now)
    for st in ("ca", "cb", "za", "zb"):
        s[pre + f"csa.kv_{st}"] = Spec((B, 2 * m, c.head_dim), "bf16")
        s[pre + f"csa.ix_{st}"] = Spec((B, 2 * m, c.idx_dim), "bf16")
    s[pre + "csa.kv_ba"] = Spec((m, c.head_dim), "f32", 1.0 / math.sqrt(m))
    s[pre + "csa.kv_bb"] = Spec((m, c.head_dim), "f32", 1.0 / math.sqrt(m))
    s[pre + "csa.ix_ba"] = Spec((m, c.idx_dim), "f32", 1.0 / math.sqrt(m))
    s[pre + "csa.ix_bb"] = Spec((m, c.idx_dim), "f32", 1.0 / math.sqrt(m))
    s[pre + "csa.kv_g"] = _gain((c.head_dim,))


def _hca_decode_specs(s: dict, pre: str, B: int, h: LayerCfg, n_hca: int):
    m = h.ratio
    s[pre + "hca.q"] = Spec((B, 1, h.n_heads, h.head_dim), "bf16")
    s[pre + "hca.q_norm_g"] = _gain((h.head_dim,))
    s[pre + "hca.sink"] = Spec((h.n_heads,), "f32")
    s[pre + "hca.pool"] = Spec((B, n_hca, h.head_dim), "bf16")
    s[pre + "hca.win"] = Spec((B, h.window, h.head_dim), "bf16")
    s[pre + "hca.kv_c"] = Spec((B, m, h.head_dim), "bf16")
    s[pre + "hca.kv_z"] = Spec((B, m, h.head_dim), "bf16")
    s[pre + "hca.kv_b"] = Spec((m, h.head_dim), "f32", 1.0 / math.sqrt(m))
    s[pre + "hca.kv_g"] = _gain((h.head_dim,))


def _swa_decode_specs(s: dict, pre: str, B: int, h: LayerCfg):
    s[pre + "swa.q"] = Spec((B, 1, h.n_heads, h.head_dim), "bf16")
    s[pre + "swa.q_norm_g"] = _gain((h.head_dim,))
    s[pre + "swa.sink"] = Spec((h.n_heads,), "f32")
    s[pre + "swa.win"] = Spec((B, h.window, h.head_dim), "bf16")


def specs(w: Workload) -> dict[str, Spec]:
    """Name -> recipe of every generated tensor of a Flash-shape workload.
    (The toy is built by ``toy_inputs`` from a hidden state and weights.)"""
    s: dict[str, Spec] = {}
    B = w.B
    if w.kind in ("csa_decode", "mix_decode"):
        _csa_decode_specs(s, "", B, w.csa, w.n_csa)
    if w.kind in ("hca_decode", "mix_decode"):
        _hca_decode_specs(s, "", B, w.hca, w.n_hca)
    if w.kind == "out_proj":
        c = w.csa
        k1 = (c.n_heads // OPROJ_GROUPS) * c.head_dim
        s["op.o"] = Spec((B, c.n_heads, c.head_dim), "bf16")
        s["op.w_a"] = Spec((OPROJ_GROUPS, OPROJ_RANK, k1), "bf16", 1.0 / math.sqrt(k1))
        s["op.w_b"] = Spec((OPROJ_HIDDEN, OPROJ_GROUPS * OPROJ_RANK), "bf16",
                           1.0 / math.sqrt(OPROJ_GROUPS * OPROJ_RANK))
    if w.kind == "schedule_decode":
        for pre, kind in schedule_layers(w):
            if kind == "csa":
                _csa_decode_specs(s, pre, B, w.csa, w.n_csa)
            elif kind == "hca":
                _hca_decode_specs(s, pre, B, w.hca, w.n_hca)
            else:
                _swa_decode_specs(s, pre, B, w.hca)
    if w.kind == "csa_prefill":
        c = w.csa
        m = c.ratio
        T = w.pos + 1
        for st in ("ca", "cb", "za", "zb"):
            s[f"csa.kv_{st}"] = Spec((B, T, c.head_dim), "bf16")
            s[f"csa.ix_{st}"] = Spec((B, T, c.idx_dim), "bf16")
        s["csa.kv_ba"] = Spec((m, c.head_dim), "f32", 1.0 / math.sqrt(m))
        s["csa.kv_bb"] = Spec((m, c.head_dim), "f32", 1.0 / math.sqrt(m))
        s["csa.ix_ba"] = Spec((m, c.idx_dim), "f32", 1.0 / math.sqrt(m))
        s["csa.ix_bb"] = Spec((m, c.idx_dim), "f32", 1.0 / math.sqrt(m))
        s["csa.kv_g"] = _gain((c.head_dim,))
        s["csa.q"] = Spec((B, T, c.n_heads, c.head_dim), "bf16")
        s["csa.q_norm_g"] = _gain((c.head_dim,))
        s["csa.sink"] = Spec((c.n_heads,), "f32")
        s["csa.qi"] = Spec((B, T, c.idx_heads, c.idx_dim), "bf16")
        s["csa.wi"] = Spec((B, T, c.idx_heads), "bf16")
        s["csa.win"] = Spec((B, T, c.head_dim), "bf16")  # raw K=V of every token
    return s


def host_tensor(w: Workload, name: str, spec: Spec | None = None) -> np.ndarray:
    spec = spec or specs(w)[name]
    if spec.dtype == "bf16":
        return host.normal_bf16(w.seed, name, spec.shape, spec.scale, spec.offset)
    return host.normal_f32(w.seed, name, spec.shape, spec.scale, spec.offset)


def host_rows(w: Workload, name: str, rows: np.ndarray, spec: Spec | None = None) -> np.ndarray:
    """Random access to whole innermost rows of a bf16 tensor: rows are flat
    row numbers over the leading dimensions; returns uint16 [len(rows), last]."""
    spec = spec or specs(w)[name]
    last = spec.shape[-1]
    rows = np.asarray(rows, dtype=np.int64).ravel()
    flat = rows[:, None] * last + np.arange(last, dtype=np.int64)[None, :]
    return host.normal_bf16_at(w.seed, name, flat, spec.scale, spec.offset)


def query_positions(w: Workload) -> np.ndarray:
    """int32 [B, T_q] absolute positions of the queries."""
    if w.kind in ("toy", "csa_prefill"):
        T = w.pos + 1
        return np.tile(np.arange(T, dtype=np.int32), (w.B, 1))
    return np.full((w.B, 1), w.pos, dtype=np.int32)


def toy_inputs(w: Workload | None = None) -> dict[str, np.ndarray]:
    """Toy CSA layer (hidden 16, 2 heads x 8, m=2, indexer 2 x 4, k=4, W=4,
    T=64).  Hidden states are N(0,1) float32, weights N(0, 1/fan_in); every
    projected tensor is H @ W in float64, rounded to float32 and then to
    bfloat16 (round-to-nearest-even)."""
    w = w or WORKLOADS[1]
    c = w.csa
    sd = w.seed
    T, d = TOY_T, TOY_HIDDEN
    H = host.normal_f32(sd, "toy.hidden", (T, d)).astype(np.float64)

    def proj(name, n_out):
        W = host.normal_f32(sd, f"toy.W_{name}", (d, n_out), 1.0 / math.sqrt(d)).astype(np.float64)
        return host.f32_to_bf16_bits((H @ W).astype(np.float32))

    out: dict[str, np.ndarray] = {}
    out["csa.q"] = proj("q", c.n_heads * c.head_dim).reshape(1, T, c.n_heads, c.head_dim)
    out["csa.qi"] = proj("qi", c.idx_heads * c.idx_dim).reshape(1, T, c.idx_heads, c.idx_dim)
    out["csa.wi"] = proj("wi", c.idx_heads).reshape(1, T, c.idx_heads)
    out["csa.win"] = proj("kv", c.head_dim).reshape(1, T, c.head_dim)
    for st in ("ca", "cb", "za", "zb"):
        out[f"csa.kv_{st}"] = proj(f"kv_{st}", c.head_dim).reshape(1, T, c.head_dim)
        out[f"csa.ix_{st}"] = proj(f"ix_{st}", c.idx_dim).reshape(1, T, c.idx_dim)
    m = c.ratio
    out["csa.kv_ba"] = host.normal_f32(sd, "csa.kv_ba", (m, c.head_dim), 1.0 / math.sqrt(m))
    out["csa.kv_bb"] = host.normal_f32(sd, "csa.kv_bb", (m, c.head_dim), 1.0 / math.sqrt(m))
    out["csa.ix_ba"] = host.normal_f32(sd, "csa.ix_ba", (m, c.idx_dim), 1.0 / math.sqrt(m))
    out["csa.ix_bb"] = host.normal_f32(sd, "csa.ix_bb", (m, c.idx_dim), 1.0 / math.sqrt(m))
    out["csa.kv_g"] = host.normal_f32(sd, "csa.kv_g", (c.head_dim,), 0.1, 1.0)
    out["csa.q_norm_g"] = host.normal_f32(sd, "csa.q_norm_g", (c.head_dim,), 0.1, 1.0)
    out["csa.sink"] = host.normal_f32(sd, "csa.sink", (c.n_heads,))
    return out
