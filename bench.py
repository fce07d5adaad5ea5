#!/usr/bin/env python
"""Benchmark of the ds4a hot path (DeepSeek-V4 hybrid CSA/HCA attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workloads 5,2,3,4,7]
                    [--impl ours|reference]

One "step" is one pass of the whole path over one batch of the workload:
  csa_decode  compress the entry that closes at the query's position (KV and
              indexer keys), index top-k over every visible entry, sparse
              attention with the window;
  hca_decode  compress the closing HCA entry, attend every visible entry and
              the window;
  csa_prefill compress every entry (KV and indexer keys), index top-k for all
              16384 queries, sparse attention for all of them;
  mix_decode  one CSA decode layer and one HCA decode layer;
  schedule_decode  one decode step through the 43 attention layers of the
              Flash schedule (two window-only layers, then CSA and HCA
              alternating).
Decode layers keep the compressor's cache (ds4a_compress_append): a step
appends the query token's C/Z rows and compresses the entry it closes.
The first workload listed is the headline line; the others are reported in
``workloads``.  Inputs are seeded synthetic tensors (gen/), resident in HBM.
Timing: W warm-up steps, then K steps, each bracketed by CUDA events on the
launch stream, with a 256 MiB write between steps (outside the events) so
that every step starts from a cold L2; a barrier and a synchronise bracket
the region; the time is the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CSA/HCA attention tokens/s (decode & prefill) at 1 B200; % of HBM/TC roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA datasheet figures for one B200 (dense bf16), reported beside the
# measured peaks
DATASHEET_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------------------
# workload state and the step
# ---------------------------------------------------------------------------
class Layer:
    """Device tensors and outputs of one attention layer of a workload."""


def _ring_state(ly, names, cap, dev):
    """The compressor cache of a decode layer: the streams' rows of the tokens
    before the query's (positions pos - len + 1 .. pos - 1) in their ring
    slots (position mod cap), and the query token's own rows as the step's
    new input ("<name>_new", [B, c])."""
    import torch

    first = ly.t[names[0]]
    B, n_rows, c = first.shape
    state = torch.zeros((B, len(names), cap, c), dtype=torch.bfloat16, device=dev)
    tb = ly.pos - n_rows + 1
    for si, nm in enumerate(names):
        for j in range(n_rows - 1):
            state[:, si, (tb + j) % cap] = ly.t[nm][:, j]
        ly.t[nm + "_new"] = ly.t[nm][:, n_rows - 1].contiguous()
    return state


def _csa_decode_layer(w, B, pos, n_c, dev, T, pre=""):
    import torch
    import long_context_hybrid_kv_b200 as L

    c = w.csa
    key = pre + "csa."
    ly = Layer()
    ly.kind, ly.cfg_py, ly.cfg, ly.prefix = "csa", c, L.layer_cfg(c), pre
    ly.t = {n[len(key):]: T[n] for n in T if n.startswith(key)}
    ly.B, ly.pos, ly.n_c, ly.m = B, pos, n_c, c.ratio
    ly.q_pos = torch.full((B, 1), pos, dtype=torch.int32, device=dev)
    ly.idx = torch.empty((B, 1, c.topk), dtype=torch.int32, device=dev)
    ly.out = torch.empty((B, 1, c.n_heads, c.head_dim), dtype=torch.bfloat16, device=dev)
    ly.ws_index = torch.empty(max(1, L.ds4a_index_topk_workspace(ly.cfg, B, 1, n_c) // 4),
                              dtype=torch.float32, device=dev)
    ly.ws_att = torch.empty(max(1, L.ds4a_attend_workspace(ly.cfg, B, 1, n_c, True) // 4),
                            dtype=torch.float32, device=dev)
    ly.entry = (pos + 1) // c.ratio - 1  # the entry that closes at this token
    ly.state_kv = _ring_state(ly, ["kv_ca", "kv_cb", "kv_za", "kv_zb"], 2 * c.ratio, dev)
    ly.state_ix = _ring_state(ly, ["ix_ca", "ix_cb", "ix_za", "ix_zb"], 2 * c.ratio, dev)
    ly.mx = w.storage == "mx"
    if ly.mx:
        # block-scaled caches made by the library's quantisers from the
        # generated bf16 pools, which are then dropped
        rb = L.ds4a_kv_fp8_row_bytes(c.head_dim, c.rope_dim)
        ly.kv8 = torch.empty((B, n_c, rb), dtype=torch.uint8, device=dev)
        L.ds4a_quantize_kv_fp8(ly.t["pool"].reshape(B * n_c, -1), c.rope_dim, ly.kv8.view(B * n_c, rb))
        ly.ki4 = torch.empty((B, n_c, c.idx_dim // 2), dtype=torch.uint8, device=dev)
        ly.ki4s = torch.empty((B, n_c, c.idx_dim // 32), dtype=torch.uint8, device=dev)
        L.ds4a_quantize_idx_fp4(ly.t["ki"].reshape(B * n_c, -1), ly.ki4.view(B * n_c, -1), ly.ki4s.view(B * n_c, -1))
        torch.cuda.synchronize()
        del ly.t["pool"], ly.t["ki"]
    _csa_jobs(ly)
    ly.step_inputs = ["q", "qi", "wi", "kv_ca_new", "kv_cb_new", "kv_za_new", "kv_zb_new", "ix_ca_new",
                      "ix_cb_new", "ix_za_new", "ix_zb_new"]
    return ly


def _csa_jobs(ly):
    """The two compressor jobs of a CSA decode layer (K=V entries and indexer
    keys), rebuilt whenever the step's input tensors move."""
    import long_context_hybrid_kv_b200 as L

    t = ly.t
    if ly.mx:
        kv = L.append_job(t["kv_ca_new"], t["kv_za_new"], t["kv_ba"], ly.state_kv, ly.kv8, cb=t["kv_cb_new"],
                          zb=t["kv_zb_new"], bias_b=t["kv_bb"], norm_g=t["kv_g"], fmt=L.DS4A_MX_KV_FP8)
        ix = L.append_job(t["ix_ca_new"], t["ix_za_new"], t["ix_ba"], ly.state_ix, ly.ki4, cb=t["ix_cb_new"],
                          zb=t["ix_zb_new"], bias_b=t["ix_bb"], fmt=L.DS4A_MX_IDX_FP4, scales=ly.ki4s)
    else:
        kv = L.append_job(t["kv_ca_new"], t["kv_za_new"], t["kv_ba"], ly.state_kv, t["pool"], cb=t["kv_cb_new"],
                          zb=t["kv_zb_new"], bias_b=t["kv_bb"], norm_g=t["kv_g"])
        ix = L.append_job(t["ix_ca_new"], t["ix_za_new"], t["ix_ba"], ly.state_ix, t["ki"], cb=t["ix_cb_new"],
                          zb=t["ix_zb_new"], bias_b=t["ix_bb"])
    ly.jobs = [kv, ix]


def _hca_decode_layer(w, B, pos, n_c, dev, T, pre=""):
    import torch
    import long_context_hybrid_kv_b200 as L

    h = w.hca
    key = pre + "hca."
    ly = Layer()
    ly.kind, ly.cfg_py, ly.cfg, ly.prefix = "hca", h, L.layer_cfg(h), pre
    ly.t = {n[len(key):]: T[n] for n in T if n.startswith(key)}
    ly.B, ly.pos, ly.n_c, ly.m = B, pos, n_c, h.ratio
    ly.q_pos = torch.full((B, 1), pos, dtype=torch.int32, device=dev)
    ly.out = torch.empty((B, 1, h.n_heads, h.head_dim), dtype=torch.bfloat16, device=dev)
    ly.ws_att = torch.empty(max(1, L.ds4a_attend_workspace(ly.cfg, B, 1, n_c, False) // 4),
                            dtype=torch.float32, device=dev)
    ly.entry = (pos + 1) // h.ratio - 1
    ly.state_kv = _ring_state(ly, ["kv_c", "kv_z"], h.ratio, dev)
    ly.step_inputs = ["q", "kv_c_new", "kv_z_new"]
    ly.mx = w.storage == "mx"
    if ly.mx:
        rb = L.ds4a_kv_fp8_row_bytes(h.head_dim, h.rope_dim)
        ly.kv8 = torch.empty((B, n_c, rb), dtype=torch.uint8, device=dev)
        L.ds4a_quantize_kv_fp8(ly.t["pool"].reshape(B * n_c, -1), h.rope_dim, ly.kv8.view(B * n_c, rb))
        torch.cuda.synchronize()
        del ly.t["pool"]
    return ly


def _swa_decode_layer(w, B, pos, dev, T, pre):
    """A sliding-window-only layer: attention over the window alone (the HCA
    call with no pool entries)."""
    import torch
    import long_context_hybrid_kv_b200 as L

    h = w.hca
    key = pre + "swa."
    ly = Layer()
    ly.kind, ly.cfg_py, ly.cfg, ly.prefix = "swa", h, L.layer_cfg(h), pre
    ly.t = {n[len(key):]: T[n] for n in T if n.startswith(key)}
    ly.B, ly.pos, ly.n_c, ly.m = B, pos, 0, h.ratio
    ly.q_pos = torch.full((B, 1), pos, dtype=torch.int32, device=dev)
    ly.out = torch.empty((B, 1, h.n_heads, h.head_dim), dtype=torch.bfloat16, device=dev)
    ly.ws_att = torch.empty(max(1, L.ds4a_attend_workspace(ly.cfg, B, 1, 0, False) // 4),
                            dtype=torch.float32, device=dev)
    ly.step_inputs = ["q"]
    return ly


def _csa_prefill_layer(w, dev, T, toy=None):
    import torch
    import long_context_hybrid_kv_b200 as L

    c = w.csa
    ly = Layer()
    ly.kind, ly.cfg_py, ly.cfg = "csa_prefill", c, L.layer_cfg(c)
    ly.t = {n[4:]: T[n] for n in T if n.startswith("csa.")}
    Tn = w.pos + 1
    ly.B, ly.T, ly.m = 1, Tn, c.ratio
    ly.n_c = Tn // c.ratio
    ly.q_pos = torch.arange(Tn, dtype=torch.int32, device=dev).reshape(1, Tn)
    ly.pool = torch.empty((1, ly.n_c, c.head_dim), dtype=torch.bfloat16, device=dev)
    ly.ki = torch.empty((1, ly.n_c, c.idx_dim), dtype=torch.bfloat16, device=dev)
    ly.idx = torch.empty((1, Tn, c.topk), dtype=torch.int32, device=dev)
    ly.out = torch.empty((1, Tn, c.n_heads, c.head_dim), dtype=torch.bfloat16, device=dev)
    ly.ws_index = torch.empty(max(1, L.ds4a_index_topk_workspace(ly.cfg, 1, Tn, ly.n_c) // 4),
                              dtype=torch.float32, device=dev)
    ly.ws_att = torch.empty(max(1, L.ds4a_attend_workspace(ly.cfg, 1, Tn, ly.n_c, True) // 4),
                            dtype=torch.float32, device=dev)
    ly.step_inputs = ["q", "qi", "wi", "win", "kv_ca", "kv_cb", "kv_za", "kv_zb", "ix_ca", "ix_cb",
                      "ix_za", "ix_zb"]
    return ly


def _out_proj_layer(w, dev, T):
    """The grouped output projection of one Flash layer for w.B tokens."""
    import torch
    import long_context_hybrid_kv_b200 as L
    from gen import workloads as W

    c = w.csa
    ly = Layer()
    ly.kind, ly.cfg_py = "out_proj", c
    ly.cfg = L.OprojCfg(c.n_heads, c.head_dim, W.OPROJ_GROUPS, W.OPROJ_RANK, W.OPROJ_HIDDEN)
    ly.t = {n[3:]: T[n] for n in T if n.startswith("op.")}
    ly.B = w.B
    ly.mid = torch.empty((w.B, W.OPROJ_GROUPS * W.OPROJ_RANK), dtype=torch.bfloat16, device=dev)
    ly.out = torch.empty((w.B, W.OPROJ_HIDDEN), dtype=torch.bfloat16, device=dev)
    ly.ws = torch.empty(max(1, L.ds4a_out_proj_workspace(ly.cfg, w.B) // 4), dtype=torch.float32, device=dev)
    ly.step_inputs = ["o"]
    return ly


def _run_layer(ly, stream=None):
    """One layer's calls on `stream` (a CUDA stream handle; None = the
    current stream, looked up by each call)."""
    import long_context_hybrid_kv_b200 as L

    t = ly.t
    S = stream
    if ly.kind == "csa" and ly.mx:
        # the layer's two compressors in one call (one launch)
        L.ds4a_compress_append_jobs(ly.cfg, ly.q_pos.view(-1), ly.n_c, ly.jobs, stream=S)
        L.ds4a_index_topk_fp4(ly.cfg, ly.q_pos, t["qi"], t["wi"], ly.ki4, ly.ki4s, ly.n_c, ly.idx, ly.ws_index,
                              stream=S)
        L.ds4a_sparse_attend_fp8(ly.cfg, ly.q_pos, t["q"], t["q_norm_g"], ly.kv8, ly.n_c, ly.idx, t["win"],
                                 t["win"].shape[1], t["sink"], ly.out, ly.ws_att, stream=S)
    elif ly.kind == "hca" and ly.mx:
        L.ds4a_compress_append_mx(ly.cfg, ly.q_pos.view(-1), t["kv_c_new"], t["kv_z_new"], t["kv_b"], ly.state_kv,
                                  L.DS4A_MX_KV_FP8, ly.kv8, norm_g=t["kv_g"], stream=S)
        L.ds4a_hca_attend_fp8(ly.cfg, ly.q_pos, t["q"], t["q_norm_g"], ly.kv8, ly.n_c, t["win"], t["win"].shape[1],
                              t["sink"], ly.out, ly.ws_att, stream=S)
    elif ly.kind == "csa":
        # the layer's two compressors in one call (one launch)
        L.ds4a_compress_append_jobs(ly.cfg, ly.q_pos.view(-1), ly.n_c, ly.jobs, stream=S)
        L.ds4a_index_topk(ly.cfg, ly.q_pos, t["qi"], t["wi"], t["ki"], ly.n_c, ly.idx, ly.ws_index, stream=S)
        L.ds4a_sparse_attend(ly.cfg, ly.q_pos, t["q"], t["q_norm_g"], t["pool"], ly.n_c, ly.idx, t["win"],
                             t["win"].shape[1], t["sink"], ly.out, ly.ws_att, stream=S)
    elif ly.kind == "hca":
        L.ds4a_compress_append(ly.cfg, ly.q_pos.view(-1), t["kv_c_new"], t["kv_z_new"], t["kv_b"], ly.state_kv,
                               t["pool"], norm_g=t["kv_g"], stream=S)
        L.ds4a_hca_attend(ly.cfg, ly.q_pos, t["q"], t["q_norm_g"], t["pool"], ly.n_c, t["win"],
                          t["win"].shape[1], t["sink"], ly.out, ly.ws_att, stream=S)
    elif ly.kind == "out_proj":
        L.ds4a_out_proj(ly.cfg, t["o"], t["w_a"], t["w_b"], ly.mid, ly.out, ly.ws, stream=S)
    elif ly.kind == "swa":
        L.ds4a_hca_attend(ly.cfg, ly.q_pos, t["q"], t["q_norm_g"], None, 0, t["win"], t["win"].shape[1],
                          t["sink"], ly.out, ly.ws_att, stream=S)
    else:  # prefill
        L.ds4a_compress(ly.cfg, t["kv_ca"], t["kv_za"], t["kv_ba"], ly.pool, cb=t["kv_cb"], zb=t["kv_zb"],
                        bias_b=t["kv_bb"], norm_g=t["kv_g"], entry_begin=0, entry_end=ly.n_c, stream=S)
        L.ds4a_compress(ly.cfg, t["ix_ca"], t["ix_za"], t["ix_ba"], ly.ki, cb=t["ix_cb"], zb=t["ix_zb"],
                        bias_b=t["ix_bb"], entry_begin=0, entry_end=ly.n_c, stream=S)
        L.ds4a_index_topk(ly.cfg, ly.q_pos, t["qi"], t["wi"], ly.ki, ly.n_c, ly.idx, ly.ws_index, stream=S)
        L.ds4a_sparse_attend(ly.cfg, ly.q_pos, t["q"], t["q_norm_g"], ly.pool, ly.n_c, ly.idx, t["win"],
                             ly.T, t["sink"], ly.out, ly.ws_att, stream=S)


class State:
    """A workload's resident inputs, outputs and its step."""

    def __init__(self, wid: int, dev="cuda"):
        import numpy as np
        import torch
        from gen import device as gd
        from gen import workloads as W

        self.w = w = W.WORKLOADS[wid]
        self.wid = wid
        self.layers = []
        if w.kind == "toy":
            x = W.toy_inputs(w)
            T = {}
            for n, a in x.items():
                if a.dtype == np.uint16:
                    T[n] = torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
                else:
                    T[n] = torch.from_numpy(a).to(dev)
            self.layers.append(_csa_prefill_layer(w, dev, T))
            self.tokens = w.pos + 1
        else:
            T = gd.workload_tensors(w, device=dev)
            if w.kind in ("csa_decode", "mix_decode"):
                self.layers.append(_csa_decode_layer(w, w.B, w.pos, w.n_csa, dev, T))
            if w.kind in ("hca_decode", "mix_decode"):
                self.layers.append(_hca_decode_layer(w, w.B, w.pos, w.n_hca, dev, T))
            if w.kind == "csa_prefill":
                self.layers.append(_csa_prefill_layer(w, dev, T))
            if w.kind == "out_proj":
                self.layers.append(_out_proj_layer(w, dev, T))
            if w.kind == "schedule_decode":
                for pre, kind in W.schedule_layers(w):
                    if kind == "csa":
                        self.layers.append(_csa_decode_layer(w, w.B, w.pos, w.n_csa, dev, T, pre))
                    elif kind == "hca":
                        self.layers.append(_hca_decode_layer(w, w.B, w.pos, w.n_hca, dev, T, pre))
                    else:
                        self.layers.append(_swa_decode_layer(w, w.B, w.pos, dev, T, pre))
            self.tokens = w.B if w.kind != "csa_prefill" else w.pos + 1
        self.tensors = T

    def step(self):
        import torch

        s = torch.cuda.current_stream().cuda_stream  # once per step
        for ly in self.layers:
            _run_layer(ly, s)

    # per-step input / output tensors for the end-to-end measurement
    def step_io(self):
        ins = [ly.t[n] for ly in self.layers for n in ly.step_inputs]
        outs = [ly.out for ly in self.layers]
        return ins, outs


# ---------------------------------------------------------------------------
# algorithmic work per kernel launch (for the roofline)
# ---------------------------------------------------------------------------
def kernel_work(state) -> dict:
    """kernel name -> (algorithmic bytes, algorithmic flops) per step, summed
    over the launches of that kernel in one step; the count of launches."""
    from gen import workloads as W

    work: dict[str, list] = {}

    def add(name, nbytes, flops=0.0, launches=1):
        e = work.setdefault(name, [0.0, 0.0, 0])
        e[0] += nbytes
        e[1] += flops
        e[2] += launches

    for ly in state.layers:
        c = ly.cfg_py
        if ly.kind == "out_proj":
            cf = ly.cfg
            M = ly.B
            k1 = (cf.n_heads // cf.n_groups) * cf.head_dim
            n1 = cf.n_groups * cf.group_rank
            nbytes = 2 * (M * cf.n_heads * cf.head_dim + n1 * k1 + cf.hidden * n1 + 2 * M * n1 + M * cf.hidden)
            add("out_proj_gemm", nbytes, 2.0 * M * (n1 * k1 + cf.hidden * n1), launches=2)
            continue
        if ly.kind == "swa":
            B, pos, D, H = ly.B, ly.pos, c.head_dim, c.n_heads
            n_win = pos - max(0, pos - c.window + 1) + 1
            add("attend", B * (n_win * D * 2 + 2 * H * D * 2 + H * 4 + D * 4), 4.0 * B * n_win * H * D)
            continue
        if ly.kind in ("csa", "hca"):
            B, pos, n_c, m = ly.B, ly.pos, ly.n_c, ly.m
            n_vis = min((pos + 1) // m, n_c)
            n_win = pos - max(0, pos - c.window + 1) + 1
            D, H = c.head_dim, c.n_heads
            mx = getattr(ly, "mx", False)
            row = (D - c.rope_dim) + 2 * c.rope_dim + (D - c.rope_dim) // 32 if mx else 2 * D  # bytes per K=V row
            krow = c.idx_dim // 2 + c.idx_dim // 32 if mx else 2 * c.idx_dim  # bytes per indexer key
            # compressor: 2m (CSA) or m (HCA) tokens x (C + Z) + biases + gain, one entry out
            streams = (4 if ly.kind == "csa" else 2) * m
            add("compress", B * (streams * D * 2 + 2 * m * D * 4 + D * 4 + row))
            if ly.kind == "csa":
                add("compress", B * (streams * c.idx_dim * 2 + 2 * m * c.idx_dim * 4 + krow))
                qb = c.idx_heads * c.idx_dim * 2 + c.idx_heads * 2
                add("index_score", B * (n_vis * krow + qb + n_vis * 4),
                    2.0 * B * n_vis * c.idx_heads * c.idx_dim)
                add("topk", B * (n_vis * 4 + c.topk * 4))
                n_keys = min(c.topk, n_vis) + n_win
            else:
                n_keys = n_vis + n_win
            n_pool = n_keys - n_win
            add("attend", B * (n_pool * row + n_win * D * 2 + 2 * H * D * 2 + H * 4 + D * 4),
                4.0 * B * n_keys * H * D)
        else:  # prefill
            Tn, m, D, H = ly.T, ly.m, c.head_dim, c.n_heads
            n_c = ly.n_c
            add("compress", Tn * (4 * D * 2 + 4 * c.idx_dim * 2) + n_c * (D + c.idx_dim) * 2, launches=2)
            pos = list(range(Tn))
            n_vis = [min((p + 1) // m, n_c) for p in pos]
            pairs = sum(n_vis)
            add("index_score", n_c * c.idx_dim * 2 + Tn * (c.idx_heads * (c.idx_dim + 1) * 2) + pairs * 4,
                2.0 * pairs * c.idx_heads * c.idx_dim)
            add("topk", pairs * 4 + Tn * c.topk * 4)
            keys = sum(min(c.topk, nv) + (p - max(0, p - c.window + 1) + 1) for p, nv in zip(pos, n_vis))
            add("attend", keys * D * 2 + Tn * 2 * H * D * 2, 4.0 * keys * H * D)
    return {k: tuple(v) for k, v in work.items()}


def kernel_family(name: str) -> str:
    for fam in ("compress", "index_score", "topk", "attend_combine", "attend", "out_proj_gemm"):
        if name.startswith(fam):
            return fam
    return name


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.proc = None
        self.dev_index = dev_index

    def __enter__(self):
        import torch
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = [r.split(",") for r in (getattr(self, "out", "") or "").strip().splitlines() if r.strip()]
        rows = [[x.strip() for x in r] for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def time_steps(step, K, W, stream, flush, graph=False, barrier=None):
    """Per-step device times (ms) of K steps after W warm-up steps; a 256 MiB
    write between steps (outside the events) empties L2."""
    import torch

    for _ in range(W):
        step()
    run = step
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        run = g.replay
        for _ in range(2):
            run()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    with torch.cuda.stream(stream):
        for e0, e1 in ev:
            flush()
            e0.record(stream)
            run()
            e1.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    del g
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def kernel_times(state, K, stream, flush):
    """Average device time per launch of every library kernel (launch trace,
    CUDA events on the launch stream) over K steps, each queued whole behind
    a spin kernel so that the events time the GPU, not the host."""
    import torch
    import long_context_hybrid_kv_b200 as L

    torch.cuda.synchronize()
    per: dict[str, list] = {}
    n_launch = 0
    with torch.cuda.stream(stream):
        for _ in range(K):
            flush()
            # a ~1 ms spin ahead of the step lets the host queue every launch
            # before the GPU reaches them, so no launch waits on the host
            torch.cuda._sleep(2_000_000)
            L.ds4a_trace_enable(True)
            state.step()
            recs = L.ds4a_trace_read()
            L.ds4a_trace_enable(False)
            n_launch += len(recs)
            for name, ms in recs:
                per.setdefault(name, []).append(ms)
    return per, n_launch / max(1, K)


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or
    None when there is none or its source has changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(f"{workload}:{kernel}")
    if not e:
        return None
    if e.get("source_hash") != source_hash(e.get("sources", [])):
        return None
    return e.get("bytes_per_launch_full")


# ---------------------------------------------------------------------------
# the oracle arm (CPU)
# ---------------------------------------------------------------------------
def oracle_step_fn(wid: int):
    """(fn, tokens, sample description): one bounded oracle pass on the host
    over a sample of the workload (test infrastructure)."""
    import numpy as np
    from gen import workloads as W
    from oracle import ds4a_oracle as O

    w = W.WORKLOADS[wid]
    if w.kind == "toy":
        x = W.toy_inputs(w)
        c = w.csa
        qp = W.query_positions(w)

        def fn():
            n = (w.pos + 1) // c.ratio
            pool = O.compress_batch(c.ratio, 0, n, 0, x["csa.kv_ca"], x["csa.kv_za"], x["csa.kv_ba"],
                                    x["csa.kv_cb"], x["csa.kv_zb"], x["csa.kv_bb"], x["csa.kv_g"], c.rope_dim)
            ki = O.compress_batch(c.ratio, 0, n, 0, x["csa.ix_ca"], x["csa.ix_za"], x["csa.ix_ba"],
                                  x["csa.ix_cb"], x["csa.ix_zb"], x["csa.ix_bb"])
            idx, _ = O.index_topk_batch(x["csa.qi"], x["csa.wi"], O.store_bf16(ki), qp, c.ratio, c.topk, n)
            O.csa_attend_batch(x["csa.q"], x["csa.q_norm_g"], O.store_bf16(pool), idx, x["csa.win"], w.pos + 1,
                               x["csa.sink"], qp, c)
        return fn, w.pos + 1, "whole toy layer (64 tokens)"
    sp = W.specs(w)
    H = {n: W.host_tensor(w, n) for n in sp if not n.endswith(("pool", "ki", "win")) and
         not (w.kind == "csa_prefill" and n in ("csa.q", "csa.qi", "csa.wi"))}
    if w.kind in ("csa_decode", "hca_decode", "mix_decode"):
        B = min(w.B, 2)
        layers = []
        if w.csa is not None and w.kind != "hca_decode":
            layers.append("csa")
        if w.hca is not None and w.kind != "csa_decode":
            layers.append("hca")
        st = {}
        for lay in layers:
            cfg = w.csa if lay == "csa" else w.hca
            n_c = w.n_csa if lay == "csa" else w.n_hca
            n_vis = min((w.pos + 1) // cfg.ratio, n_c)
            win = W.host_tensor(w, f"{lay}.win")[:B]
            st[lay] = (cfg, n_c, n_vis, win)
            if lay == "csa":
                st["ki"] = W.host_rows(w, "csa.ki", np.arange(B * w.n_csa)).reshape(B, w.n_csa, -1)
        rng_rows = np.arange(B)

        def fn():
            for lay in layers:
                cfg, n_c, n_vis, win = st[lay]
                for b in rng_rows:
                    if lay == "csa":
                        tb = w.pos - 2 * cfg.ratio + 1
                        e = O.compress(cfg.ratio, n_c - 1, n_c, tb, H["csa.kv_ca"][b], H["csa.kv_za"][b],
                                       H["csa.kv_ba"], H["csa.kv_cb"][b], H["csa.kv_zb"][b], H["csa.kv_bb"],
                                       H["csa.kv_g"], cfg.rope_dim)
                        ek = O.compress(cfg.ratio, n_c - 1, n_c, tb, H["csa.ix_ca"][b], H["csa.ix_za"][b],
                                        H["csa.ix_ba"], H["csa.ix_cb"][b], H["csa.ix_zb"][b], H["csa.ix_bb"])
                        ki = st["ki"][b].copy()
                        ki[n_c - 1] = O.store_bf16(ek[0])
                        idx, _ = O.index_topk(H["csa.qi"][b, 0], H["csa.wi"][b, 0], ki, w.pos, cfg.ratio,
                                              cfg.topk, n_c)
                        sel = idx[idx >= 0]
                        rows = W.host_rows(w, "csa.pool", b * n_c + sel)
                        rows[sel == n_c - 1] = O.store_bf16(e[0])
                        pool = np.zeros((n_c, cfg.head_dim), np.uint16)
                        pool[sel] = rows
                        O.csa_attend(H["csa.q"][b, 0], H["csa.q_norm_g"], pool, idx, win[b], cfg.window,
                                     H["csa.sink"], w.pos, cfg)
                    else:
                        tb = w.pos - cfg.ratio + 1
                        e = O.compress(cfg.ratio, n_c - 1, n_c, tb, H["hca.kv_c"][b], H["hca.kv_z"][b],
                                       H["hca.kv_b"], norm_g=H["hca.kv_g"], rope_dim=cfg.rope_dim)
                        pool = W.host_rows(w, "hca.pool", b * n_c + np.arange(n_vis))
                        pool[n_c - 1] = O.store_bf16(e[0])
                        O.hca_attend(H["hca.q"][b, 0], H["hca.q_norm_g"], pool, n_c, win[b], cfg.window,
                                     H["hca.sink"], w.pos, cfg)
        return fn, len(rng_rows), f"{len(rng_rows)} of {w.B} sequences, every layer of the step"
    # prefill: the compressor over all tokens once, then a few query rows
    c = w.csa
    n_c = w.n_csa
    rows = np.array([n_c * c.ratio - 1, 8191, 12000, 16383])
    qi = W.host_rows(w, "csa.qi", rows * c.idx_heads + np.arange(c.idx_heads)[:, None]).reshape(
        c.idx_heads, len(rows), -1).transpose(1, 0, 2)
    wi = W.host_rows(w, "csa.wi", rows).reshape(len(rows), -1)
    q = W.host_rows(w, "csa.q", rows * c.n_heads + np.arange(c.n_heads)[:, None]).reshape(
        c.n_heads, len(rows), -1).transpose(1, 0, 2)
    win_all = W.host_tensor(w, "csa.win")[0]

    def fn():
        pool = O.compress(c.ratio, 0, n_c, 0, H["csa.kv_ca"][0], H["csa.kv_za"][0], H["csa.kv_ba"],
                          H["csa.kv_cb"][0], H["csa.kv_zb"][0], H["csa.kv_bb"], H["csa.kv_g"], c.rope_dim)
        ki = O.compress(c.ratio, 0, n_c, 0, H["csa.ix_ca"][0], H["csa.ix_za"][0], H["csa.ix_ba"],
                        H["csa.ix_cb"][0], H["csa.ix_zb"][0], H["csa.ix_bb"])
        pb, kb = O.store_bf16(pool), O.store_bf16(ki)
        for r, t in enumerate(rows):
            idx, _ = O.index_topk(qi[r], wi[r], kb, int(t), c.ratio, c.topk, n_c)
            O.csa_attend(q[r], H["csa.q_norm_g"], pb, idx, win_all, w.pos + 1, H["csa.sink"], int(t), c)
    return fn, len(rows), f"compressor over all 16384 tokens + {len(rows)} of 16384 query rows"


def host_cores() -> int:
    """Cores of this host that the process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def time_oracle(wid: int, budget_s: float = 12.0, min_reps: int = 1, threads: int | None = None):
    """Oracle throughput on the host with its BLAS limited to `threads`
    (every host core by default); returns (tokens/s, s per pass, sample,
    threads used)."""
    from threadpoolctl import threadpool_limits

    n = threads or host_cores()
    fn, tokens, sample = oracle_step_fn(wid)
    with threadpool_limits(limits=n, user_api="blas"):
        fn()  # warm-up
        t0 = time.perf_counter()
        reps = 0
        while reps < min_reps or time.perf_counter() - t0 < budget_s:
            fn()
            reps += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = (time.perf_counter() - t0) / reps
    return tokens / dt, dt, sample, n


def cpu_baseline_line(wid: int) -> dict:
    """The oracle on every host core, and on one core, over a bounded sample."""
    v, dt, sample, n = time_oracle(wid)
    v1, dt1, _, _ = time_oracle(wid, budget_s=8.0, threads=1)
    return {"value": v, "unit": UNIT, "cores": n, "kind": "oracle", "sample": sample,
            "single_core": {"value": v1, "unit": UNIT, "cores": 1}}


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_label(wid):
    from gen import workloads as W
    return W.WORKLOADS[wid].name


def measure_workload(wid, args, stream, flush, barrier, world, dev, primary):
    import torch
    import long_context_hybrid_kv_b200 as L

    st = State(wid, dev)
    torch.cuda.synchronize()
    step_ms = time_steps(st.step, args.steps, args.warmup, stream, flush, graph=not args.no_graph,
                         barrier=barrier)
    local_ms = statistics.mean(step_ms)
    ms = max_over_ranks(local_ms, world, dev)
    rc, bits = L.ds4a_check()
    if rc != 0:
        raise RuntimeError(f"device error word {bits:#x} after the timed steps")
    per, launches_per_step = kernel_times(st, max(3, min(args.steps, 20)), stream, flush)
    work = kernel_work(st)
    fam_ms: dict[str, float] = {}
    fam_launches: dict[str, int] = {}
    for name, v in per.items():
        f = kernel_family(name)
        fam_ms[f] = fam_ms.get(f, 0.0) + sum(v) / max(1, min(args.steps, 20) if args.steps >= 3 else 3)
        fam_launches[f] = fam_launches.get(f, 0) + len(v)
    res = {
        "tokens_per_step": st.tokens,
        "ms_per_step": ms,
        "value": st.tokens * world / (ms / 1e3),
        "kernels": {name: {"launches_per_step": len(v) / max(1, max(3, min(args.steps, 20))),
                           "avg_ms": statistics.mean(v)} for name, v in sorted(per.items())},
        "launches_per_step": launches_per_step,
        "state": st,
        "work": work,
    }
    lib_ref = library_gemm_ms(st)
    if lib_ref is not None:
        res["library_reference"] = lib_ref
    return res


def step_roofline(res, peaks, peak_src, workload):
    """The whole step against the roofline: decode moves its algorithmic
    bytes in one step time (HBM bound); prefill runs its indexer and
    attention flops, over the step and over those kernels' own time."""
    work = res["work"]
    ms = res["ms_per_step"]
    if "outproj_prefill" in workload:
        flops = work.get("out_proj_gemm", (0, 0, 0))[1]
        ach = flops / (ms / 1e3) / 1e12
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        return {"bound": "tensor", "unit": "TFLOP/s", "what": "projection flops per step", "algorithmic": flops,
                "achieved": ach, "frac": ach / peak, "frac_datasheet": ach / DATASHEET_PEAKS["bf16_tflops"],
                "peak": peak, "peak_source": peak_src, "peak_datasheet": DATASHEET_PEAKS["bf16_tflops"]}
    if "prefill" in workload:
        flops = work.get("index_score", (0, 0, 0))[1] + work.get("attend", (0, 0, 0))[1]
        fam_ms = {}
        for name, k in res["kernels"].items():
            f = kernel_family(name)
            fam_ms[f] = fam_ms.get(f, 0.0) + k["avg_ms"] * k["launches_per_step"]
        # the indexer's top-k and the prepared-query kernel belong to the
        # indexer + attention work
        ia_ms = sum(v for f, v in fam_ms.items() if f in ("index_score", "topk", "attend", "qhat_prep",
                                                          "attend_combine"))
        ach = flops / (ms / 1e3) / 1e12
        ach_ia = flops / (ia_ms / 1e3) / 1e12 if ia_ms > 0 else None
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        return {"bound": "tensor", "unit": "TFLOP/s", "what": "indexer + attention flops per step",
                "algorithmic": flops, "achieved": ach, "frac": ach / peak,
                "frac_datasheet": ach / DATASHEET_PEAKS["bf16_tflops"],
                "indexer_attention_kernels": {"ms": ia_ms, "achieved": ach_ia,
                                              "frac": None if ach_ia is None else ach_ia / peak,
                                              "frac_datasheet": None if ach_ia is None else
                                              ach_ia / DATASHEET_PEAKS["bf16_tflops"]},
                "peak": peak, "peak_source": peak_src, "peak_datasheet": DATASHEET_PEAKS["bf16_tflops"]}
    nbytes = sum(v[0] for v in work.values())
    ach = nbytes / (ms / 1e3) / 1e9
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    return {"bound": "hbm", "unit": "GB/s", "what": "algorithmic bytes of the whole step / step time",
            "algorithmic": nbytes, "achieved": ach, "frac": ach / peak,
            "frac_datasheet": ach / DATASHEET_PEAKS["hbm_gbs"], "peak": peak, "peak_source": peak_src,
            "peak_datasheet": DATASHEET_PEAKS["hbm_gbs"]}


def library_gemm_ms(st, K: int = 10) -> dict | None:
    """For the output-projection workloads: the same two products through
    torch (cuBLAS), timed with CUDA events as a reference point (not part of
    this library's path)."""
    import torch

    ly = st.layers[0]
    if ly.kind != "out_proj":
        return None
    cf = ly.cfg
    M = ly.B
    o = ly.t["o"].view(M, cf.n_groups, -1).transpose(0, 1)         # [g, M, K1]
    wa = ly.t["w_a"].transpose(1, 2)                                 # [g, K1, r]
    wb = ly.t["w_b"]

    def run():
        mid = torch.bmm(o, wa).transpose(0, 1).reshape(M, -1)
        return mid @ wb.t()

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    ts = []
    for _ in range(K):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = statistics.mean(ts)
    flops = st_flops = 2.0 * M * 2 * (cf.n_groups * cf.group_rank) * ((cf.n_heads // cf.n_groups) * cf.head_dim)
    return {"what": "torch bmm + matmul (cuBLAS), same products, context only", "ms": ms,
            "tflops": st_flops / (ms / 1e3) / 1e12}


def roofline_for(res, peaks, peak_src, workload):
    """Roofline of the kernel with the largest share of the step (and the
    whole step's, under "step")."""
    kinfo = res["kernels"]
    if not kinfo:
        return None
    share = {n: k["avg_ms"] * k["launches_per_step"] for n, k in kinfo.items()}
    top = max(share, key=share.get)
    fam = kernel_family(top)
    nbytes, flops, launches = res["work"].get(fam, (0.0, 0.0, 1))
    per_launch_ms = kinfo[top]["avg_ms"]
    n_l = max(1, kinfo[top]["launches_per_step"])
    b_launch = nbytes / max(1, launches)
    f_launch = flops / max(1, launches)
    dense = "prefill" in workload
    if dense and f_launch > 0:
        achieved = f_launch / (per_launch_ms / 1e3) / 1e12
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
             "frac": achieved / peak}
    else:
        achieved = b_launch / (per_launch_ms / 1e3) / 1e9
        peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        r = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak}
    r.update({"kernel": top, "traffic": ncu_traffic(top, workload), "peak_source": peak_src,
              "frac_datasheet": achieved / DATASHEET_PEAKS["bf16_tflops" if r["bound"] == "tensor" else "hbm_gbs"],
              "algorithmic_bytes_per_launch": b_launch, "algorithmic_flops_per_launch": f_launch,
              "avg_launch_ms": per_launch_ms, "share_of_step": share[top] / max(1e-12, sum(share.values())),
              "step": step_roofline(res, peaks, peak_src, workload)})
    return r


def stage_inputs(st):
    """Make every per-step input of the workload a view of one device buffer
    (256-byte aligned slots) and return it with a pinned host copy: a
    step's inputs then cross in one transfer instead of one per tensor, as a
    serving loop with a single staging buffer would send them."""
    import torch

    align = 256
    slots, off = [], 0
    for ly in st.layers:
        for n in ly.step_inputs:
            t = ly.t[n]
            nb = t.numel() * t.element_size()
            slots.append((ly, n, off, nb))
            off += (nb + align - 1) // align * align
    dbuf = torch.empty(off, dtype=torch.uint8, device=st.layers[0].out.device)
    hbuf = torch.empty(off, dtype=torch.uint8, pin_memory=True)
    for ly, n, o, nb in slots:
        t = ly.t[n].contiguous()
        view = dbuf[o:o + nb].view(t.dtype).view(t.shape)
        view.copy_(t)
        hbuf[o:o + nb].copy_(t.reshape(-1).view(torch.uint8).cpu())
        ly.t[n] = view
    for ly in st.layers:
        if ly.kind == "csa":
            _csa_jobs(ly)
    return dbuf, hbuf


def measure_e2e(st, args, stream):
    """Same metric through the public API with host buffers: every step
    copies its inputs from pinned host memory (one staging transfer) and
    reads its result back."""
    import torch

    dbuf, hbuf = stage_inputs(st)
    _, outs = st.step_io()
    h_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    bi = hbuf.numel()
    bo = sum(t.numel() * t.element_size() for t in h_out)

    def e2e_step():
        dbuf.copy_(hbuf, non_blocking=True)
        st.step()
        for h, d in zip(h_out, outs):
            h.copy_(d, non_blocking=True)
        torch.cuda.current_stream().synchronize()  # the host reads the result

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        K = max(3, args.steps)
        t0 = time.perf_counter()
        for _ in range(K):
            e2e_step()
        dt = (time.perf_counter() - t0) / K
    return {"value": st.tokens / dt, "unit": UNIT, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "ms_per_step": dt * 1e3}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from threadpoolctl import threadpool_limits

    wid = args.workload_ids[0]
    steps = []
    fn, tokens, sample = oracle_step_fn(wid)
    cores = host_cores()
    with threadpool_limits(limits=cores, user_api="blas"):
        for _ in range(args.warmup):
            fn()
        for _ in range(args.steps):
            t0 = time.perf_counter()
            fn()
            steps.append(time.perf_counter() - t0)
    dt = statistics.mean(steps)
    value = tokens / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_label(wid), "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workloads", default="5,2,3,4,7")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    args.workload_ids = [int(x) for x in args.workloads.split(",") if x.strip()]
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import long_context_hybrid_kv_b200 as L

    rank, world, local = dist_env()
    L.lib()  # fails loudly if the library is missing
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    barrier = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        barrier = dist.barrier
    stream = torch.cuda.Stream(device=dev)
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.fill_(1.0)

    peaks, peak_src = load_peaks()
    wids = args.workload_ids if world == 1 else args.workload_ids[:1]
    results = {}
    with ClockSampler(local) as clk:
        for i, wid in enumerate(wids):
            results[wid] = measure_workload(wid, args, stream, flush, barrier, world, dev, i == 0)
    clocks = clk.summary()
    prim = wids[0]
    r = results[prim]
    label = workload_label(prim)
    line = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": label, "tokens_per_step": r["tokens_per_step"],
                       "l2": "256 MiB write between steps, outside the step events",
                       "graph": not args.no_graph, "parallelism": f"replicas x{world}"},
            "gpu_launches": int(round(r["launches_per_step"] * args.steps)),
            "roofline": roofline_for(r, peaks, peak_src, label),
            "clocks": clocks}
    if not args.no_e2e:
        line["e2e"] = measure_e2e(r["state"], args, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_line(prim)
    others = {}
    for wid in wids[1:]:
        rr = results[wid]
        lab = workload_label(wid)
        others[lab] = {"value": rr["value"], "unit": UNIT, "ms_per_step": rr["ms_per_step"],
                       "tokens_per_step": rr["tokens_per_step"],
                       "roofline": roofline_for(rr, peaks, peak_src, lab),
                       "kernels": rr["kernels"]}
        if "library_reference" in rr:
            others[lab]["library_reference"] = rr["library_reference"]
    line["kernels"] = r["kernels"]
    if others:
        line["workloads"] = others
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
