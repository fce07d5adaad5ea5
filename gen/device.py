"""Device side of the seeded generator: fills CUDA tensors with the numbers
``gen.host`` produces for the same (seed, name, element), using the kernel in
``gen/device.cu`` (built into gen/_lib/libds4gen.so by ``build()``)."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import host, workloads

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "_lib", "libds4gen.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "device.cu")
    if force or not os.path.exists(SO) or os.path.getmtime(src) > os.path.getmtime(SO):
        os.makedirs(os.path.dirname(SO), exist_ok=True)
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-shared",
               "-Xcompiler", "-fPIC", "-o", SO, src]
        subprocess.run(cmd, check=True)
    return SO


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(f"{SO} is missing: run __graft_entry__.build()")
        _lib = ctypes.CDLL(SO)
        _lib.ds4gen_fill.restype = ctypes.c_int
        _lib.ds4gen_fill.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
                                     ctypes.c_uint64, ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                                     ctypes.c_int, ctypes.c_float, ctypes.c_void_p]
    return _lib


_tables: dict = {}


def _table(device):
    """The host's normal table, uploaded once per device."""
    import torch

    key = str(device)
    if key not in _tables:
        _tables[key] = torch.from_numpy(host.normal_table().reshape(-1).copy()).to(device)
    return _tables[key]


def fill(t, seed: int, name: str, scale=None, offset=None, start: int = 0, stream=None):
    """Fill the contiguous CUDA tensor t (bfloat16 or float32) in place."""
    import torch

    assert t.is_cuda and t.is_contiguous()
    is_bf16 = {torch.bfloat16: 1, torch.float32: 0}[t.dtype]
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    rc = lib().ds4gen_fill(
        ctypes.c_void_p(t.data_ptr()), is_bf16, t.numel(), host.stream_key(seed, name), start,
        ctypes.c_void_p(_table(t.device).data_ptr()), scale is not None, 0.0 if scale is None else float(np.float32(scale)),
        offset is not None, 0.0 if offset is None else float(np.float32(offset)), ctypes.c_void_p(s))
    if rc != 0:
        raise RuntimeError(f"ds4gen_fill failed ({rc})")
    return t


def tensor(w: "workloads.Workload", name: str, device="cuda"):
    """A new CUDA tensor with the named workload tensor."""
    import torch

    spec = workloads.specs(w)[name]
    dt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    t = torch.empty(spec.shape, dtype=dt, device=device)
    return fill(t, w.seed, name, spec.scale, spec.offset)


def workload_tensors(w: "workloads.Workload", names=None, device="cuda") -> dict:
    """Every generated tensor of a Flash-shape workload as CUDA tensors
    (the toy is built on the host by ``workloads.toy_inputs``)."""
    sp = workloads.specs(w)
    return {n: tensor(w, n, device) for n in (names or sp)}
