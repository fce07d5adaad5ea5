"""Helpers of the GPU tests: uploads of generator arrays and downloads."""
from __future__ import annotations

import numpy as np
import torch

import long_context_hybrid_kv_b200 as L


def dev():
    return torch.device("cuda:0")


def bf(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bfloat16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(dev()).view(torch.bfloat16)


def f32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())


def bits(t: torch.Tensor) -> np.ndarray:
    """CUDA bfloat16 tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def ws_f32(nbytes: int) -> torch.Tensor:
    return torch.empty(max(1, (nbytes + 3) // 4), dtype=torch.float32, device=dev())


def check_ok():
    rc, b = L.ds4a_check()
    assert rc == L.DS4A_OK, f"device error word {b:#x}: {L.ds4a_strerror(rc)}"


def kernels_used(fn) -> list[str]:
    """Names of the library kernels one call of fn launches."""
    L.ds4a_trace_enable(True)
    try:
        fn()
        return [n for n, _ in L.ds4a_trace_read()]
    finally:
        L.ds4a_trace_enable(False)
