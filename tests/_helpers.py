"""Shared helpers of the GPU parity tests: moving seeded host arrays to the
device and comparing device results with the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances. bf16 storage with fp32 accumulation: the bound stated for the
# method (max abs error <= 2e-2, max relative error <= 1e-2, relative error
# taken as max|err| / max|ref| because elementwise ratios are undefined near
# zero). float32 storage: fp32 arithmetic over at most a few thousand terms
# keeps the error below 1e-4 absolute.
TOL = {"bf16": (2e-2, 1e-2), "f32": (1e-4, 1e-4)}

GUARD = 4096  # bytes of sentinel before and after every output buffer


def dev(a: np.ndarray) -> torch.Tensor:
    """Host array -> contiguous CUDA tensor (uint16 arrays are bfloat16 bits)."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def kind(a) -> str:
    if isinstance(a, torch.Tensor):
        return "bf16" if a.dtype == torch.bfloat16 else "f32"
    return "bf16" if a.dtype == np.uint16 else "f32"


def errors(got: np.ndarray, ref: np.ndarray):
    """(max abs error, max|err|/max|ref|, rms relative error) of stored values vs float64."""
    g = oracle.widen(got)
    err = np.abs(g - ref)
    mref = float(np.max(np.abs(ref))) if ref.size else 0.0
    max_abs = float(np.max(err)) if err.size else 0.0
    rel = max_abs / mref if mref > 0 else max_abs
    rms = float(np.sqrt(np.sum(err**2) / max(np.sum(ref**2), 1e-300))) if ref.size else 0.0
    return max_abs, rel, rms


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert np.all(np.isfinite(oracle.widen(got))), f"{what}: non-finite output"
    tol_abs, tol_rel = TOL[kind(got)]
    max_abs, rel, rms = errors(got, ref)
    assert max_abs <= tol_abs and rel <= tol_rel, f"{what}: max abs {max_abs:.3e}, rel {rel:.3e}, rms {rms:.3e}"
    return max_abs, rel


class Guarded:
    """A CUDA buffer with sentinel bytes on both sides, checked after use."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        esz = torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD * 2 + n * esz,), 0xA5, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n * esz].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.raw[:GUARD] == 0xA5).all().item() and (self.raw[-GUARD:] == 0xA5).all().item())
