"""Helpers shared by the GPU parity tests."""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from diffusion_decoding_step_b200 import abi, build

_built = False


def ensure_lib():
    global _built
    if not _built:
        build.build()
        abi.lib()
        _built = True
    return abi


def ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_ulp_close(gpu: np.ndarray, ref: np.ndarray, ulps: float = 1.0, atol: float = 0.0):
    """Assert |gpu - ref| <= ulps * spacing(bf16 at |ref|) + atol, elementwise."""
    mag = np.maximum(np.abs(ref), 1e-30)
    spacing = 2.0 ** (np.floor(np.log2(mag)) - 7)
    err = np.abs(gpu - ref)
    bad = err > ulps * spacing + atol
    if bad.any():
        i = np.argmax(err - ulps * spacing - atol)
        raise AssertionError(f"{bad.sum()} of {bad.size} elements off by more than {ulps} ulp; "
                             f"worst gpu={gpu.flat[i]} ref={ref.flat[i]}")


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
