"""Shared helpers for the GPU parity tests (device copies of the seeded
inputs, tolerance checks).  Tolerances: max|gpu - oracle| <= 1e-2 * max|oracle|
for bf16 storage with fp32 accumulation, <= 1e-5 * max|oracle| for fp32."""
from __future__ import annotations

import numpy as np

TOL = {"bf16": 1e-2, "f32": 1e-5}


def dev(a, dtype: str):
    """numpy storage array (bf16 bit patterns or fp32/int32) -> CUDA tensor."""
    import torch
    if a is None:
        return None
    if dtype == "bf16" and a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def empty(shape, dtype: str):
    import torch
    td = {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32}[dtype]
    return torch.empty(shape, dtype=td, device="cuda")


def f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def bits(t) -> np.ndarray:
    """Raw storage of a CUDA tensor as numpy (bf16 -> uint16)."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def assert_close(gpu: np.ndarray, ref: np.ndarray, rel: float, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    if ref.size == 0:
        return
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    scale = float(np.max(np.abs(ref)))
    err = float(np.max(np.abs(gpu - ref)))
    assert err <= rel * max(scale, 1e-30), f"{what}: max err {err:.3e} > {rel:g} * {scale:.3e}"


def read_device(ptr: int, nbytes: int) -> np.ndarray:
    """Copy nbytes from a raw device address into a uint8 numpy array."""
    import ctypes
    import glob
    import os

    import torch
    torch.cuda.synchronize()
    cands = ["libcudart.so.12"] + glob.glob(os.path.join(
        os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib", "libcudart.so*"))
    rt = None
    for c in cands:
        try:
            rt = ctypes.CDLL(c)
            break
        except OSError:
            continue
    assert rt is not None, "libcudart not found"
    out = np.empty(nbytes, dtype=np.uint8)
    rt.cudaMemcpy.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int]
    assert rt.cudaMemcpy(out.ctypes.data, ptr, nbytes, 4) == 0
    return out
