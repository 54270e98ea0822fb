"""Device-side counter-based fill (same definition and bits as synth.fill), via ctypes."""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import torch

from .fill import FillSpec

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fill_gpu.cu")
_LIB = os.path.join(_HERE, "libsynth_fill.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
        subprocess.check_call([nvcc if os.path.exists(nvcc) else "nvcc", "-gencode",
                               "arch=compute_100a,code=sm_100a", "-O3", "-Xcompiler", "-fPIC", "-shared",
                               "-o", _LIB, _SRC])
    return _LIB


def _get():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB):
            raise ImportError(f"{_LIB} is missing; run synth.fill_gpu.build()")
        L = C.CDLL(_LIB)
        L.synth_fill_bf16.restype = C.c_int
        L.synth_fill_bf16.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64, C.c_float, C.c_void_p]
        L.synth_fill_fp8.restype = C.c_int
        L.synth_fill_fp8.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64, C.c_void_p]
        L.synth_host_alloc_mapped.restype = C.c_int
        L.synth_host_alloc_mapped.argtypes = [C.c_uint64, C.POINTER(C.c_void_p)]
        L.synth_host_free.restype = C.c_int
        L.synth_host_free.argtypes = [C.c_void_p]
        _lib = L
    return _lib


def fill_(t: torch.Tensor, spec: FillSpec, offset: int = 0, stream=None) -> torch.Tensor:
    """Fill a contiguous bf16/int16 tensor (device or pinned-mapped) in place."""
    assert t.is_contiguous() and t.element_size() == 2
    if stream is None:
        stream = torch.cuda.current_stream()
    rc = _get().synth_fill_bf16(C.c_void_p(t.data_ptr()), t.numel(), offset, spec.key,
                                float(spec.scale), C.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_bf16 failed with CUDA error {rc}")
    return t


def fill_fp8_(t: torch.Tensor, spec: FillSpec, stream=None) -> torch.Tensor:
    """Fill a contiguous uint8 tensor (device or pinned-mapped) with e4m3 codes."""
    assert t.is_contiguous() and t.element_size() == 1
    if stream is None:
        stream = torch.cuda.current_stream()
    rc = _get().synth_fill_fp8(C.c_void_p(t.data_ptr()), t.numel(), 0, spec.key, C.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_fp8 failed with CUDA error {rc}")
    return t


def filled_fp8(shape, spec: FillSpec, device="cuda") -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.uint8, device=device)
    return fill_fp8_(t, spec)


def filled(shape, spec: FillSpec, device="cuda") -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.bfloat16, device=device)
    return fill_(t, spec)


class HostMapped:
    """A pinned, device-mapped host buffer viewed as a CPU torch tensor of bf16 [rows, cols].
    Its data_ptr() is valid on the device too (unified addressing).  Freed by close()."""

    def __init__(self, rows: int, cols: int, elem_bytes: int = 2):
        self.ptr = C.c_void_p()
        nbytes = int(rows) * int(cols) * elem_bytes
        rc = _get().synth_host_alloc_mapped(nbytes, C.byref(self.ptr))
        if rc != 0 or not self.ptr.value:
            raise MemoryError(f"cudaHostAlloc({nbytes} bytes, mapped) failed with CUDA error {rc}")
        import numpy as np
        if elem_bytes == 2:
            arr = np.ctypeslib.as_array((C.c_int16 * (int(rows) * int(cols))).from_address(self.ptr.value))
            self.tensor = torch.from_numpy(arr).view(torch.bfloat16).view(int(rows), int(cols))
        else:
            arr = np.ctypeslib.as_array((C.c_uint8 * (int(rows) * int(cols))).from_address(self.ptr.value))
            self.tensor = torch.from_numpy(arr).view(int(rows), int(cols))

    def close(self):
        if self.ptr is not None and self.ptr.value:
            self.tensor = None
            _get().synth_host_free(self.ptr)
            self.ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
