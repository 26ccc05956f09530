"""GPU fill of large synthetic tensors with the generator of ``datagen`` (bit-identical)."""
from __future__ import annotations

import ctypes

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        lib.dg_fill_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32,
                                       ctypes.c_uint32, ctypes.c_uint64, ctypes.c_void_p]
        lib.dg_fill_normal.restype = ctypes.c_int
        _lib = lib
    return _lib


def fill_normal(t, seed: int, tensor_id: int, first_index: int = 0, stream=None) -> None:
    """Fill a contiguous CUDA tensor (float32 or bfloat16) with x_{first_index + i}."""
    import torch
    assert t.is_cuda and t.is_contiguous() and t.dtype in (torch.float32, torch.bfloat16)
    if stream is None:
        stream = torch.cuda.current_stream(t.device).cuda_stream
    rc = _load().dg_fill_normal(ctypes.c_void_p(t.data_ptr()), 1 if t.dtype == torch.bfloat16 else 0,
                                t.numel(), seed, tensor_id, first_index, ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"dg_fill_normal failed ({rc})")
