"""Device-side table filling with the generator of synth/gen.py (needs a GPU)."""
from __future__ import annotations

import ctypes
import os

from . import gen

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libngram_synth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run `python -m synth.build` first")
        lib = ctypes.CDLL(path)
        lib.synth_fill_table.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.c_uint64, ctypes.c_int32, ctypes.c_float,
                                         ctypes.c_int32, ctypes.c_void_p]
        lib.synth_fill_table.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def fill_table(t, seed: int, tag: int, std: float, stream=None) -> None:
    """Fill a contiguous 2-D torch CUDA tensor (bf16 or fp32) in place."""
    import torch
    assert t.is_cuda and t.is_contiguous() and t.dim() == 2
    dtype = {torch.bfloat16: 0, torch.float32: 1}[t.dtype]
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    rc = _lib().synth_fill_table(ctypes.c_void_p(t.data_ptr()), t.shape[0], t.shape[1],
                                 ctypes.c_uint64(seed), tag, float(gen.value_scale(std)), dtype,
                                 ctypes.c_void_p(s.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_table failed with CUDA error {rc}")
