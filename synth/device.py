"""Loader of synth/libsynth.so: the device twin of the expert-byte generator.

Only draws inputs (natural-layout expert bytes); no layer arithmetic.
"""
from __future__ import annotations

import ctypes
import os

from . import LayerShape

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsynth.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} missing: run synth/_build.py")
        _lib = ctypes.CDLL(LIB_PATH)
        _lib.synth_fill_experts.restype = ctypes.c_int
        _lib.synth_fill_experts.argtypes = [
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
            ctypes.c_double, ctypes.c_double, ctypes.c_uint64, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    return _lib


def fill_experts(dst_ptr: int, blob_stride: int, shape: LayerShape, seed: int,
                 layer: int, expert0: int, nexperts: int, stream: int) -> None:
    """Write natural-layout blobs of experts expert0.. of `layer` at
    dst_ptr + i * blob_stride (device memory)."""
    rc = _load().synth_fill_experts(
        dst_ptr, blob_stride, shape.fmt_up_gate, shape.fmt_down, shape.H,
        shape.F, shape.d_up_gate[0], shape.d_up_gate[1], shape.d_down[0],
        shape.d_down[1], seed, layer, expert0, nexperts, stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_experts: CUDA error {rc}")
