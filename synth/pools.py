"""Device expert pools for tests and the benchmark.

Draws the natural-layout expert bytes on the GPU with the generator twin
(synth/csrc/synth.cu) and converts them to the library's packed layout with
its C-ABI call moe_pack_tensor.  No layer arithmetic here.
"""
from __future__ import annotations

import numpy as np
import torch

from . import LayerShape
from . import device as sdev


def dev(a) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if not a.flags.writeable:      # e.g. a view of an immutable buffer
        a = a.copy()
    return torch.from_numpy(a).cuda()


def build_pool(shape: LayerShape, seed: int, layer: int,
               n_experts: int | None = None, chunk: int = 64,
               pool: torch.Tensor | None = None, blob0: int = 0
               ) -> torch.Tensor:
    """Packed expert pool of one layer (experts 0..n-1); blob e at byte
    offset (blob0 + e) * shape.blob_stride."""
    import quantized_moe_expert_02_b200 as moe
    n = shape.E if n_experts is None else n_experts
    stride = shape.blob_stride
    if pool is None:
        pool = torch.empty((blob0 + n) * stride, dtype=torch.uint8,
                           device="cuda")
    stage = torch.empty(min(chunk, n) * stride, dtype=torch.uint8,
                        device="cuda")
    off = shape.tensor_offsets()
    s = torch.cuda.current_stream().cuda_stream
    for e0 in range(0, n, chunk):
        m = min(chunk, n - e0)
        sdev.fill_experts(stage.data_ptr(), stride, shape, seed, layer, e0, m,
                          s)
        for i in range(m):
            nat = stage.data_ptr() + i * stride
            dst = pool.data_ptr() + (blob0 + e0 + i) * stride
            for name, fmt, rows, cols in (
                    ("up", shape.fmt_up_gate, shape.F, shape.H),
                    ("gate", shape.fmt_up_gate, shape.F, shape.H),
                    ("down", shape.fmt_down, shape.H, shape.F)):
                moe.moe_pack_tensor(fmt, nat + off[name], rows, cols,
                                    dst + off[name], s)
    torch.cuda.synchronize()
    del stage
    return pool


def layer_desc(shape: LayerShape, pool: torch.Tensor, base_blob: int = 0):
    import quantized_moe_expert_02_b200 as moe
    return moe.moe_layer_desc(
        H=shape.H, F=shape.F, E=shape.E, fmt_up_gate=shape.fmt_up_gate,
        fmt_down=shape.fmt_down,
        pool=pool.data_ptr() + base_blob * shape.blob_stride,
        blob_stride=shape.blob_stride)
