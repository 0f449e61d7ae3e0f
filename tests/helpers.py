"""Shared helpers of the GPU parity tests: device pools from the seeded
generator, host-side oracle inputs, error metrics."""
from __future__ import annotations

import numpy as np
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe

TOL = 2e-3   # max relative error of FFN outputs (per row, max-norm)


from synth.pools import build_pool, dev, layer_desc  # noqa: F401


def stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def pack_natural(fmt: int, natural: torch.Tensor, rows: int, cols: int
                 ) -> torch.Tensor:
    out = torch.empty(moe.moe_tensor_bytes(fmt, rows, cols), dtype=torch.uint8,
                      device="cuda")
    moe.moe_pack_tensor(fmt, natural, rows, cols, out)
    return out


def oracle_experts(shape: synth.LayerShape, seed: int, layer: int
                   ) -> o.ExpertSource:
    return o.ExpertSource(shape.H, shape.F, shape.fmt_up_gate, shape.fmt_down,
                          lambda e: synth.gen_expert_blob(shape, seed, layer,
                                                          e))


def route_inputs(shape, seed, layer, T, step=0, zipf=False):
    x = synth.gen_x(seed, T, shape.H, step)
    wr = synth.gen_router(seed, layer, shape.E, shape.H)
    bias = synth.gen_zipf_bias(seed, layer, shape.E)[0] if zipf else None
    return x, wr, bias


def row_max_rel(y: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of max_h |y - ref| / max_h |ref|."""
    y = np.asarray(y, np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, np.float64).reshape(ref.shape[0], -1)
    num = np.abs(y - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((num / den).max())


def logit_bound(x: np.ndarray, wr: np.ndarray, H: int) -> np.ndarray:
    """Forward error bound of an fp32 dot product of length H per (t, e):
    gamma_H * sum_h |x_h w_eh| with gamma_H = H * 2^-24 (plus one rounding
    of the bias add)."""
    s = np.abs(x) @ np.abs(wr).T
    return (H + 2) * 2.0 ** -24 * s + 1e-7


class Ws:
    """A zero-initialised device workspace."""

    def __init__(self, nbytes: int):
        self.nbytes = int(nbytes)
        self.t = torch.zeros(max(self.nbytes, 256), dtype=torch.uint8,
                             device="cuda")

    @property
    def ptr(self):
        return self.t.data_ptr()


def run_route(x, wr, bias, k, T, H, E):
    xd, wd = dev(x), dev(wr)
    bd = dev(bias) if bias is not None else None
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    moe.moe_route_topk(xd, T, H, wd, E, bd, k, idx, w, lg)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), lg.cpu().numpy()


def run_group(idx: np.ndarray, E: int):
    T, k = idx.shape
    ws = Ws(moe.moe_group_workspace_bytes(T, k, E))
    d_idx = dev(idx.astype(np.int32))
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pairs = torch.empty(T * k, dtype=torch.int32, device="cuda")
    act = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    na = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_group_tokens(d_idx, T, k, E, off, pairs, act, na, ws.t,
                         ws.nbytes)
    err = moe.moe_get_device_status(ws.t)
    n = int(na.item())
    return (off.cpu().numpy(), pairs.cpu().numpy(), act.cpu().numpy()[:n],
            err, (d_idx, off, pairs, act, na))
