"""GPU: this library's two further up/gate formats end to end -- the 3-bit
non-uniform-codebook super-block (MOE_NL3_256, stand-in for the 3-bit
non-linear type the model card lists) and the 2-bit super-block
(MOE_SB2_256, stand-in for the card's 2-bit up/gate type) -- with down in
NL4, through the one-kernel decode layer, the split decode kernels and the
tensor-core prefill path, against the fp64 oracle (whose dequantisation of
both formats is pinned on the CPU)."""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import (TOL, Ws, build_pool, dev, layer_desc, oracle_experts,
                     route_inputs, row_max_rel, run_group, run_route)

pytestmark = pytest.mark.gpu

SHAPES = {"nl3": synth.NL3_SHAPE, "sb2": synth.SB2_SHAPE}
_POOL = {}


@pytest.fixture(params=sorted(SHAPES))
def fmt_shape(request):
    """(name, shape); one resident pool per format, the previous one freed."""
    name = request.param
    if name not in _POOL:
        _POOL.clear()
        torch.cuda.empty_cache()
        _POOL[name] = build_pool(SHAPES[name], 0, 0)
    return SHAPES[name], _POOL[name]


def oracle_y(SHAPE, x_bits, idx):
    src = oracle_experts(SHAPE, 0, 0)
    x = o.bf16_to_f64(x_bits)
    T, k = idx.shape
    off, pairs, act = o.group_pairs(idx, SHAPE.E)
    y = np.zeros((T * k, SHAPE.H))
    for e in act:
        pp = pairs[off[e]:off[e + 1]]
        y[pp] = o.expert_ffn(x[pp // k], *src.weights(int(e)))[1]
    return y


@pytest.mark.parametrize("T", [1, 3, 8, 40, 300])
def test_expert_ffn_vs_oracle(fmt_shape, T):
    """T <= 8: split decode kernels; T > 8: the prefill GEMMs."""
    SHAPE, pool = fmt_shape
    desc = layer_desc(SHAPE, pool)
    x, wr, _ = route_inputs(SHAPE, 0, 0, T, step=1)
    idx, _, _ = run_route(x, wr, None, SHAPE.k, T, SHAPE.H, SHAPE.E)
    _, _, _, err, (d_idx, off, pairs, act, na) = run_group(idx, SHAPE.E)
    assert err == 0
    ws = Ws(moe.moe_ffn_workspace_bytes(T, SHAPE.k, SHAPE.H, SHAPE.F))
    y = torch.full((T * SHAPE.k, SHAPE.H), float("nan"), device="cuda")
    moe.moe_expert_ffn_q(desc, dev(x), T, SHAPE.k, off, pairs, act, na, None,
                         y, ws.t, ws.nbytes)
    assert moe.moe_get_device_status(ws.t) == 0
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    assert row_max_rel(got, oracle_y(SHAPE, x, idx)) <= TOL


@pytest.mark.parametrize("T", [1, 3, 5])
def test_layer_forward_vs_oracle(fmt_shape, T):
    """The one-kernel decode layer with NL3 or SB2 up/gate."""
    SHAPE, pool = fmt_shape
    desc = layer_desc(SHAPE, pool)
    k, E, H = SHAPE.k, SHAPE.E, SHAPE.H
    x, wr, _ = route_inputs(SHAPE, 0, 0, T, step=2)
    ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, SHAPE.F))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    lg = torch.empty((T, E), device="cuda")
    out = torch.empty((T, H), device="cuda")
    moe.moe_layer_forward(desc, dev(x), T, k, dev(wr), None, None, None, out,
                          None, idx, w, lg, ws.t, ws.nbytes)
    assert moe.moe_get_device_status(ws.t) == 0
    gi = idx.cpu().numpy()
    assert np.array_equal(gi, o.topk_select(lg.cpu().numpy(), k))
    ref = o.moe_layer(o.bf16_to_f64(x), o.bf16_to_f64(wr), None, k,
                      oracle_experts(SHAPE, 0, 0), topk_idx=gi)
    assert row_max_rel(out.cpu().numpy(), ref["out"]) <= TOL
