"""GPU: edge cases of the one-kernel decode layer (moe_layer_forward with
T <= 8 runs routing, top-k, grouping, FFN and combine in one launch, with
its own top-k code, not moe_route_topk's).

  * ties: duplicated router rows give equal logits; the layer's own top-k
    must order them by ascending expert index (the rule of the tiny
    configuration), for the 16- and the 32-keys-per-lane variants;
  * k = E: every expert chosen, the weights are the full softmax;
  * outlier activations: one channel 2^8 or 2^12 times the row's rms, and
    a row scaled down by 2^-20, against the oracle at the 2e-3 bound.
"""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import (TOL, Ws, build_pool, dev, layer_desc, oracle_experts,
                     route_inputs, row_max_rel)

pytestmark = pytest.mark.gpu

_POOLS = {}

WIDE = synth.LayerShape(H=512, F=256, E=1024, k=8,
                        fmt_up_gate=synth.SB3_256, fmt_down=synth.NL4_B32,
                        d_up_gate=(0.002, 0.01), d_down=(0.002, 0.01))


def pool_for(shape, seed=0, layer=0):
    key = (shape, seed, layer)
    if key not in _POOLS:
        _POOLS.clear()
        torch.cuda.empty_cache()
        _POOLS[key] = build_pool(shape, seed, layer)
    return _POOLS[key]


def run_layer(shape, x_bits, wr_bits, k, bias=None):
    """moe_layer_forward; returns (out, idx, w, logits) as numpy."""
    T = x_bits.shape[0]
    E, H = shape.E, shape.H
    desc = layer_desc(shape, pool_for(shape))
    ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, shape.F))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    lg = torch.empty((T, E), device="cuda")
    out = torch.full((T, H), float("nan"), device="cuda")
    moe.moe_layer_forward(desc, dev(x_bits), T, k, dev(wr_bits),
                          dev(bias) if bias is not None else None, None,
                          None, out, None, idx, w, lg, ws.t, ws.nbytes)
    assert moe.moe_get_device_status(ws.t) == 0
    return (out.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(),
            lg.cpu().numpy())


def oracle_out(shape, x_bits, wr_bits, k, idx, bias=None):
    src = oracle_experts(shape, 0, 0)
    return o.moe_layer(o.bf16_to_f64(x_bits), o.bf16_to_f64(wr_bits), bias,
                       k, src, topk_idx=idx)


def tied_router(shape, layer, tied):
    """Router whose rows `tied` are equal and non-negative, and activations
    that are non-negative: the tied experts share the largest logit."""
    _, wr, _ = route_inputs(shape, 0, layer, 1)
    row = (wr[tied[0]].astype(np.uint32) & 0x7FFF).astype(np.uint16)
    for e in tied:
        wr[e] = row
    return wr


@pytest.mark.parametrize("shape,T,tied", [
    (synth.BIG, 1, [7, 300, 450]), (synth.BIG, 3, [7, 300, 450]),
    (synth.BIG, 8, [7, 300, 450]),
    (WIDE, 3, [5, 600, 1000]), (WIDE, 8, [31, 32, 1023]),
])
def test_layer_topk_ties_to_lower_index(shape, T, tied):
    wr = tied_router(shape, 2, tied)
    x, _, _ = route_inputs(shape, 0, 2, T, step=1)
    xpos = (x.astype(np.uint32) & 0x7FFF).astype(np.uint16)   # |x|
    k = shape.k
    out, idx, w, lg = run_layer(shape, xpos, wr, k)
    # the tie is exact in the kernel's own logits, and wins
    assert np.all(lg[:, tied[0]] == lg[:, tied[1]])
    assert np.all(lg[:, tied[0]] == lg[:, tied[2]])
    assert np.all(idx[:, :3] == tied)
    # the whole selection is the oracle's rule on the kernel's logits
    assert np.array_equal(idx, o.topk_select(lg, k))
    # equal logits give equal weights
    assert np.all(w[:, 0] == w[:, 1]) and np.all(w[:, 0] == w[:, 2])
    ref = oracle_out(shape, xpos, wr, k, idx)
    assert row_max_rel(out, ref["out"]) <= TOL


@pytest.mark.parametrize("T", [1, 3, 6])
def test_layer_k_equals_e(T):
    """All 16 experts of the tiny shape chosen: the weights are the
    softmax over all experts (checked against scipy's), in descending
    order with ties to the lower index."""
    from scipy.special import softmax as sp_softmax
    shape = synth.TINY
    k = shape.E
    x, wr, _ = route_inputs(shape, 0, 0, T, step=2)
    out, idx, w, lg = run_layer(shape, x, wr, k)
    for t in range(T):
        assert sorted(idx[t].tolist()) == list(range(shape.E))
    assert np.array_equal(idx, o.topk_select(lg, k))
    p = sp_softmax(lg.astype(np.float64), axis=1)
    assert np.allclose(w, np.take_along_axis(p, idx.astype(np.int64), 1),
                       rtol=2e-6, atol=1e-7)
    ref = oracle_out(shape, x, wr, k, idx)
    assert row_max_rel(out, ref["out"]) <= TOL


def outlier_rows(shape, T, kind):
    x, wr, _ = route_inputs(shape, 0, 0, T, step=4)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    rms = np.sqrt(np.mean(xf * xf, axis=1))
    if kind == "tiny":
        xf[0] *= 2.0 ** -20
    else:
        mag = 2.0 ** (8 if kind == "2^8" else 12)
        for t in range(T):
            xf[t, (977 * t + 5) % shape.H] = mag * rms[t]
    return synth.f32_to_bf16_bits(xf.astype(np.float32)), wr


@pytest.mark.parametrize("T", [1, 3])
@pytest.mark.parametrize("kind", ["2^8", "2^12", "tiny"])
def test_layer_outlier_activations(T, kind):
    shape = synth.BIG
    x, wr = outlier_rows(shape, T, kind)
    out, idx, _, lg = run_layer(shape, x, wr, shape.k)
    assert np.array_equal(idx, o.topk_select(lg, shape.k))
    ref = oracle_out(shape, x, wr, shape.k, idx)
    assert np.isfinite(out).all()
    assert row_max_rel(out, ref["out"]) <= TOL


@pytest.mark.parametrize("T", [1, 3])
@pytest.mark.parametrize("kind", ["2^8", "2^12", "tiny"])
def test_split_decode_outlier_activations(T, kind):
    """The same rows through the split decode kernels (moe_expert_ffn_q,
    T <= 8), which share the activation quantisation."""
    from helpers import run_group, run_route
    shape = synth.BIG
    x, wr = outlier_rows(shape, T, kind)
    idx, _, _ = run_route(x, wr, None, shape.k, T, shape.H, shape.E)
    _, _, _, err, (d_idx, off, pairs, act, na) = run_group(idx, shape.E)
    assert err == 0
    desc = layer_desc(shape, pool_for(shape))
    ws = Ws(moe.moe_ffn_workspace_bytes(T, shape.k, shape.H, shape.F))
    y = torch.full((T * shape.k, shape.H), float("nan"), device="cuda")
    moe.moe_expert_ffn_q(desc, dev(x), T, shape.k, off, pairs, act, na, None,
                         y, ws.t, ws.nbytes)
    assert moe.moe_get_device_status(ws.t) == 0
    src = oracle_experts(shape, 0, 0)
    xd = o.bf16_to_f64(x)
    offs, prs, acts = o.group_pairs(idx, shape.E)
    ref = np.zeros((T * shape.k, shape.H))
    for e in acts:
        pp = prs[offs[e]:offs[e + 1]]
        ref[pp] = o.expert_ffn(xd[pp // shape.k], *src.weights(int(e)))[1]
    assert row_max_rel(y.cpu().numpy(), ref) <= TOL
