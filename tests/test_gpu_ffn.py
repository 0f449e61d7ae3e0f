"""GPU: expert FFN (decode and general paths), combine and whole layers
against the fp64 oracle, on the tiny and the 512-expert decode shapes."""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import (TOL, Ws, build_pool, dev, layer_desc, oracle_experts,
                     route_inputs, row_max_rel, run_group, run_route)

pytestmark = pytest.mark.gpu

_POOLS = {}


def pool_for(shape, seed=0, layer=0):
    key = (shape, seed, layer)
    if key not in _POOLS:
        _POOLS.clear()
        torch.cuda.empty_cache()
        _POOLS[key] = build_pool(shape, seed, layer)
    return _POOLS[key]


def _oracle_y(shape, x_bits, idx, seed=0, layer=0):
    src = oracle_experts(shape, seed, layer)
    x = o.bf16_to_f64(x_bits)
    T, k = idx.shape
    off, pairs, act = o.group_pairs(idx, shape.E)
    y = np.zeros((T * k, shape.H))
    for e in act:
        pp = pairs[off[e]:off[e + 1]]
        wu, wg, wd = src.weights(int(e))
        y[pp] = o.expert_ffn(x[pp // k], wu, wg, wd)[1]
    return y


@pytest.mark.parametrize("shape,T", [
    (synth.TINY, 8), (synth.TINY, 1), (synth.TINY, 5),     # decode path
    (synth.TINY, 12), (synth.TINY, 40),                    # general path
    (synth.BIG, 1), (synth.BIG, 3), (synth.BIG, 8),        # decode path
    (synth.BIG, 9),                                        # general path
])
def test_expert_ffn_vs_oracle(shape, T):
    pool = pool_for(shape)
    desc = layer_desc(shape, pool)
    x, wr, _ = route_inputs(shape, 0, 0, T)
    idx, w, _ = run_route(x, wr, None, shape.k, T, shape.H, shape.E)
    _, _, _, err, (d_idx, off, pairs, act, na) = run_group(idx, shape.E)
    assert err == 0
    ws = Ws(moe.moe_ffn_workspace_bytes(T, shape.k, shape.H, shape.F))
    y = torch.full((T * shape.k, shape.H), float("nan"), device="cuda")
    xd = dev(x)
    moe.moe_expert_ffn_q(desc, xd, T, shape.k, off, pairs, act, na, None, y,
                         ws.t, ws.nbytes)
    assert moe.moe_get_device_status(ws.t) == 0
    y_ref = _oracle_y(shape, x, idx)
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    assert row_max_rel(got, y_ref) <= TOL
    # fused FFN + combine equals FFN then combine, bit for bit
    wd = dev(w)
    out1 = torch.empty((T, shape.H), device="cuda")
    out2 = torch.empty((T, shape.H), device="cuda")
    moe.moe_combine(y, wd, T, shape.k, shape.H, None, out1, None)
    moe.moe_expert_ffn_combine_q(desc, xd, T, shape.k, off, pairs, act, na,
                                 None, wd, None, out2, None, ws.t, ws.nbytes)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)
    ref_out = o.combine(y_ref, w.astype(np.float64))
    assert row_max_rel(out2.cpu().numpy(), ref_out) <= TOL


# 1024 experts top-8 (the wide top-k of the one-kernel layer: 32 keys per
# lane), SB3 up/gate and NL4 down at a small hidden size
WIDE = synth.LayerShape(H=512, F=256, E=1024, k=8,
                        fmt_up_gate=synth.SB3_256, fmt_down=synth.NL4_B32,
                        d_up_gate=(0.002, 0.01), d_down=(0.002, 0.01))


# 1024 experts top-20: 8 tokens make 160 pairs, more than the SM count and
# the one-kernel layer's pair limit, so the layer takes the general path
WIDE20 = synth.LayerShape(H=512, F=256, E=1024, k=20,
                          fmt_up_gate=synth.SB3_256, fmt_down=synth.NL4_B32,
                          d_up_gate=(0.002, 0.01), d_down=(0.002, 0.01))


@pytest.mark.parametrize("shape,T,zipf", [
    (synth.TINY, 8, False), (synth.BIG, 1, False), (synth.BIG, 3, False),
    (synth.BIG, 3, True), (synth.TINY, 16, False),
    (synth.BIG, 2, False), (synth.BIG, 4, False), (synth.BIG, 5, False),
    (synth.BIG, 8, True),
    (WIDE, 3, False), (WIDE, 7, True), (WIDE20, 8, False),
])
def test_layer_forward_vs_oracle(shape, T, zipf):
    pool = pool_for(shape)
    desc = layer_desc(shape, pool)
    x, wr, bias = route_inputs(shape, 0, 0, T, step=7, zipf=zipf)
    k, E, H = shape.k, shape.E, shape.H
    ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, shape.F))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    lg = torch.empty((T, E), device="cuda")
    torch.manual_seed(T)
    res = torch.randn((T, H), device="cuda") * 0.5
    out = torch.empty((T, H), device="cuda")
    outb = torch.empty((T, H), dtype=torch.int16, device="cuda")
    bd = dev(bias) if bias is not None else None
    outs = []
    for _ in range(2):
        moe.moe_layer_forward(desc, dev(x), T, k, dev(wr), bd, None, res, out,
                              outb, idx, w, lg, ws.t, ws.nbytes)
        assert moe.moe_get_device_status(ws.t) == 0
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1])           # deterministic
    gi = idx.cpu().numpy()
    assert np.array_equal(gi, o.topk_select(lg.cpu().numpy(), k))
    src = oracle_experts(shape, 0, 0)
    ref = o.moe_layer(o.bf16_to_f64(x), o.bf16_to_f64(wr), bias, k, src,
                      residual=None, topk_idx=gi)
    got = out.cpu().numpy().astype(np.float64) - res.cpu().numpy()
    assert row_max_rel(got, ref["out"]) <= TOL
    # bf16 copy is the rounding of the fp32 output
    ob = outb.cpu().numpy().view(np.uint16)
    assert np.array_equal(ob, o.f64_to_bf16_bits(out.cpu().numpy()))


def test_ffn_rejects_small_workspace():
    shape = synth.TINY
    pool = pool_for(shape)
    desc = layer_desc(shape, pool)
    z = torch.zeros(64, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_expert_ffn_q(desc, z, 2, 2, z, z, z, z, None, z, z, 16)
    assert ei.value.code == moe.MOE_ERR_WORKSPACE


def test_bad_blob_index_sets_error_word():
    shape = synth.TINY
    pool = pool_for(shape)
    desc = layer_desc(shape, pool)
    T = 4
    x, wr, _ = route_inputs(shape, 0, 0, T)
    idx, w, _ = run_route(x, wr, None, shape.k, T, shape.H, shape.E)
    _, _, _, _, (d_idx, off, pairs, act, na) = run_group(idx, shape.E)
    bi = torch.arange(shape.E, dtype=torch.int32, device="cuda")
    bi[int(idx[0, 0])] = -1
    ws = Ws(moe.moe_ffn_workspace_bytes(T, shape.k, shape.H, shape.F))
    y = torch.zeros((T * shape.k, shape.H), device="cuda")
    moe.moe_expert_ffn_q(desc, dev(x), T, shape.k, off, pairs, act, na, bi, y,
                         ws.t, ws.nbytes)
    assert moe.moe_get_device_status(ws.t) == moe.MOE_ERR_DEVICE


@pytest.mark.parametrize("T,k,H", [(7, 10, 3072), (5, 3, 20), (3, 2, 6)])
def test_combine_paths_bit_identical(T, k, H):
    """moe_combine on 16-byte aligned rows (four columns per thread) and on
    misaligned views (one column per thread) gives the same bits, equal to
    the oracle's weighted sum; residual and bf16 output included."""
    g = torch.Generator().manual_seed(T * 100 + H)
    yh = torch.randn((T * k * H + 4,), generator=g)
    wh = torch.rand((T, k), generator=g)
    rh = torch.randn((T * H + 4,), generator=g)
    y_al = yh[:T * k * H].cuda().view(T * k, H)
    r_al = rh[:T * H].cuda().view(T, H)
    ybuf = torch.empty(T * k * H + 1, device="cuda")
    ybuf[1:].copy_(yh[:T * k * H])
    rbuf = torch.empty(T * H + 1, device="cuda")
    rbuf[1:].copy_(rh[:T * H])
    wd = wh.cuda()
    outs = []
    for y, r, off in ((y_al, r_al, 0), (ybuf[1:].view(T * k, H),
                                        rbuf[1:].view(T, H), 1)):
        ob = torch.empty(T * H + 1, device="cuda")
        out = ob[off:off + T * H].view(T, H)
        bb = torch.empty(T * H + 1, dtype=torch.int16, device="cuda")
        outb = bb[off:off + T * H].view(T, H)
        moe.moe_combine(y, wd, T, k, H, r, out, outb)
        torch.cuda.synchronize()
        outs.append((out.clone(), outb.clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    ref = o.combine(yh[:T * k * H].view(T * k, H).double().numpy(),
                    wh.double().numpy(),
                    rh[:T * H].view(T, H).double().numpy())
    assert row_max_rel(outs[0][0].cpu().numpy(), ref) <= 1e-5
