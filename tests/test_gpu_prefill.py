"""GPU: the tensor-core prefill path (T > 8) against the fp64 oracle.

Routings are built so that the per-expert token lists cross the 256-row
unit boundary (exactly 256, 257, 512 rows), hit the 16-row MMA granularity
(1, 15, 16, 17 rows) and leave experts empty; the full prefill chunk
(9536 tokens, Zipf-skewed routing) is checked on every row."""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import (TOL, Ws, build_pool, dev, layer_desc, oracle_experts,
                     route_inputs, row_max_rel, run_group)

pytestmark = pytest.mark.gpu

_POOLS = {}


def pool_for(shape, seed=0, layer=0):
    key = (shape, seed, layer)
    if key not in _POOLS:
        _POOLS.clear()
        torch.cuda.empty_cache()
        _POOLS[key] = build_pool(shape, seed, layer)
    return _POOLS[key]


def routing_with_counts(counts: dict, T: int, k: int, E: int, seed: int):
    """topk_idx [T, k] (distinct experts per row) whose per-expert pair
    counts are `counts`; the remaining slots go to experts outside
    `counts`, spread evenly.  Rows are shuffled."""
    rng = np.random.default_rng(seed)
    need = T * k
    named = sum(counts.values())
    assert named <= need
    others = [e for e in range(E) if e not in counts]
    slots = []
    for e, c in counts.items():
        slots += [e] * c
    filler = need - named
    slots += [others[i % len(others)] for i in range(filler)]
    # deal round-robin: slot i -> row i % T, so a row never repeats an
    # expert as long as every expert has at most T pairs
    slots = np.array(slots, np.int32)
    idx = np.empty((T, k), np.int32)
    for i, e in enumerate(slots):
        idx[i % T, i // T] = e
    for r in range(T):
        assert len(set(idx[r])) == k
    idx = idx[rng.permutation(T)]
    return idx


def run_ffn(shape, desc, x_bits, idx, blob_index=None):
    T, k = idx.shape
    _, _, _, err, (d_idx, off, pairs, act, na) = run_group(idx, shape.E)
    assert err == 0
    ws = Ws(moe.moe_ffn_workspace_bytes(T, k, shape.H, shape.F))
    y = torch.full((T * k, shape.H), float("nan"), device="cuda")
    moe.moe_expert_ffn_q(desc, dev(x_bits), T, k, off, pairs, act, na,
                         blob_index, y, ws.t, ws.nbytes)
    st = moe.moe_get_device_status(ws.t)
    return y, st, (off, pairs, act, na, ws)


def oracle_y(shape, x_bits, idx, rows=None):
    src = oracle_experts(shape, 0, 0)
    x = o.bf16_to_f64(x_bits)
    T, k = idx.shape
    off, pairs, act = o.group_pairs(idx, shape.E)
    want = None if rows is None else set(int(r) for r in rows)
    y = np.full((T * k, shape.H), np.nan)
    for e in act:
        pp = pairs[off[e]:off[e + 1]]
        if want is not None:
            pp = np.array([q for q in pp if int(q) in want], np.int64)
            if pp.size == 0:
                continue
        wu, wg, wd = src.weights(int(e))
        y[pp] = o.expert_ffn(x[pp // k], wu, wg, wd)[1]
    return y


def test_tiny_ragged_tiles():
    # tiny shape (Q4 up/gate and down): 16 experts, 2 per token
    shape = synth.TINY
    T = 700
    counts = {0: 256, 1: 257, 2: 1, 3: 15, 4: 16, 5: 17, 6: 512, 7: 255}
    idx = routing_with_counts(counts, T, shape.k, shape.E, seed=1)
    desc = layer_desc(shape, pool_for(shape))
    x, _, _ = route_inputs(shape, 0, 0, T, step=3)
    y, st, _ = run_ffn(shape, desc, x, idx)
    assert st == 0
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    ref = oracle_y(shape, x, idx)
    assert row_max_rel(got, ref) <= TOL


def test_tiny_every_expert_empty_but_one():
    shape = synth.TINY
    T = 300
    idx = np.zeros((T, shape.k), np.int32)
    idx[:, 0] = 9
    idx[:, 1] = 3
    desc = layer_desc(shape, pool_for(shape))
    x, _, _ = route_inputs(shape, 0, 0, T, step=4)
    y, st, _ = run_ffn(shape, desc, x, idx)
    assert st == 0
    ref = oracle_y(shape, x, idx)
    assert row_max_rel(y.cpu().numpy(), ref) <= TOL


def test_big_tile_boundaries():
    # 512-expert shape (SB3 up/gate, NL4 down), 12 experts in use
    shape = synth.BIG
    T = 520
    counts = {5: 256, 77: 257, 300: 1, 301: 15, 302: 16, 303: 17, 510: 512,
              0: 255, 64: 240, 128: 200, 200: 100, 256: 31}
    rest = T * shape.k - sum(counts.values())
    assert rest >= 0
    # fill the remaining slots with 30 more experts
    extra = {e: 0 for e in range(400, 430)}
    for i in range(rest):
        extra[400 + i % 30] += 1
    counts.update(extra)
    idx = routing_with_counts(counts, T, shape.k, shape.E, seed=2)
    desc = layer_desc(shape, pool_for(shape))
    x, _, _ = route_inputs(shape, 0, 0, T, step=5)
    y, st, _ = run_ffn(shape, desc, x, idx)
    assert st == 0
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    # the oracle on the rows of the 12 named experts
    pair_e = idx.reshape(-1)
    rows = np.nonzero(np.isin(pair_e, list(counts.keys())[:12]))[0]
    ref = oracle_y(shape, x, idx, rows=rows)
    assert row_max_rel(got[rows], ref[rows]) <= TOL


def test_up_then_down_matches_ffn():
    shape = synth.TINY
    T = 200
    desc = layer_desc(shape, pool_for(shape))
    x, wr, _ = route_inputs(shape, 0, 0, T, step=6)
    idx = routing_with_counts({1: 150, 2: 100}, T, shape.k, shape.E, seed=3)
    y1, st, (off, pairs, act, na, ws) = run_ffn(shape, desc, x, idx)
    assert st == 0
    y2 = torch.full_like(y1, float("nan"))
    moe.moe_expert_up_q(desc, dev(x), T, shape.k, off, pairs, act, na, None,
                        ws.t, ws.nbytes)
    moe.moe_expert_down_q(desc, T, shape.k, off, pairs, act, na, None, y2,
                          None, None, None, None, ws.t, ws.nbytes)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    # the up/gate GEMM launch alone, on the activations staged above
    y3 = torch.full_like(y1, float("nan"))
    moe.moe_expert_up_gemm_q(desc, T, shape.k, off, pairs, act, na, None,
                             ws.t, ws.nbytes)
    moe.moe_expert_down_q(desc, T, shape.k, off, pairs, act, na, None, y3,
                          None, None, None, None, ws.t, ws.nbytes)
    torch.cuda.synchronize()
    assert torch.equal(y1, y3)
    # decode shapes have no separate GEMM launch
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_expert_up_gemm_q(desc, 4, shape.k, off, pairs, act, na, None,
                                 ws.t, ws.nbytes)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED


def test_prefill_bad_blob_index_sets_error_word():
    shape = synth.TINY
    T = 64
    desc = layer_desc(shape, pool_for(shape))
    x, _, _ = route_inputs(shape, 0, 0, T)
    idx = routing_with_counts({4: 64}, T, shape.k, shape.E, seed=4)
    bi = torch.arange(shape.E, dtype=torch.int32, device="cuda")
    bi[4] = -1
    _, st, _ = run_ffn(shape, desc, x, idx, blob_index=bi)
    assert st == moe.MOE_ERR_DEVICE


def test_prefill_h_overflow_sets_error_word():
    # activations scaled by 2^20: x itself is handled by the per-token
    # power-of-two scale, but h leaves the fp16 range
    shape = synth.TINY
    T = 32
    desc = layer_desc(shape, pool_for(shape))
    x, _, _ = route_inputs(shape, 0, 0, T)
    xf = synth.bf16_bits_to_f32(x) * np.float32(2.0 ** 20)
    xb = synth.f32_to_bf16_bits(xf)
    idx = routing_with_counts({4: 32, 5: 32}, T, shape.k, shape.E, seed=5)
    _, st, _ = run_ffn(shape, desc, xb, idx)
    assert st == moe.MOE_ERR_DEVICE


def test_prefill_layer_full_size_all_rows():
    """The prefill chunk: 9536 tokens, 512 experts top-10, Zipf(1.1)
    routing bias; whole layer through moe_layer_forward, every one of the
    9536 output rows against the oracle (its expert FFNs run in a pool of
    spawned worker processes), and run twice: bit-identical."""
    from oracle_pool import expert_outputs
    shape = synth.BIG
    T = synth.WORKLOADS["prefill"].T
    k, E, H = shape.k, shape.E, shape.H
    desc = layer_desc(shape, pool_for(shape))
    x, wr, bias = route_inputs(shape, 0, 0, T, step=0, zipf=True)
    ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, shape.F))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    lg = torch.empty((T, E), device="cuda")
    out = torch.empty((T, H), device="cuda")
    outs = []
    for _ in range(2):
        moe.moe_layer_forward(desc, dev(x), T, k, dev(wr), dev(bias), None,
                              None, out, None, idx, w, lg, ws.t, ws.nbytes)
        assert moe.moe_get_device_status(ws.t) == 0
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[1])
    got_idx = idx.cpu().numpy()
    # selection is the oracle's rule applied to the kernel's logits
    assert np.array_equal(got_idx, o.topk_select(lg.cpu().numpy(), k))
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    del ws, outs
    # the oracle: routing weights from its fp64 logits on the kernel's
    # selection, every pair's expert FFN, the weighted combine
    logits = o.router_logits(o.bf16_to_f64(x), o.bf16_to_f64(wr), bias)
    p = o.softmax(logits)
    ps = np.take_along_axis(p, got_idx.astype(np.int64), axis=1)
    w_ref = ps / ps.sum(axis=1, keepdims=True)
    y_ref = expert_outputs(shape, 0, 0, x, got_idx)
    ref = o.combine(y_ref, w_ref)
    del y_ref
    assert row_max_rel(got, ref) <= TOL


def test_prefill_past_int32_elements_sampled():
    """70,000 tokens x top-10: y_pairs holds 700,000 x 3072 > 2^31 fp32
    elements and x_g 4.3 GB, so every pair/row index of the prefill path
    needs 64-bit arithmetic.  Sampled tokens against the oracle; the last
    token's rows sit past element 2^31."""
    shape = synth.BIG
    T = 70000
    k, E, H = shape.k, shape.E, shape.H
    assert T * k * H > 2 ** 31
    desc = layer_desc(shape, pool_for(shape))
    x, wr, bias = route_inputs(shape, 0, 0, T, step=9, zipf=True)
    ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, shape.F))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    out = torch.empty((T, H), device="cuda")
    moe.moe_layer_forward(desc, dev(x), T, k, dev(wr), dev(bias), None, None,
                          out, None, idx, w, None, ws.t, ws.nbytes)
    assert moe.moe_get_device_status(ws.t) == 0
    toks = [0, T // 2, T - 2, T - 1]
    got_idx = idx[toks].cpu().numpy()
    src = oracle_experts(shape, 0, 0)
    ref = o.moe_layer(o.bf16_to_f64(x[toks]), o.bf16_to_f64(wr), bias, k,
                      src, topk_idx=got_idx)
    got = out[toks].cpu().numpy()
    assert np.isfinite(got).all()
    assert row_max_rel(got, ref["out"]) <= TOL
    del ws
    torch.cuda.empty_cache()
