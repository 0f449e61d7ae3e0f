"""GPU: router + top-k, grouping, slot resolution against the oracle."""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import dev, logit_bound, route_inputs, run_group, run_route, Ws

pytestmark = pytest.mark.gpu


def _check_route(x_bits, wr_bits, bias, k):
    T, H = x_bits.shape
    E = wr_bits.shape[0]
    idx, w, lg = run_route(x_bits, wr_bits, bias, k, T, H, E)
    x = o.bf16_to_f64(x_bits)
    wr = o.bf16_to_f64(wr_bits)
    l64 = o.router_logits(x, wr, bias)
    bound = logit_bound(x, wr, H)
    # fp32 logits within the forward error bound of the fp64 ones
    assert np.all(np.abs(lg - l64) <= bound)
    # selection decided on the kernel's own fp32 logits: bit-exact
    assert np.array_equal(idx, o.topk_select(lg, k))
    # weights: renormalised softmax of those logits
    _, w_ref = o.route(lg.astype(np.float64), k)
    assert np.allclose(w, w_ref, rtol=2e-6, atol=1e-7)
    assert np.allclose(w.sum(1), 1.0, atol=2e-6)
    # against the fp64 selection: equal except within the error bound
    ref_idx = o.topk_select(l64, k)
    near = 0
    for t in range(T):
        if not np.array_equal(idx[t], ref_idx[t]):
            diff = np.nonzero(idx[t] != ref_idx[t])[0]
            a, b = idx[t][diff], ref_idx[t][diff]
            assert np.all(np.abs(l64[t, a] - l64[t, b]) <=
                          bound[t, a] + bound[t, b]), t
            near += 1
    assert near <= max(1, T // 100)
    return idx, w


@pytest.mark.parametrize("T,shape,zipf", [
    (8, synth.TINY, False), (1, synth.BIG, False), (3, synth.BIG, False),
    (3, synth.BIG, True), (8, synth.BIG, True), (300, synth.BIG, True),
    (9536, synth.BIG, True), (40, synth.TINY, False),
])
def test_route_topk_vs_oracle(T, shape, zipf):
    x, wr, bias = route_inputs(shape, 0, 1, T, zipf=zipf)
    _check_route(x, wr, bias, shape.k)


def test_route_ties_go_to_lower_index():
    shape = synth.BIG
    x, wr, _ = route_inputs(shape, 0, 2, 4)
    # duplicate rows: experts 7, 300 and 450 get equal logits; make them top
    wr[300] = wr[7]
    wr[450] = wr[7]
    wr[7] = (wr[7].astype(np.uint32) & 0x7FFF).astype(np.uint16)  # |w|
    wr[300] = wr[7]
    wr[450] = wr[7]
    xpos = (x.astype(np.uint32) & 0x7FFF).astype(np.uint16)          # |x|
    for T_, xx in ((4, xpos), (12, np.tile(xpos, (3, 1)))):
        idx, _ = _check_route(xx, wr, None, 10)
        assert np.all(idx[:, :3] == [7, 300, 450])


def test_route_k_equals_e():
    x, wr, _ = route_inputs(synth.TINY, 0, 0, 5)
    idx, w = _check_route(x, wr, None, 16)
    assert sorted(idx[0].tolist()) == list(range(16))


@pytest.mark.parametrize("T,k,E,zipf", [(3, 10, 512, False), (8, 2, 16, False),
                                        (1, 10, 512, False),
                                        (1000, 10, 512, True),
                                        (2000, 10, 512, True),
                                        (9536, 10, 512, True)])
def test_group_vs_oracle(T, k, E, zipf):
    rng = np.random.default_rng(T)
    if zipf:
        p = synth.zipf_popularity(E)[rng.permutation(E)]
        idx = np.array([rng.choice(E, k, replace=False, p=p) for _ in range(T)])
    else:
        idx = np.array([rng.choice(E, k, replace=False) for _ in range(T)])
    off, pairs, act, err, _ = run_group(idx, E)
    r_off, r_pairs, r_act = o.group_pairs(idx, E)
    assert err == 0
    assert np.array_equal(off, r_off)
    assert np.array_equal(pairs, r_pairs)
    assert np.array_equal(act, r_act)


def test_group_invalid_expert_sets_error_word():
    idx = np.array([[0, 3], [99, 1]], np.int32)
    off, pairs, act, err, _ = run_group(idx, 8)
    assert err == moe.MOE_ERR_DEVICE
    assert off[-1] == 3                  # the bad pair is dropped
    assert act.tolist() == [0, 1, 3]


def test_slot_resolve_replay():
    rng = np.random.default_rng(3)
    E, cap, T, k = 64, 24, 3, 6
    hot = list(rng.permutation(E)[:cap])
    ref = o.SlotCache(E, cap, hot)
    table = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    owner = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    for s, e in enumerate(hot):
        table[e] = s
        owner[s] = e
    last = torch.zeros(cap, dtype=torch.int32, device="cuda")
    blob = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    mexp = torch.empty(T * k, dtype=torch.int32, device="cuda")
    mslot = torch.empty(T * k, dtype=torch.int32, device="cuda")
    nmiss = torch.zeros(1, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    base = 1000
    p = synth.zipf_popularity(E)[rng.permutation(E)]
    for step in range(1, 120):
        chosen = np.array([rng.choice(E, k, replace=False, p=p)
                           for _ in range(T)], np.int32)
        moe.moe_slot_resolve(dev(chosen), T, k, E, table, owner, last, cap,
                             base, step, blob, mexp, mslot, nmiss, err)
        slot_of, misses, victims = ref.resolve(chosen, step)
        torch.cuda.synchronize()
        assert err.item() == 0
        n = int(nmiss.item())
        assert mexp[:n].cpu().tolist() == misses
        assert mslot[:n].cpu().tolist() == victims
        b = blob.cpu().numpy()
        for e, s in slot_of.items():
            assert b[e] == base + s
        assert np.array_equal(table.cpu().numpy(), ref.table)
        assert np.array_equal(owner.cpu().numpy(), ref.owner)
        assert np.array_equal(last.cpu().numpy().astype(np.int64), ref.stamp)


def test_slot_resolve_capacity_error_leaves_state():
    E, cap = 16, 2
    table = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    owner = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    last = torch.zeros(cap, dtype=torch.int32, device="cuda")
    blob = torch.zeros(E, dtype=torch.int32, device="cuda")
    mexp = torch.empty(4, dtype=torch.int32, device="cuda")
    mslot = torch.empty(4, dtype=torch.int32, device="cuda")
    nmiss = torch.zeros(1, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    chosen = dev(np.array([[1, 2, 3]], np.int32))
    moe.moe_slot_resolve(chosen, 1, 3, E, table, owner, last, cap, 0, 1, blob,
                         mexp, mslot, nmiss, err)
    torch.cuda.synchronize()
    assert err.item() == moe.MOE_ERR_CAPACITY
    assert int(nmiss.item()) == 0
    assert (table.cpu() == -1).all() and (owner.cpu() == -1).all()
