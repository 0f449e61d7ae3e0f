"""GPU: prefill through the expert-slot pool (the prefill prefetch of the
"Avalon" README's feature list: a few slots taken over from the expert
cache stream the missing experts, cached experts are used in their slots).

* moe_group_subset restricts a grouping to a list of experts exactly (the
  oracle's grouping of the same routing, filtered);
* a prefill chunk through one layer's partition -- resident experts in
  place, the others streamed from a pinned host store through borrowed
  slots in waves, copies overlapping the previous wave's compute -- gives
  output bit-identical to the all-resident layer, call after call.
"""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import Ws, build_pool, dev, route_inputs, run_group
from synth.prefill_slots import Partition, PrefillSlots

pytestmark = pytest.mark.gpu


def test_group_subset_matches_filtered_oracle_grouping():
    rng = np.random.default_rng(3)
    T, k, E = 700, 10, 512
    idx = np.array([rng.choice(E, k, replace=False) for _ in range(T)])
    off, pairs, act, err, (d_idx, d_off, d_pairs, d_act, d_na) = \
        run_group(idx, E)
    assert err == 0
    for sel in (act[::3], act[:1], np.array([], np.int64), act):
        lst = torch.tensor(np.asarray(sel, np.int32), device="cuda")
        if lst.numel() == 0:
            lst = torch.zeros(1, dtype=torch.int32, device="cuda")
        s_off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        s_pairs = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
        s_act = torch.empty(E, dtype=torch.int32, device="cuda")
        s_na = torch.empty(1, dtype=torch.int32, device="cuda")
        e_word = torch.zeros(1, dtype=torch.int32, device="cuda")
        moe.moe_group_subset(d_off, d_pairs, E, lst, len(sel), s_off,
                             s_pairs, s_act, s_na, e_word)
        torch.cuda.synchronize()
        assert int(e_word.item()) == 0
        r_off, r_pairs, r_act = o.group_pairs(idx, E)
        keep = np.isin(np.arange(E), sel)
        cnt = np.where(keep, np.diff(r_off), 0)
        want_off = np.concatenate([[0], np.cumsum(cnt)])
        want_pairs = np.concatenate(
            [r_pairs[r_off[e]:r_off[e + 1]] for e in range(E) if keep[e]] +
            [np.zeros(0, np.int32)])
        n = int(want_off[-1])
        assert np.array_equal(s_off.cpu().numpy(), want_off)
        assert np.array_equal(s_pairs.cpu().numpy()[:n], want_pairs)
        assert np.array_equal(s_act.cpu().numpy()[:int(s_na.item())],
                              np.sort(np.asarray(sel)))


@pytest.mark.parametrize("T,cap,borrow", [(2000, 92, 8), (300, 60, 4)])
def test_prefill_through_slots_bit_exact_vs_resident(T, cap, borrow):
    shape = synth.BIG
    k, E, H = shape.k, shape.E, shape.H
    pool = build_pool(shape, 0, 0)
    from synth.pools import layer_desc
    desc = layer_desc(shape, pool)
    _, rank = synth.gen_zipf_bias(0, 0, E)
    part = Partition(shape, pool, synth.hottest_experts(rank, cap), cap)
    # pinned host store of every expert's blob
    blob = shape.blob_bytes
    store = torch.empty((E, blob), dtype=torch.uint8).pin_memory()
    for e in range(E):
        store[e].copy_(pool[e * shape.blob_stride:e * shape.blob_stride + blob])
    ps = PrefillSlots(shape, part, store, {e: e for e in range(E)}, T,
                      borrow=borrow)
    for step in (0, 1):
        x, wr, bias = route_inputs(shape, 0, 0, T, step=step, zipf=True)
        xd, wd, bd = dev(x), dev(wr), dev(bias)
        ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, shape.F))
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), device="cuda")
        ref = torch.empty((T, H), device="cuda")
        moe.moe_layer_forward(desc, xd, T, k, wd, bd, None, None, ref, None,
                              idx, w, None, ws.t, ws.nbytes)
        assert moe.moe_get_device_status(ws.t) == 0
        out = torch.full((T, H), float("nan"), device="cuda")
        stats = ps.forward(xd, wd, bd, out)
        torch.cuda.synchronize()
        assert stats["hits"] > 0 and stats["misses"] > 0
        assert stats["hits"] + stats["misses"] == stats["chosen"]
        assert int(ps.err.item()) == 0
        assert moe.moe_get_device_status(ps.fws) == 0
        assert torch.equal(out, ref), step
    del ps, part, store, pool
    torch.cuda.empty_cache()
