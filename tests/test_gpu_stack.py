"""GPU: the residual decode stack and the expert-slot cache.

* The routing and FFN halves of a layer reproduce the one-call layer bit
  for bit (one-kernel decode path and the many-token path).
* Each layer of the stack, teacher-forced on the GPU's own layer input and
  routing, matches the fp64 oracle within 2e-3.
* Running the stack through a small slot pool -- misses copied from a
  pinned host store, one copy per expert -- gives output bit-identical to
  the all-resident run, and the miss lists equal the oracle's LRU replay.
"""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import TOL, dev, oracle_experts, row_max_rel
from synth.stack import SlotPool, Stack, hottest

pytestmark = pytest.mark.gpu

_POOLS = []


def stack_for(L, T=3):
    """A stack of L layers with T tokens; the device pools of the first
    layers are built once and shared."""
    st = Stack(L, synth.BIG, seed=0, T=T, build_pools=False)
    from synth.pools import build_pool, layer_desc
    while len(_POOLS) < L:
        _POOLS.append(build_pool(synth.BIG, 0, len(_POOLS)))
    st.pools = _POOLS[:L]
    st.descs = [layer_desc(synth.BIG, p) for p in st.pools]
    return st


@pytest.mark.parametrize("T", [3, 1, 12])
def test_halves_equal_one_call(T):
    st = stack_for(2, T)
    shp = st.shape
    r_a = st.x0(5)
    r_b = r_a.clone()
    st.run_resident(r_a)
    idx = torch.empty((T, shp.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, shp.k), device="cuda")
    for l in range(st.L):
        moe.moe_layer_route_residual(st.descs[l], r_b, T, shp.k, st.wr[l],
                                     st.bias[l], idx, w, None, st.ws,
                                     st.ws_bytes)
        moe.moe_layer_ffn_residual(st.descs[l], r_b, T, shp.k, idx, w, None,
                                   r_b, None, st.ws, st.ws_bytes)
    assert moe.moe_get_device_status(st.ws) == 0
    assert torch.equal(r_a, r_b)
    assert torch.isfinite(r_a).all()


def test_stack_teacher_forced_vs_oracle():
    st = stack_for(3)
    shp = st.shape
    r = st.x0(2)
    for l in range(st.L):
        r_in = r.clone()
        lg = torch.empty((st.T, shp.E), device="cuda")
        moe.moe_layer_forward_residual(st.descs[l], r, st.T, shp.k, st.wr[l],
                                       st.bias[l], None, r, None, st.idx,
                                       st.w, lg, st.ws, st.ws_bytes)
        assert moe.moe_get_device_status(st.ws) == 0
        gi = st.idx.cpu().numpy()
        # selection = the oracle's rule on the kernel's own logits
        assert np.array_equal(gi, o.topk_select(lg.cpu().numpy(), shp.k))
        x = o.bf16_to_f64(o.f64_to_bf16_bits(
            o.rmsnorm(r_in.cpu().numpy().astype(np.float64))))
        ref = o.moe_layer(x, o.bf16_to_f64(synth.gen_router(0, l, shp.E,
                                                            shp.H)),
                          st.bias_np[l], shp.k, oracle_experts(shp, 0, l),
                          topk_idx=gi)
        got = (r - r_in).cpu().numpy().astype(np.float64)
        assert row_max_rel(got, ref["out"]) <= TOL, l


def test_slot_cache_bit_exact_vs_resident():
    L, steps, cap = 3, 8, 32   # cap >= T*k: one step fits; misses still occur
    st = stack_for(L)
    shp = st.shape
    # the all-resident run, recording each layer's routing
    resident, routing = [], []
    for s in range(steps):
        rec = []
        resident.append(st.run_resident(st.x0(s), record=rec).clone())
        routing.append([i.cpu().numpy() for i in rec])
    # the oracle's LRU replay on that routing gives every miss
    replay = [o.SlotCache(shp.E, cap, list(hottest(st, l, cap)))
              for l in range(L)]
    expect, keys = [], set()
    for s in range(steps):
        for l in range(L):
            _, miss, victims = replay[l].resolve(routing[s][l], s + 1)
            expect.append((l, s + 1, miss, victims))
            keys.update((l, e) for e in miss)
    assert keys, "the pool is large enough to hide every miss"
    pool = SlotPool(st, [cap] * L, sorted(keys))
    log = []
    for s in range(steps):
        r = pool.run(st.x0(s), s + 1, log)
        assert torch.equal(r, resident[s]), s
    torch.cuda.synchronize()
    assert int(pool.err.item()) == 0
    assert moe.moe_get_device_status(st.ws) == 0
    assert log == expect
    assert pool.misses == sum(len(m) for _, _, m, _ in expect)
