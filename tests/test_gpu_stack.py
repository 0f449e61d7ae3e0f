"""GPU: the residual decode stack and the expert-slot cache.

* The routing and FFN halves of a layer reproduce the one-call layer bit
  for bit (one-kernel decode path and the many-token path).
* Each layer of the stack, teacher-forced on the GPU's own layer input and
  routing, matches the fp64 oracle within 2e-3.
* Running the stack through a small slot pool -- misses copied from a
  pinned host store, one copy per expert -- gives output bit-identical to
  the all-resident run, and the miss lists equal the oracle's LRU replay;
  the same holds with the misses handled in-stream (doorbell + stager).
* A device wait on a done word that nothing raises gives up after its
  bound with MOE_ERR_TIMEOUT, and the device stays usable.
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


def _replay_misses(st, routing, L, steps, cap):
    replay = [o.SlotCache(st.shape.E, cap, list(hottest(st, l, cap)))
              for l in range(L)]
    expect, keys = [], set()
    for s in range(steps):
        for l in range(L):
            _, miss, victims = replay[l].resolve(routing[s][l], s + 1)
            expect.append((l, s + 1, miss, victims))
            keys.update((l, e) for e in miss)
    return expect, keys


def test_slot_cache_doorbell_bit_exact_vs_resident():
    L, steps, cap = 3, 8, 32
    st = stack_for(L)
    resident, routing = [], []
    for s in range(steps):
        rec = []
        resident.append(st.run_resident(st.x0(s), record=rec).clone())
        routing.append([i.cpu().numpy() for i in rec])
    expect, keys = _replay_misses(st, routing, L, steps, cap)
    assert keys
    pool = SlotPool(st, [cap] * L, sorted(keys))
    pool.start_stager()
    try:
        outs = [pool.run_doorbell(st.x0(s), s + 1).clone()
                for s in range(steps)]
    finally:
        status, requests, copies = pool.stop_stager()
    for s in range(steps):
        assert torch.equal(outs[s], resident[s]), s
    assert status == 0
    assert int(pool.err.item()) == 0
    assert moe.moe_get_device_status(st.ws) == 0
    n_miss = sum(len(m) for _, _, m, _ in expect)
    assert copies == n_miss
    assert requests == sum(1 for _, _, m, _ in expect if m)
    # every layer posted one request; the last one is done
    sync = pool.sync.cpu().numpy()
    done = int(pool.mailbox[12:16].view(torch.int32).item())
    assert sync[0] == L * steps
    assert max(int(sync[1]), done) == L * steps


def test_wait_done_times_out_and_device_stays_usable():
    mb = torch.zeros(moe.moe_mailbox_bytes(), dtype=torch.uint8).pin_memory()
    sync = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_wait_done(mb, sync, 2000, err)      # request 1 is never done
    torch.cuda.synchronize()
    assert int(err.item()) == moe.MOE_ERR_TIMEOUT
    # the same wait passes at once on a done request: device word ...
    err.zero_()
    sync[1] = 1
    moe.moe_wait_done(mb, sync, 2000, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # ... or the mailbox's done word, written by the host
    sync[0] = 2
    mb[12:16].view(torch.int32)[0] = 2
    moe.moe_wait_done(mb, sync, 2000, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # a mailbox that is not pinned host memory is an argument error
    with pytest.raises(moe.MoeError):
        moe.moe_wait_done(sync, sync, 2000, err)
    # a miss count out of range is a device error, not a post
    n = torch.tensor([99], dtype=torch.int32, device="cuda")
    lst = torch.zeros(30, dtype=torch.int32, device="cuda")
    moe.moe_miss_post(n, lst, lst, 30, 0, 0, mb, sync, err)
    torch.cuda.synchronize()
    assert int(err.item()) == moe.MOE_ERR_DEVICE
    assert int(mb[:4].view(torch.int32).item()) == 0   # nothing posted
    assert int(sync[1].item()) == 3                   # marked done at once
