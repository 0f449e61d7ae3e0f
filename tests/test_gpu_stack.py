"""GPU: the residual decode stack and the expert-slot cache.

* The routing and FFN halves of a layer reproduce the one-call layer bit
  for bit (one-kernel decode path and the many-token path).
* Each layer of the stack, teacher-forced on the GPU's own layer input and
  routing, matches the fp64 oracle within 2e-3; run free, the stack's
  accumulated update stays within depth x 2e-3 of the free-running oracle
  while the routing agrees (the drift is reported).
* Running the stack through a small slot pool -- misses copied from a
  pinned host store, one copy per expert -- gives output bit-identical to
  the all-resident run, and the miss lists equal the oracle's LRU replay;
  the same holds with the misses pulled from the host store on the stream
  (no host round trip per layer), eagerly and as one CUDA graph per step,
  and at the workload's real shape (48 layers, 240 / 92 / 60 slots).
* The in-stream copy moves blobs byte for byte, rejects host memory that is
  not mapped pinned memory on the host, and reports a missing host copy or
  a bad miss count in the device error word.
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


def test_stack_free_running_drift():
    """The stack run free on the GPU against the fp64 oracle run free on its
    own outputs (its own routing too): while the routing agrees layer by
    layer, the accumulated update r - r0 stays within the per-layer bound
    times the depth; the drift is reported either way."""
    st = stack_for(3)
    shp = st.shape
    r0 = st.x0(4)
    rec = []
    r_gpu = st.run_resident(r0.clone(), record=rec)
    assert moe.moe_get_device_status(st.ws) == 0
    r = r0.cpu().numpy().astype(np.float64)
    same = True
    for l in range(st.L):
        x = o.bf16_to_f64(o.f64_to_bf16_bits(o.rmsnorm(r)))
        res = o.moe_layer(x, o.bf16_to_f64(synth.gen_router(0, l, shp.E,
                                                            shp.H)),
                          st.bias_np[l], shp.k, oracle_experts(shp, 0, l))
        same &= bool(np.array_equal(np.sort(res["topk_idx"], axis=1),
                                    np.sort(rec[l].cpu().numpy(), axis=1)))
        r = r + res["out"]
    r0n = r0.cpu().numpy().astype(np.float64)
    drift = row_max_rel(r_gpu.cpu().numpy().astype(np.float64) - r0n,
                        r - r0n)
    print(f"free-running drift after {st.L} layers: {drift:.2e} "
          f"(routing {'identical' if same else 'differs'})")
    assert np.isfinite(drift)
    if same:
        assert drift <= st.L * TOL


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


def test_slot_cache_in_stream_staging_bit_exact_vs_resident():
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
    pool.start_staging()
    outs = [pool.run_staged(st.x0(s)).clone() for s in range(steps)]
    for s in range(steps):
        assert torch.equal(outs[s], resident[s]), s
    assert int(pool.err.item()) == 0
    assert moe.moe_get_device_status(st.ws) == 0
    # the slot tables end where the host-round-trip run ends (host stamps
    # = step numbers; the device counters reach the same values)
    ref = SlotPool(st, [cap] * L, sorted(keys))
    for s in range(steps):
        ref.run(st.x0(s), s + 1)
    for l in range(L):
        assert torch.equal(pool.table[l], ref.table[l])
        assert torch.equal(pool.owner[l], ref.owner[l])
        assert torch.equal(pool.last[l], ref.last[l])
    assert pool.stamps.tolist() == [steps] * L


def test_slot_cache_step_as_one_graph_bit_exact():
    """The slot-cache step (route, device-stamped resolve, in-stream pull
    and FFN of every layer) captured once as one CUDA graph and replayed
    once per step: bit-identical to the all-resident run on every step,
    slot state equal to the eager run's."""
    L, steps, cap = 3, 8, 32
    st = stack_for(L)
    resident, routing = [], []
    for s in range(steps):
        rec = []
        resident.append(st.run_resident(st.x0(s), record=rec).clone())
        routing.append([i.cpu().numpy() for i in rec])
    expect, keys = _replay_misses(st, routing, L, steps, cap)
    pool = SlotPool(st, [cap] * L, sorted(keys))
    pool.start_staging()
    x_in = st.x0(0)
    r = torch.empty_like(x_in)
    # capturing records the launches without running them
    g = pool.capture_step(x_in, r)
    torch.cuda.synchronize()
    assert pool.stamps.tolist() == [0] * L
    for s in range(steps):
        x_in.copy_(st.x0(s))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(r, resident[s]), s
    assert int(pool.err.item()) == 0
    assert moe.moe_get_device_status(st.ws) == 0
    eager = SlotPool(st, [cap] * L, sorted(keys))
    eager.start_staging()
    for s in range(steps):
        eager.run_staged(st.x0(s))
    for l in range(L):
        assert torch.equal(pool.table[l], eager.table[l])
        assert torch.equal(pool.last[l], eager.last[l])
    del g


def test_slot_cache_fused_staging_bit_exact():
    """The pull inside the FFN launch (moe_layer_ffn_residual_staged: the
    misses computed last, their blobs copied by every block while the hits
    compute): bit-identical to the resident run, eagerly and as one graph
    per step, with the slot state of the separate-pull run."""
    L, steps, cap = 3, 8, 32
    st = stack_for(L)
    resident, routing = [], []
    for s in range(steps):
        rec = []
        resident.append(st.run_resident(st.x0(s), record=rec).clone())
        routing.append([i.cpu().numpy() for i in rec])
    expect, keys = _replay_misses(st, routing, L, steps, cap)
    assert keys
    fused = SlotPool(st, [cap] * L, sorted(keys))
    fused.start_staging()
    for s in range(steps):
        r = fused.run_staged(st.x0(s), fused=True)
        assert torch.equal(r, resident[s]), s
    assert int(fused.err.item()) == 0
    assert moe.moe_get_device_status(st.ws) == 0
    ref = SlotPool(st, [cap] * L, sorted(keys))
    ref.start_staging()
    for s in range(steps):
        ref.run_staged(st.x0(s))
    for l in range(L):
        assert torch.equal(fused.table[l], ref.table[l])
        assert torch.equal(fused.last[l], ref.last[l])
    # one graph per step
    fused.reset()
    x_in = st.x0(0)
    r = torch.empty_like(x_in)
    g = fused.capture_step(x_in, r, fused=True)
    for s in range(steps):
        x_in.copy_(st.x0(s))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(r, resident[s]), s
    assert moe.moe_get_device_status(st.ws) == 0
    del g


def test_slot_cache_full_capacities_48_layers():
    """The slot-cache workload at its real shape: 48 layers, 240 / 92 / 60
    slots per layer, Zipf-hot initial fill, 3 tokens per step.  Misses
    copied after a host round trip (from the resident pools) and, in a
    second pool, pulled in-stream from a pinned host store by one graph
    replay per step: both bit-identical to the all-resident run on every
    step; the miss lists and victims equal the oracle's LRU replay."""
    L, steps = 48, 4
    st = stack_for(L)
    caps = [synth.slot_capacity(l) for l in range(L)]
    assert caps[0] == 240 and caps[5] == 92 and caps[47] == 60
    resident, routing = [], []
    for s in range(steps):
        rec = []
        resident.append(st.run_resident(st.x0(s), record=rec).clone())
        routing.append([i.cpu().numpy() for i in rec])
    replay = [o.SlotCache(st.shape.E, caps[l], list(hottest(st, l, caps[l])))
              for l in range(L)]
    expect, keys = [], set()
    for s in range(steps):
        for l in range(L):
            _, miss, victims = replay[l].resolve(routing[s][l], s + 1)
            expect.append((l, s + 1, miss, victims))
            keys.update((l, e) for e in miss)
    assert keys
    disc = SlotPool(st, caps, None)          # misses copied device to device
    log = []
    for s in range(steps):
        r = disc.run(st.x0(s), s + 1, log)
        assert torch.equal(r, resident[s]), s
    assert log == expect
    assert int(disc.err.item()) == 0
    del disc
    torch.cuda.empty_cache()
    pool = SlotPool(st, caps, sorted(keys))  # pinned host store
    pool.start_staging()
    x_in = st.x0(0)
    r = torch.empty_like(x_in)
    g = pool.capture_step(x_in, r)
    for s in range(steps):
        x_in.copy_(st.x0(s))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(r, resident[s]), s
    assert int(pool.err.item()) == 0
    assert moe.moe_get_device_status(st.ws) == 0
    del g
    # the same with the pulls inside the FFN launches
    pool.reset()
    g = pool.capture_step(x_in, r, fused=True)
    for s in range(steps):
        x_in.copy_(st.x0(s))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(r, resident[s]), s
    assert int(pool.err.item()) == 0
    assert moe.moe_get_device_status(st.ws) == 0
    del g, pool
    torch.cuda.empty_cache()


def test_stage_misses_copies_and_errors():
    E, L, blob, stride, slots = 4, 2, 4096 + 256, 4608, 6
    host = torch.randint(0, 256, (L * E, blob), dtype=torch.uint8)
    host = host.pin_memory()
    table_host = [host[i].data_ptr() for i in range(L * E)]
    table_host[1 * E + 3] = 0                      # (layer 1, expert 3) absent
    table = torch.zeros(L * E, dtype=torch.int64, device="cuda")
    moe.moe_stage_table(table_host, table)
    pool = torch.zeros(slots * stride, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mexp = torch.tensor([2, 0, 3], dtype=torch.int32, device="cuda")
    mslot = torch.tensor([1, 0, 2], dtype=torch.int32, device="cuda")
    n = torch.tensor([3], dtype=torch.int32, device="cuda")
    # layer 1, partition of 3 slots at base 3: blobs (1,2) -> slot 4,
    # (1,0) -> slot 3, (1,3) absent
    moe.moe_stage_misses(n, mexp, mslot, 3, 1, L, E, table, pool, 3, 3,
                         slots, stride, blob, err)
    torch.cuda.synchronize()
    assert int(err.item()) == moe.MOE_ERR_CAPACITY
    got = pool.cpu()
    assert torch.equal(got[4 * stride:4 * stride + blob], host[1 * E + 2])
    assert torch.equal(got[3 * stride:3 * stride + blob], host[1 * E + 0])
    assert int(got[5 * stride:6 * stride].sum()) == 0     # skipped
    assert int(got[:3 * stride].sum()) == 0               # untouched
    # a miss count out of range: device error, nothing copied
    err.zero_()
    pool.zero_()
    n[0] = 7
    moe.moe_stage_misses(n, mexp, mslot, 3, 0, L, E, table, pool, 0, 3,
                         slots, stride, blob, err)
    torch.cuda.synchronize()
    assert int(err.item()) == moe.MOE_ERR_DEVICE
    assert int(pool.sum()) == 0
    # a victim slot inside the pool but outside the layer's partition (a
    # corrupted miss list): that blob is skipped, the other one copied
    err.zero_()
    n[0] = 2
    bad = torch.tensor([3, 1, 0], dtype=torch.int32, device="cuda")
    moe.moe_stage_misses(n, mexp, bad, 3, 0, L, E, table, pool, 0, 3, slots,
                         stride, blob, err)
    torch.cuda.synchronize()
    assert int(err.item()) == moe.MOE_ERR_CAPACITY
    got = pool.cpu()
    assert int(got[3 * stride:4 * stride].sum()) == 0     # not overwritten
    assert torch.equal(got[1 * stride:1 * stride + blob], host[0 * E + 0])
    # host memory that is not pinned, and a layer outside the table, are
    # argument errors found on the host
    plain = torch.zeros(blob, dtype=torch.uint8)
    with pytest.raises(moe.MoeError):
        moe.moe_stage_table([plain.data_ptr()], table)
    with pytest.raises(moe.MoeError):
        moe.moe_stage_misses(n, mexp, mslot, 3, L, L, E, table, pool, 0, 3,
                             slots, stride, blob, err)
    with pytest.raises(moe.MoeError):        # partition past the pool
        moe.moe_stage_misses(n, mexp, mslot, 3, 0, L, E, table, pool, 4, 3,
                             slots, stride, blob, err)
