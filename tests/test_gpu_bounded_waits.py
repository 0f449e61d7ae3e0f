"""GPU: a bounded device wait that runs out.

Every wait of the one-kernel decode layer (grid barriers, mbarrier phases,
completion counters) gives up after 0.5 s of %globaltimer and sets
MOE_ERR_TIMEOUT in the device error word, so a launch always ends and the
context stays usable.  The test makes the first grid barrier unreachable by
planting a large negative value in its arrival counter (a count that no
arrival can complete -- the failure is made on the host, nothing faults):
the launch must end with MOE_ERR_TIMEOUT, its last block must re-arm the
counters, and the next call on the same workspace must give exactly the
result of a clean call.
"""
import numpy as np
import pytest
import torch

import synth
import quantized_moe_expert_02_b200 as moe
from helpers import Ws, build_pool, dev, layer_desc, route_inputs

pytestmark = pytest.mark.gpu


def _r256(n):
    return (n + 255) // 256 * 256


def fused_offset(T, k, E, H, F):
    """Byte offset of the one-kernel layer's own region (its grid-barrier
    counter is the first int32) in a moe_layer_forward workspace: the
    region is the last non-empty one for T <= 8, of the size below."""
    P = T * k
    fused = 1024 + _r256(P * F * 4) + _r256(P * 4) + _r256(P * H * 4)
    return moe.moe_layer_workspace_bytes(T, k, E, H, F) - _r256(fused)


def test_layer_grid_barrier_timeout_is_reported_and_recovers():
    shape = synth.BIG
    T, k, E, H, F = 3, shape.k, shape.E, shape.H, shape.F
    pool = build_pool(shape, 0, 0)
    desc = layer_desc(shape, pool)
    x, wr, _ = route_inputs(shape, 0, 0, T, step=3)
    xd, wd = dev(x), dev(wr)
    ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, F))
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    out = torch.empty((T, H), device="cuda")

    def call():
        moe.moe_layer_forward(desc, xd, T, k, wd, None, None, None, out,
                              None, idx, w, None, ws.t, ws.nbytes)

    call()
    assert moe.moe_get_device_status(ws.t) == 0
    ref = out.clone()
    off = fused_offset(T, k, E, H, F)
    bar = ws.t[off:off + 8].view(torch.int32)
    assert bar.tolist() == [0, 0]        # re-armed after a clean call
    bar[0] = -(1 << 30)                  # barrier 1 can never complete
    out.fill_(float("nan"))
    call()
    assert moe.moe_get_device_status(ws.t) == moe.MOE_ERR_TIMEOUT
    assert bar.tolist() == [0, 0]        # the last block re-armed them
    call()
    assert moe.moe_get_device_status(ws.t) == 0
    assert torch.equal(out, ref)
    del pool
    torch.cuda.empty_cache()


def test_staged_pull_wait_timeout_is_reported_and_recovers():
    """The wait of the staged FFN (moe_layer_ffn_residual_staged) for a
    missed expert's blob: its ready counter is planted with a value that the
    blocks' arrivals cannot bring up to the grid size, so the producers'
    bounded waits run out -- MOE_ERR_TIMEOUT, counters re-armed, and the
    pulls themselves complete: the plain FFN half on the same routing then
    gives the resident result bit for bit."""
    from synth.stack import SlotPool, Stack
    shape = synth.BIG
    T, k, E, H, F = 3, shape.k, shape.E, shape.H, shape.F
    st = Stack(1, shape, seed=0, T=T)
    ref = st.run_resident(st.x0(0)).clone()
    # the first step's misses with a 32-slot partition
    disc = SlotPool(st, [32], None)
    disc.run(st.x0(0), 1)
    keys = sorted(disc.seen_keys)
    del disc
    assert keys
    pool = SlotPool(st, [32], keys)
    pool.start_staging()
    r = st.x0(0)
    r_in = r.clone()
    moe.moe_layer_route_residual(pool.descs[0], r, T, k, st.wr[0], st.bias[0],
                                 st.idx, st.w, None, st.ws, st.ws_bytes)
    moe.moe_slot_resolve_dev(st.idx, T, k, E, pool.table[0], pool.owner[0],
                             pool.last[0], 32, 0, pool.stamps.data_ptr(),
                             pool.blob_index, pool.mexp, pool.mslot,
                             pool.nmiss, pool.err)
    assert int(pool.nmiss.item()) > 0
    off = fused_offset(T, k, E, H, F)
    ready = st.ws[off + 512:off + 516].view(torch.int32)
    assert int(ready.item()) == 0
    ready[0] = -(1 << 30)
    moe.moe_layer_ffn_residual_staged(
        pool.descs[0], r, T, k, st.idx, st.w, pool.blob_index, r, None,
        pool.nmiss, pool.mexp, pool.mslot, 0, 1, pool.table_dev, 0, 32,
        pool.n_slots, st.ws, st.ws_bytes)
    assert moe.moe_get_device_status(st.ws) == moe.MOE_ERR_TIMEOUT
    assert int(ready.item()) == 0          # re-armed by the last block
    r2 = r_in.clone()
    moe.moe_layer_ffn_residual(pool.descs[0], r2, T, k, st.idx, st.w,
                               pool.blob_index, r2, None, st.ws, st.ws_bytes)
    assert moe.moe_get_device_status(st.ws) == 0
    assert torch.equal(r2, ref)
    del pool, st
    torch.cuda.empty_cache()
