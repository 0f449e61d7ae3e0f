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
