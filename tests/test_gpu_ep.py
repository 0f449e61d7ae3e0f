"""GPU: the expert-parallel layer (quantized_moe_expert_02_b200.ep) end to
end on one GPU -- a one-rank NCCL group, so the dispatch and combine go
through real NCCL all-to-alls (to the rank itself) around the library's
routing, expert FFN and combine.  Multi-rank bookkeeping is covered by the
gloo test on CPU; every GPU run here has one GPU."""
import socket

import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import (TOL, Ws, build_pool, dev, layer_desc, oracle_experts,
                     route_inputs, row_max_rel)

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_layer_one_rank_nccl():
    import datetime
    import torch.distributed as dist
    from quantized_moe_expert_02_b200.ep import (ExpertParallel,
                                                 ExpertParallelLayer)
    shape = synth.BIG
    k, E, H = shape.k, shape.E, shape.H
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:"
                            f"{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=120))
    try:
        pool = build_pool(shape, 0, 0)
        ep = ExpertParallel(E, k)
        assert ep.n_local == E
        layer, first = None, {}
        # one layer object for all calls: its reused workspaces change
        # layout between the decode and prefill row counts and back
        for T in (3, 40, 3, 40):
            x, wr, _ = route_inputs(shape, 0, 0, T, step=8)
            if layer is None:
                layer = ExpertParallelLayer(ep, shape, pool, dev(wr))
            out = torch.full((T, H), float("nan"), device="cuda")
            idx, w = layer.forward(dev(x), out)
            torch.cuda.synchronize()
            assert layer.last_rows == T * k
            if T in first:
                assert torch.equal(out, first[T])
                continue
            first[T] = out.clone()
            gi = idx.cpu().numpy()
            ref = o.moe_layer(o.bf16_to_f64(x), o.bf16_to_f64(wr), None, k,
                              oracle_experts(shape, 0, 0), topk_idx=gi)
            assert row_max_rel(out.cpu().numpy(), ref["out"]) <= TOL
            if T > 8:
                # the received rows take the same prefill path as the
                # one-GPU layer: bit-identical
                desc = layer_desc(shape, pool)
                ws = Ws(moe.moe_layer_workspace_bytes(T, k, E, H, shape.F))
                i2 = torch.empty((T, k), dtype=torch.int32, device="cuda")
                w2 = torch.empty((T, k), device="cuda")
                o2 = torch.empty((T, H), device="cuda")
                moe.moe_layer_forward(desc, dev(x), T, k, dev(wr), None,
                                      None, None, o2, None, i2, w2, None,
                                      ws.t, ws.nbytes)
                torch.cuda.synchronize()
                assert torch.equal(o2, out)
        del pool
    finally:
        dist.destroy_process_group()
        torch.cuda.empty_cache()
