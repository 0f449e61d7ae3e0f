"""CPU: expert parallelism's dispatch and combine over real collectives --
2 and 3 gloo ranks on 127.0.0.1, each with its own tokens (unequal counts),
experts placed on rank e % G.  The expert compute on every rank is the fp64
oracle on that rank's own experts (no GPU here); the combined result of
each rank must equal the single-process oracle layer on its tokens, and the
rows each rank receives must be exactly the pairs its experts own."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(rank: int):
    import oracle as o
    import synth
    shape = synth.TINY
    T = 5 + 2 * rank
    x = o.bf16_to_f64(synth.gen_x(0, T, shape.H, 100 + rank))
    wr = o.bf16_to_f64(synth.gen_router(0, 0, shape.E, shape.H))
    idx, w = o.route(o.router_logits(x, wr), shape.k)
    return shape, x, wr, idx, w


def _rank(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import oracle as o
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from quantized_moe_expert_02_b200.ep import ExpertParallel
    from helpers import oracle_experts
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shape, x, wr, idx, w = _inputs(rank)
        ep = ExpertParallel(shape.E, shape.k)
        assert ep.local_experts() == list(range(rank, shape.E, world))
        xt = torch.from_numpy(x)
        x_recv, lid, plan = ep.dispatch(xt, torch.from_numpy(idx))
        # this rank's experts on the rows it received (fp64 oracle)
        src = oracle_experts(shape, 0, 0)
        xr = x_recv.numpy()
        y = np.zeros((xr.shape[0], shape.H))
        for i, l in enumerate(lid.tolist()):
            e = l * world + rank
            assert ep.owner(e) == rank
            y[i] = o.expert_ffn(xr[i:i + 1], *src.weights(e))[1][0]
        y_pairs = ep.combine(torch.from_numpy(y), plan).numpy()
        ref = o.moe_layer(x, wr, None, shape.k, src, topk_idx=idx)
        # equal up to fp64 rounding: rows computed one at a time here, per
        # expert in a batch by the reference
        def close(a, b):
            return bool(np.abs(a - b).max() <= 1e-12 * np.abs(b).max())
        out[rank] = dict(rows=xr.shape[0],
                         y_ok=close(y_pairs, ref["y_pairs"]),
                         out_ok=close(o.combine(y_pairs, w), ref["out"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_dispatch_combine_matches_oracle(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world,
                       join=True, start_method="spawn")
    # rows received by each rank = the pairs (over all ranks) its experts own
    owned = [0] * world
    for r in range(world):
        _, _, _, idx, _ = _inputs(r)
        for e in idx.reshape(-1).tolist():
            owned[e % world] += 1
    for r in range(world):
        assert out[r]["y_ok"] and out[r]["out_ok"], r
        assert out[r]["rows"] == owned[r], r
