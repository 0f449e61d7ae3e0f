"""Expert parallelism: one MoE layer's experts sharded over the ranks of a
process group, one process per GPU (the "Avalon" README's multi-GPU
paragraph, where an added GPU holds more of the experts and a decode step
exchanges only small activation rows between the GPUs).

Placement: expert e lives on rank e % G as that rank's local expert e // G.
Per layer, every rank with its own tokens:

  1. routes them (library: moe_route_topk) -> topk_idx [T, k], topk_w;
  2. dispatch: the T*k pairs, sorted by owner rank (stable in pair order),
     send their token rows and local expert ids to the owners -- the
     counts, then the rows, with one all-to-all each;
  3. computes every pair it received on its own experts (library: the
     grouping of the received rows by local expert, then the expert FFN,
     one expert per row);
  4. combine: the output rows travel back with the reverse all-to-all, go
     back to pair order, and the weighted combine (library: moe_combine)
     gives the layer output.

Steps 2 and 4 are index bookkeeping and collectives (torch.distributed:
NCCL between GPUs, gloo on CPU); every step of the layer's arithmetic runs
in the library's kernels.  The collectives move rows as raw bytes, so any
row type crosses unchanged.
"""
from __future__ import annotations

from typing import List, Optional, Tuple


class ExpertParallel:
    """Dispatch and combine of one layer's pairs over a process group."""

    def __init__(self, E: int, k: int, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E, self.k = E, k
        if E < self.world:
            raise ValueError("fewer experts than ranks")

    # ------------------------------------------------------- placement --
    def owner(self, e: int) -> int:
        return e % self.world

    def local_experts(self) -> List[int]:
        """Global ids of this rank's experts, in local order."""
        return list(range(self.rank, self.E, self.world))

    @property
    def n_local(self) -> int:
        return len(self.local_experts())

    # -------------------------------------------------------- exchange --
    def _a2a(self, out, inp, out_splits, in_splits) -> None:
        self.dist.all_to_all_single(out, inp, out_splits, in_splits,
                                    group=self.group)

    def dispatch(self, x, topk_idx) -> Tuple[object, object, tuple]:
        """x [T x row] (any dtype), topk_idx [T x k] int32 on x's device.
        Returns the rows this rank must compute [N x row], their local
        expert ids [N] (int32) and the plan that combine() needs."""
        import torch
        T = x.shape[0]
        flat = topk_idx.reshape(-1).to(torch.int64)
        dest = torch.remainder(flat, self.world)
        order = torch.sort(dest, stable=True).indices
        send = torch.bincount(dest, minlength=self.world)
        recv = torch.empty_like(send)
        self._a2a(recv, send, None, None)
        send_l, recv_l = send.tolist(), recv.tolist()
        xb = x.contiguous().view(torch.uint8).reshape(T, -1)
        x_send = xb.index_select(0, torch.div(order, self.k,
                                              rounding_mode="floor"))
        lid_send = torch.div(flat.index_select(0, order), self.world,
                             rounding_mode="floor").to(torch.int32)
        n = sum(recv_l)
        x_recv = torch.empty((n, xb.shape[1]), dtype=torch.uint8,
                             device=x.device)
        lid_recv = torch.empty(n, dtype=torch.int32, device=x.device)
        self._a2a(x_recv, x_send, recv_l, send_l)
        self._a2a(lid_recv, lid_send, recv_l, send_l)
        x_recv = x_recv.view(x.dtype).reshape(n, *x.shape[1:])
        return x_recv, lid_recv, (order, send_l, recv_l, T)

    def combine(self, y_recv, plan):
        """y_recv [N x H] rows of the received pairs (dispatch order) ->
        y_pairs [T*k x H] of this rank's own pairs, in pair order."""
        import torch
        order, send_l, recv_l, T = plan
        H = y_recv.shape[1]
        yb = y_recv.contiguous().view(torch.uint8).reshape(y_recv.shape[0],
                                                           -1)
        back = torch.empty((sum(send_l), yb.shape[1]), dtype=torch.uint8,
                           device=y_recv.device)
        self._a2a(back, yb, send_l, recv_l)
        back = back.view(y_recv.dtype).reshape(-1, H)
        y_pairs = torch.empty((T * self.k, H), dtype=y_recv.dtype,
                              device=y_recv.device)
        y_pairs[order] = back
        return y_pairs


class ExpertParallelLayer:
    """One MoE layer under expert parallelism on the GPU: routing, local
    expert FFN and combine in the library, the exchange in ExpertParallel.

    pool: packed blobs of this rank's experts, local expert i at
    i * shape.blob_stride; w_router / bias: the full router (every rank
    routes its own tokens over all E experts)."""

    def __init__(self, ep: ExpertParallel, shape, pool, w_router,
                 bias=None):
        import torch
        from . import moe_layer_desc
        self.ep, self.shape = ep, shape
        self.wr, self.bias = w_router, bias
        self.desc = moe_layer_desc(
            H=shape.H, F=shape.F, E=ep.n_local, fmt_up_gate=shape.fmt_up_gate,
            fmt_down=shape.fmt_down, pool=pool.data_ptr(),
            blob_stride=shape.blob_stride)
        self.torch = torch
        self.last_rows: Optional[int] = None
        # name -> (device buffer, rows it was last laid out for): reused
        # while the received row count stays the same; a workspace laid out
        # for another count is zeroed first (its counters sit elsewhere)
        self._ws = {}

    def _buf(self, name: str, n: int, dtype, device, rows: int):
        """The first n elements of a reusable device buffer, zero unless it
        served a call with the same received row count before."""
        b, last = self._ws.get(name, (None, None))
        if b is None or b.numel() < n or b.device != device:
            b, last = self.torch.zeros(max(n, 1), dtype=dtype,
                                       device=device), rows
        elif last != rows:
            b.zero_()
        self._ws[name] = (b, rows)
        return b[:n]

    def forward(self, x, out) -> None:
        """x bf16 bits [T x H] (int16 tensor, device); out fp32 [T x H]."""
        import quantized_moe_expert_02_b200 as moe
        torch, shp, ep = self.torch, self.shape, self.ep
        T, k, E, H = x.shape[0], shp.k, shp.E, shp.H
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, k), device=x.device)
        lg = torch.empty((T, E), device=x.device)
        moe.moe_route_topk(x, T, H, self.wr, E, self.bias, k, idx, w, lg)
        x_recv, lid, plan = ep.dispatch(x, idx)
        n = x_recv.shape[0]
        self.last_rows = n
        y_recv = torch.zeros((n, H), device=x.device)
        if n:
            El, dev = ep.n_local, x.device
            i32, u8 = torch.int32, torch.uint8
            gws_b = moe.moe_group_workspace_bytes(n, 1, El)
            gws = self._buf("gws", max(256, gws_b), u8, dev, n)
            off = self._buf("off", El + 1, i32, dev, n)
            prs = self._buf("prs", n, i32, dev, n)
            act = self._buf("act", El, i32, dev, n)
            na = self._buf("na", 1, i32, dev, n)
            moe.moe_group_tokens(lid, n, 1, El, off, prs, act, na, gws,
                                 gws_b)
            fws_b = moe.moe_ffn_workspace_bytes(n, 1, H, shp.F)
            fws = self._buf("fws", fws_b, u8, dev, n)
            moe.moe_expert_ffn_q(self.desc, x_recv, n, 1, off, prs, act, na,
                                 None, y_recv, fws, fws_b)
        y_pairs = ep.combine(y_recv, plan)
        moe.moe_combine(y_pairs, w, T, k, H, None, out, None)
        return idx, w
