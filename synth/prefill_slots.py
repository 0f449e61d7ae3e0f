"""Driver of the prefill chunk through one layer's expert-slot partition
(the prefill prefetch of the "Avalon" README's feature list: a few slots
taken over from the GPU expert cache stream the missing experts while the
cached ones are used in their slots).

Everything here is orchestration through the library's C ABI -- buffers,
host-side lists of experts, copies of whole blobs, streams and events; no
arithmetic of the layer happens here.  Per call:

  1. the chunk is routed and grouped on the device (moe_route_topk,
     moe_group_tokens); the host reads the chosen experts and the
     partition's slot table (one synchronisation);
  2. `borrow` slots are taken from the partition -- the least recently
     used ones, ties to the lowest slot -- and their experts leave the
     table;
  3. the chosen experts still in the partition are computed first, in
     place (moe_group_subset restricts the grouping to them, then the
     expert FFN);
  4. the other chosen experts go through the borrowed slots in waves of
     borrow/2 experts, the two halves used in turn: while wave w computes,
     the blobs of wave w+1 are copied from the pinned host store into the
     other half on a copy stream (one copy per expert);
  5. the weighted combine of all pairs.

Every pair's output row is the row the all-resident layer computes, so the
result is bit-identical to moe_layer_forward on a pool holding every
expert.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np


class Partition:
    """One layer's slot partition: `n_slots` blobs in device memory, the
    slot table (expert -> slot or -1), slot owners and last-use stamps,
    filled with the given experts (slot i holds experts[i])."""

    def __init__(self, shape, resident_pool, experts, n_slots: int):
        import torch
        self.shape, self.n = shape, int(n_slots)
        stride = shape.blob_stride
        self.pool = torch.empty(self.n * stride, dtype=torch.uint8,
                                device="cuda")
        self.table = torch.full((shape.E,), -1, dtype=torch.int32,
                                device="cuda")
        self.owner = torch.full((self.n,), -1, dtype=torch.int32,
                                device="cuda")
        self.last = torch.zeros(self.n, dtype=torch.int32, device="cuda")
        for s, e in enumerate(list(experts)[:self.n]):
            e = int(e)
            self.pool[s * stride:s * stride + shape.blob_bytes].copy_(
                resident_pool[e * stride:e * stride + shape.blob_bytes])
            self.table[e] = s
            self.owner[s] = e


class PrefillSlots:
    """Prefill of one layer through a Partition, with the misses streamed
    from a pinned host store (`store` [n, blob_bytes] pinned uint8 tensor,
    `store_index` expert -> row)."""

    def __init__(self, shape, part: Partition, store, store_index: Dict[int,
                 int], T: int, borrow: int = 8):
        import torch
        import quantized_moe_expert_02_b200 as moe
        from .pools import layer_desc
        assert borrow >= 2 and borrow % 2 == 0 and borrow < part.n
        self.torch, self.moe = torch, moe
        self.shape, self.part, self.T = shape, part, T
        self.store, self.store_index = store, store_index
        self.borrow = borrow
        E, k, H, F = shape.E, shape.k, shape.H, shape.F
        self.desc = layer_desc(shape, part.pool)
        P = T * k
        dev = dict(device="cuda")
        self.idx = torch.empty((T, k), dtype=torch.int32, **dev)
        self.w = torch.empty((T, k), **dev)
        self.logits = torch.empty((T, E), **dev)
        self.off = torch.empty(E + 1, dtype=torch.int32, **dev)
        self.pairs = torch.empty(P, dtype=torch.int32, **dev)
        self.act = torch.empty(E, dtype=torch.int32, **dev)
        self.na = torch.zeros(1, dtype=torch.int32, **dev)
        self.s_off = torch.empty(E + 1, dtype=torch.int32, **dev)
        self.s_pairs = torch.empty(P, dtype=torch.int32, **dev)
        self.s_act = torch.empty(E, dtype=torch.int32, **dev)
        self.s_na = torch.zeros(1, dtype=torch.int32, **dev)
        self.err = torch.zeros(1, dtype=torch.int32, **dev)
        self.blob_index = torch.full((E,), -1, dtype=torch.int32, **dev)
        self.lists = torch.empty(E, dtype=torch.int32, **dev)
        self.y = torch.empty((P, H), **dev)
        self.gws_bytes = moe.moe_group_workspace_bytes(T, k, E)
        self.gws = torch.zeros(max(256, self.gws_bytes), dtype=torch.uint8,
                               **dev)
        self.fws_bytes = moe.moe_ffn_workspace_bytes(T, k, H, F)
        self.fws = torch.zeros(self.fws_bytes, dtype=torch.uint8, **dev)
        self.copy_stream = torch.cuda.Stream()
        self.last_stats: Optional[dict] = None

    def _ffn(self, experts_dev_off: int, n: int) -> None:
        """The expert FFN of n experts listed at self.lists[off:off+n]."""
        moe, shp = self.moe, self.shape
        moe.moe_group_subset(self.off, self.pairs, shp.E,
                             self.lists.data_ptr() + 4 * experts_dev_off, n,
                             self.s_off, self.s_pairs, self.s_act, self.s_na,
                             self.err)
        moe.moe_expert_ffn_q(self.desc, self.x, self.T, shp.k, self.s_off,
                             self.s_pairs, self.s_act, self.s_na,
                             self.blob_index, self.y, self.fws,
                             self.fws_bytes)

    def forward(self, x, wr, bias, out) -> dict:
        """out fp32 [T x H] = the layer on x (bf16 bits [T x H], device)."""
        torch, moe, shp, part = self.torch, self.moe, self.shape, self.part
        T, k, E, H = self.T, shp.k, shp.E, shp.H
        self.x = x
        cur = torch.cuda.current_stream()
        moe.moe_route_topk(x, T, H, wr, E, bias, k, self.idx, self.w,
                           self.logits)
        moe.moe_group_tokens(self.idx, T, k, E, self.off, self.pairs,
                             self.act, self.na, self.gws, self.gws_bytes)
        # the host learns the chosen experts and the partition's state
        na = int(self.na.item())
        act = self.act[:na].cpu().numpy()
        table = part.table.cpu().numpy()
        last = part.last.cpu().numpy()
        # borrowed slots: the least recently used, ties to the lowest slot
        borrowed = [int(s) for s in
                    np.lexsort((np.arange(part.n), last))[:self.borrow]]
        for s in borrowed:
            e = int(part.owner[s].item())
            if e >= 0:
                table[e] = -1
                part.table[e] = -1
            part.owner[s] = -1
        hits = [int(e) for e in act if table[e] >= 0]
        misses = [int(e) for e in act if table[e] < 0]
        half = self.borrow // 2
        waves: List[List[int]] = [misses[i:i + half]
                                  for i in range(0, len(misses), half)]
        # blob of every chosen expert: its slot, or its borrowed slot
        bi = np.full(E, -1, np.int32)
        for e in hits:
            bi[e] = table[e]
        for w, wave in enumerate(waves):
            for i, e in enumerate(wave):
                bi[e] = borrowed[(w % 2) * half + i]
        self.blob_index.copy_(torch.from_numpy(bi))
        lists = np.array(hits + misses, np.int32)
        if lists.size:
            self.lists[:lists.size].copy_(torch.from_numpy(lists))
        # resident experts first, in place
        if hits:
            self._ffn(0, len(hits))
        # misses in waves through the borrowed halves; the blobs of a wave
        # are copied on the copy stream once the wave two back is done
        cs, stride, blob = self.copy_stream, shp.blob_stride, shp.blob_bytes
        copied = [torch.cuda.Event() for _ in waves]
        free = [torch.cuda.Event(), torch.cuda.Event()]
        cs.wait_stream(cur)
        for w, wave in enumerate(waves):
            with torch.cuda.stream(cs):
                if w >= 2:
                    cs.wait_event(free[w % 2])
                for i, e in enumerate(wave):
                    s = borrowed[(w % 2) * half + i]
                    part.pool[s * stride:s * stride + blob].copy_(
                        self.store[self.store_index[e]], non_blocking=True)
                copied[w].record(cs)
            cur.wait_event(copied[w])
            self._ffn(len(hits) + w * half, len(wave))
            free[w % 2].record(cur)
        moe.moe_combine(self.y, self.w, T, k, H, None, out, None)
        # the borrowed slots keep the last experts copied into them
        for w in range(max(0, len(waves) - 2), len(waves)):
            for i, e in enumerate(waves[w]):
                s = borrowed[(w % 2) * half + i]
                part.table[e] = s
                part.owner[s] = e
        self.last_stats = dict(chosen=na, hits=len(hits),
                               misses=len(misses), waves=len(waves),
                               h2d_bytes=len(misses) * blob)
        return self.last_stats
