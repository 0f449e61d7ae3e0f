"""Drivers of the multi-layer decode workloads through the library's C ABI:
the all-resident residual stack and the same stack over an expert-slot
pool (misses copied after a host round trip per layer, or pulled from the
pinned host store by the library on the stream itself).  No arithmetic of the layer happens
here -- every layer runs in the library; this module only owns buffers,
builds the device pools with the seeded generator, and moves missed expert
blobs (one copy per expert).

Step semantics (the 48-layer workloads): step s starts from the residual
r = x_s (the seeded bf16 activations of step s, widened to fp32); each
layer l then does r <- r + MoE_l(bf16(rmsnorm(r))) with its own router and
Zipf(1.1) popularity bias.  Steps are independent except through the slot
pool's state.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

import synth
from synth.pools import build_pool, dev, layer_desc


class Stack:
    """L resident layers of one shape, with per-layer routers and biases."""

    def __init__(self, L: int, shape: synth.LayerShape = synth.BIG,
                 seed: int = 0, T: int = 3, zipf: bool = True,
                 build_pools: bool = True):
        import torch
        import quantized_moe_expert_02_b200 as moe
        self.torch, self.moe = torch, moe
        self.L, self.shape, self.seed, self.T = L, shape, seed, T
        self.pools = [build_pool(shape, seed, l) for l in range(L)] \
            if build_pools else []
        self.descs = [layer_desc(shape, p) for p in self.pools]
        self.wr = [dev(synth.gen_router(seed, l, shape.E, shape.H))
                   for l in range(L)]
        self.bias_np = [synth.gen_zipf_bias(seed, l, shape.E)[0] if zipf
                        else None for l in range(L)]
        self.ranks = [synth.gen_zipf_bias(seed, l, shape.E)[1]
                      for l in range(L)]
        self.bias = [dev(b) if b is not None else None for b in self.bias_np]
        k, E, H, F = shape.k, shape.E, shape.H, shape.F
        self.ws_bytes = moe.moe_layer_workspace_bytes(T, k, E, H, F)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        self.w = torch.empty((T, k), device="cuda")

    # ------------------------------------------------------------ inputs --
    def x0(self, step: int):
        """Residual at the stack's input for step s: x_s widened to fp32."""
        xb = synth.gen_x(self.seed, self.T, self.shape.H, step)
        return dev(synth.bf16_bits_to_f32(xb).copy())

    # ----------------------------------------------------------- resident --
    def layer(self, l: int, r, record: Optional[List] = None):
        """One resident layer, in place (one launch for T <= 8)."""
        shp = self.shape
        self.moe.moe_layer_forward_residual(
            self.descs[l], r, self.T, shp.k, self.wr[l], self.bias[l], None,
            r, None, self.idx, self.w, None, self.ws, self.ws_bytes)
        if record is not None:
            record.append(self.idx.clone())

    def run_resident(self, r, layers: Optional[Sequence[int]] = None,
                     record: Optional[List] = None):
        for l in (range(self.L) if layers is None else layers):
            self.layer(l, r, record)
        return r


def hottest(stack: Stack, l: int, n: int) -> np.ndarray:
    return synth.hottest_experts(stack.ranks[l], n)


class SlotPool:
    """The expert-slot pool of the slot-cache workload: per-layer
    partitions of a device pool of blobs, their slot tables, and a pinned
    host store of the blobs that may be copied in.

    The pool starts filled with each layer's hottest experts (slot i holds
    the (i+1)-th hottest); misses are copied from `store`, a pinned host
    tensor with one blob per (layer, expert) key in `store_index`.  With
    store_keys=None the misses are copied from the stack's resident pools
    instead (device to device) and their keys collected in `seen_keys`:
    a discovery run that tells which blobs a host store must hold.
    """

    def __init__(self, stack: Stack, capacities: Sequence[int],
                 store_keys: Optional[Sequence[Tuple[int, int]]],
                 copy_streams: int = 2):
        torch, moe, shp = stack.torch, stack.moe, stack.shape
        self.stack, self.torch, self.moe = stack, torch, moe
        self.caps = [int(c) for c in capacities]
        self.base = np.concatenate([[0], np.cumsum(self.caps)])[:-1]
        n_slots = int(sum(self.caps))
        stride = shp.blob_stride
        self.stride = stride
        self.blob = shp.blob_bytes
        self.pool = torch.empty(n_slots * stride, dtype=torch.uint8,
                                device="cuda")
        E = shp.E
        self._reset_slots()
        self.descs = [layer_desc(shp, self.pool) for _ in self.caps]
        # pinned host store, filled from the resident pools
        self.device_source = store_keys is None
        self.seen_keys = set()
        keys = [] if store_keys is None else \
            sorted(set((int(l), int(e)) for l, e in store_keys))
        self.store_index: Dict[Tuple[int, int], int] = {
            key: i for i, key in enumerate(keys)}
        self.store = torch.empty((max(1, len(keys)), self.blob),
                                 dtype=torch.uint8).pin_memory()
        for (l, e), i in self.store_index.items():
            src = e * stride
            self.store[i].copy_(stack.pools[l][src:src + self.blob])
        torch.cuda.synchronize()
        P = stack.T * shp.k
        self.blob_index = torch.full((E,), -1, dtype=torch.int32,
                                     device="cuda")
        self.mexp = torch.empty(P, dtype=torch.int32, device="cuda")
        self.mslot = torch.empty(P, dtype=torch.int32, device="cuda")
        self.nmiss = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.h_n = torch.zeros(1 + 2 * P, dtype=torch.int32).pin_memory()
        self.misses = 0
        # host-store copies are spread over these streams (half a blob per
        # copy), so that more than one copy engine moves them
        self.copy_streams = [torch.cuda.Stream() for _ in range(copy_streams)]

    def _reset_slots(self) -> None:
        """The starting state: each layer's slots hold its hottest experts,
        every last-use stamp is zero."""
        torch, st, E = self.torch, self.stack, self.stack.shape.E
        self.table, self.owner, self.last = [], [], []
        for l, cap in enumerate(self.caps):
            hot = hottest(st, l, cap)
            tab = torch.full((E,), -1, dtype=torch.int32, device="cuda")
            own = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
            for s, e in enumerate(hot):
                tab[int(e)] = s
                own[s] = int(e)
                dst = (int(self.base[l]) + s) * self.stride
                src = int(e) * self.stride
                self.pool[dst:dst + self.blob].copy_(
                    st.pools[l][src:src + self.blob])
            self.table.append(tab)
            self.owner.append(own)
            self.last.append(torch.zeros(cap, dtype=torch.int32,
                                         device="cuda"))
        self.misses = 0

    def layer(self, l: int, r, stamp: int, log: Optional[List] = None):
        """One layer through the slot pool, in place."""
        st, torch, moe, shp = self.stack, self.torch, self.moe, \
            self.stack.shape
        T, k, E = st.T, shp.k, shp.E
        moe.moe_layer_route_residual(self.descs[l], r, T, k, st.wr[l],
                                     st.bias[l], st.idx, st.w, None, st.ws,
                                     st.ws_bytes)
        moe.moe_slot_resolve(st.idx, T, k, E, self.table[l], self.owner[l],
                             self.last[l], self.caps[l], int(self.base[l]),
                             stamp, self.blob_index, self.mexp, self.mslot,
                             self.nmiss, self.err)
        # the miss list to the host, then one copy per missed expert
        P = T * k
        self.h_n[0:1].copy_(self.nmiss, non_blocking=True)
        self.h_n[1:1 + P].copy_(self.mexp, non_blocking=True)
        self.h_n[1 + P:].copy_(self.mslot, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        n = int(self.h_n[0])
        me = self.h_n[1:1 + n].tolist()
        ms = self.h_n[1 + P:1 + P + n].tolist()
        cur = torch.cuda.current_stream()
        side = self.copy_streams if (n and not self.device_source) else []
        for cs in side:
            cs.wait_stream(cur)
        half = (self.blob // 2 + 255) // 256 * 256
        j = 0
        for e, s in zip(me, ms):
            dst = (int(self.base[l]) + s) * self.stride
            if self.device_source:
                self.seen_keys.add((l, e))
                src = e * self.stride
                self.pool[dst:dst + self.blob].copy_(
                    st.pools[l][src:src + self.blob], non_blocking=True)
            else:
                i = self.store_index[(l, e)]
                for a, b in ((0, half), (half, self.blob)):
                    with torch.cuda.stream(side[j % len(side)]):
                        self.pool[dst + a:dst + b].copy_(self.store[i][a:b],
                                                         non_blocking=True)
                    j += 1
        for cs in side:
            cur.wait_stream(cs)
        self.misses += n
        if log is not None:
            log.append((l, stamp, me, ms))
        moe.moe_layer_ffn_residual(self.descs[l], r, T, k, st.idx, st.w,
                                   self.blob_index, r, None, st.ws,
                                   st.ws_bytes)

    def run(self, r, stamp: int, log: Optional[List] = None):
        for l in range(len(self.caps)):
            self.layer(l, r, stamp, log)
        return r

    # ------------------------------------------- in-stream staging mode --
    def start_staging(self) -> None:
        """Miss handling without a host round trip per layer: after the
        resolve, moe_stage_misses pulls each missed blob from the pinned
        host store into its slot on the same stream.  The resolve keeps its
        LRU stamp in a per-layer device counter (moe_slot_resolve_dev), so
        that no host argument changes from one step to the next and a whole
        step can be captured once as a CUDA graph."""
        torch, moe = self.torch, self.moe
        assert not self.device_source, "in-stream staging needs a host store"
        L, E = len(self.caps), self.stack.shape.E
        table = [0] * (L * E)
        for (l, e), i in self.store_index.items():
            table[l * E + e] = self.store[i].data_ptr()
        self.table_dev = torch.zeros(L * E, dtype=torch.int64, device="cuda")
        moe.moe_stage_table(table, self.table_dev)
        self.n_slots = int(sum(self.caps))
        # stamp counters: counter l = number of steps layer l has resolved
        self.stamps = torch.zeros(L, dtype=torch.int32, device="cuda")

    def reset(self) -> None:
        self._reset_slots()
        if hasattr(self, "stamps"):
            self.stamps.zero_()

    def layer_staged(self, l: int, r, fused: bool = False) -> None:
        """One layer through the slot pool, in place, with no host sync.
        fused: the pull inside the FFN launch, overlapping the hits'
        compute (moe_layer_ffn_residual_staged); else the pull kernel
        (moe_stage_misses), then the FFN."""
        st, moe, shp = self.stack, self.moe, self.stack.shape
        T, k, E = st.T, shp.k, shp.E
        moe.moe_layer_route_residual(self.descs[l], r, T, k, st.wr[l],
                                     st.bias[l], st.idx, st.w, None, st.ws,
                                     st.ws_bytes)
        moe.moe_slot_resolve_dev(st.idx, T, k, E, self.table[l],
                                 self.owner[l], self.last[l], self.caps[l],
                                 int(self.base[l]),
                                 self.stamps.data_ptr() + 4 * l,
                                 self.blob_index, self.mexp, self.mslot,
                                 self.nmiss, self.err)
        if fused:
            moe.moe_layer_ffn_residual_staged(
                self.descs[l], r, T, k, st.idx, st.w, self.blob_index, r,
                None, self.nmiss, self.mexp, self.mslot, l, len(self.caps),
                self.table_dev, int(self.base[l]), self.caps[l],
                self.n_slots, st.ws, st.ws_bytes)
            return
        moe.moe_stage_misses(self.nmiss, self.mexp, self.mslot, T * k, l,
                             len(self.caps), E, self.table_dev, self.pool,
                             int(self.base[l]), self.caps[l], self.n_slots,
                             self.stride, self.blob, self.err)
        moe.moe_layer_ffn_residual(self.descs[l], r, T, k, st.idx, st.w,
                                   self.blob_index, r, None, st.ws,
                                   st.ws_bytes)

    def run_staged(self, r, fused: bool = False):
        """One step: every layer in order, in place on r."""
        for l in range(len(self.caps)):
            self.layer_staged(l, r, fused)
        return r

    def capture_step(self, x_in, r, fused: bool = False):
        """The whole step -- r <- x_in, then route, resolve, pull and FFN of
        every layer -- captured once as one CUDA graph; each replay runs
        the next step (the slot state and the stamp counters live on the
        device).  Returns the graph."""
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g):
            r.copy_(x_in)
            self.run_staged(r, fused)
        return g
