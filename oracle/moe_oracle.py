"""Plain fp64 CPU oracle of the routed Mixture-of-Experts FFN layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code, header, table or
helper with the CUDA library; the only thing both sides share is the seeded
input generator in ``synth``.

It computes, in float64 and in the order the sources describe, what the
layer is defined to compute (sources: the "Avalon" README and the Avalon
GGUF model card -- the model has 512 routed experts with 10 active per token
over 48 layers; the card lists per-tensor expert quant types, among them a
3.25-bpw super-block variant with one scale per 256 weights and 4-bit
sub-scales per 32 weights for up/gate, and a 4-bit non-uniform-codebook type
for down; experts are stored packed as up | gate | down; the "Betelgeuse"
post describes the per-layer VRAM slot pool with on-device hit resolution):

  1. router logits   l[t,e] = sum_h x[t,h] * Wr[e,h] + bias[e]
  2. softmax over all E experts, then the top-k by probability (equal
     values go to the lower expert index), renormalised over the k chosen
  3. grouping of the (token, slot) pairs by expert, stable in pair order
  4. dequantisation of the chosen experts by each format's closed form
  5. h = silu(Wg x) * (Wu x),  silu(z) = z / (1 + exp(-z))
  6. y = Wd h
  7. out[t] = sum_j w[t,j] * y[t,j]  (+ residual)
  8. the expert-slot cache replay (hits, misses, LRU victims)

Readings of points the sources leave open are listed in the repository's
design notes; the ones that shape arithmetic here are:
  * SB3 value: w = d * (2s+1) * c / 8 with c = 2q - 7 (q the 3-bit code).
  * NL4 value: w = d * cb[q] with the 16-entry int8 codebook below.
  * NL3 value: w = d * (2s+1) * (cb3[q] + e) / 16 with the 8-entry codebook
    below and one shift bit e per 32 weights (this repository's own 3-bit
    non-uniform format; the model card lists such a type, IQ3_K, by name
    and bit rate only).
  * SB2 value: w = d * (2s+1) * c / 4 with c = 2q - 3 (q the 2-bit code;
    this repository's 2-bit super-block format, a stand-in for the 2-bit
    up/gate type, IQ2_S, that the model card names without its layout).
  * Q4 value:  w = d * (q - 8).
  * Stacked decode layers use the pre-norm residual r <- r + MoE(x),
    x = bf16(rmsnorm(r)), rmsnorm without a learned weight, eps = 1e-6.

Parity of every function here is pinned by tests against brute force,
closed forms, invariants and library routines (see tests/test_oracle_pins.py).
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np

Q4_B32, SB3_256, NL4_B32, NL3_256, SB2_256 = 1, 2, 3, 4, 5

# 16-entry non-uniform codebook of the 4-bit NL format (ascending).
NL4_CODEBOOK = np.array([-127, -104, -83, -65, -49, -35, -22, -10,
                         1, 13, 25, 38, 53, 69, 89, 113], dtype=np.float64)

# 8-entry non-uniform codebook of the 3-bit NL format (ascending); each
# 32-weight block may shift it up by one (its shift bit e).
NL3_CODEBOOK = np.array([-15, -10, -6, -2, 1, 5, 9, 14], dtype=np.float64)

RMS_EPS = 1e-6


# ------------------------------------------------------------ bit helpers ---
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def fp16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns (uint16 or raw little-endian bytes) -> f64."""
    a = np.asarray(bits)
    if a.dtype == np.uint8:
        a = a.view("<u2")
    return a.astype(np.uint16).view(np.float16).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round to bfloat16 the way a float32 producer does: f64 -> f32 -> bf16,
    both roundings to nearest even."""
    b = np.asarray(v, dtype=np.float64).astype(np.float32).view(np.uint32)
    r = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (r >> np.uint32(16)).astype(np.uint16)


def _bits_le(raw: np.ndarray, nbytes_per_item: int) -> np.ndarray:
    """[n, nbytes] bytes -> [n, 8*nbytes] bits, least significant bit first."""
    a = np.asarray(raw, dtype=np.uint8).reshape(-1, nbytes_per_item)
    return np.unpackbits(a, axis=1, bitorder="little")


# --------------------------------------------------------- dequantisation ---
def tensor_plane_sizes(fmt: int, rows: int, cols: int) -> List[int]:
    if fmt == SB3_256:
        assert cols % 256 == 0
        n = rows * cols // 256
        return [96 * n, 4 * n, 2 * n]
    if fmt == NL3_256:
        assert cols % 256 == 0
        n = rows * cols // 256
        return [96 * n, 4 * n, 2 * n, n]
    if fmt == SB2_256:
        assert cols % 256 == 0
        n = rows * cols // 256
        return [64 * n, 4 * n, 2 * n]
    assert fmt in (Q4_B32, NL4_B32) and cols % 32 == 0
    n = rows * cols // 32
    return [16 * n, 2 * n]


def dequant_sb3(raw: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """3-bit super-block format -> float64 [rows, cols].

    Each row is split into super-blocks of 256 weights.  A super-block has a
    fp16 scale d, eight 4-bit sub-scales s_j (one per 32 weights) and 256
    3-bit codes q.  Weight i of the super-block is
        w_i = d * (2*s_{i//32} + 1) * (2*q_i - 7) / 8.
    """
    n_codes, n_sc, n_d = tensor_plane_sizes(SB3_256, rows, cols)
    raw = np.asarray(raw, dtype=np.uint8)
    codes = raw[:n_codes]
    scales = raw[n_codes:n_codes + n_sc]
    dbits = raw[n_codes + n_sc:n_codes + n_sc + n_d]
    nsb = rows * cols // 256
    # code i of a super-block = bits 3i, 3i+1, 3i+2 of its 96-byte stream
    bits = _bits_le(codes, 96).reshape(nsb, 256, 3)
    q = (bits[:, :, 0] | (bits[:, :, 1] << 1) | (bits[:, :, 2] << 2))
    # sub-scale j = bits 4j..4j+3 of the 32-bit little-endian scale word
    sbits = _bits_le(scales, 4).reshape(nsb, 8, 4)
    s = (sbits[:, :, 0] | (sbits[:, :, 1] << 1) | (sbits[:, :, 2] << 2) |
         (sbits[:, :, 3] << 3))                                      # [nsb,8]
    d = fp16_to_f64(dbits)                                           # [nsb]
    sub = np.repeat(2.0 * s.astype(np.float64) + 1.0, 32, axis=1)    # [nsb,256]
    c = 2.0 * q.astype(np.float64) - 7.0
    w = d[:, None] * sub * c / 8.0
    return w.reshape(rows, cols)


def dequant_nl3(raw: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """3-bit non-uniform-codebook super-block format -> float64 [rows, cols].

    A super-block of 256 weights has a fp16 scale d, eight 4-bit sub-scales
    s_j, eight shift bits e_j (one per 32 weights) and 256 3-bit codes q.
    Weight i of the super-block (j = i // 32) is
        w_i = d * (2*s_j + 1) * (cb3[q_i] + e_j) / 16,
    cb3 = NL3_CODEBOOK.  Codes, sub-scales and d sit exactly as in the SB3
    format; the shift bits are bit j of one byte per super-block.
    """
    n_codes, n_sc, n_d, n_ex = tensor_plane_sizes(NL3_256, rows, cols)
    raw = np.asarray(raw, dtype=np.uint8)
    codes = raw[:n_codes]
    scales = raw[n_codes:n_codes + n_sc]
    dbits = raw[n_codes + n_sc:n_codes + n_sc + n_d]
    extra = raw[n_codes + n_sc + n_d:n_codes + n_sc + n_d + n_ex]
    nsb = rows * cols // 256
    bits = _bits_le(codes, 96).reshape(nsb, 256, 3)
    q = (bits[:, :, 0] | (bits[:, :, 1] << 1) | (bits[:, :, 2] << 2))
    sbits = _bits_le(scales, 4).reshape(nsb, 8, 4)
    s = (sbits[:, :, 0] | (sbits[:, :, 1] << 1) | (sbits[:, :, 2] << 2) |
         (sbits[:, :, 3] << 3))                                      # [nsb,8]
    e = _bits_le(extra, 1).reshape(nsb, 8).astype(np.float64)        # [nsb,8]
    d = fp16_to_f64(dbits)                                           # [nsb]
    sub = np.repeat(2.0 * s.astype(np.float64) + 1.0, 32, axis=1)    # [nsb,256]
    v = NL3_CODEBOOK[q] + np.repeat(e, 32, axis=1)
    w = d[:, None] * sub * v / 16.0
    return w.reshape(rows, cols)


def dequant_sb2(raw: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """2-bit super-block format -> float64 [rows, cols].

    A super-block of 256 weights has a fp16 scale d, eight 4-bit sub-scales
    s_j (one per 32 weights, in a little-endian 32-bit word as in SB3) and
    256 2-bit codes q, code i at bits 2i, 2i+1 of its 64-byte stream.
    Weight i of the super-block is
        w_i = d * (2*s_{i//32} + 1) * (2*q_i - 3) / 4.
    """
    n_codes, n_sc, n_d = tensor_plane_sizes(SB2_256, rows, cols)
    raw = np.asarray(raw, dtype=np.uint8)
    codes = raw[:n_codes]
    scales = raw[n_codes:n_codes + n_sc]
    dbits = raw[n_codes + n_sc:n_codes + n_sc + n_d]
    nsb = rows * cols // 256
    bits = _bits_le(codes, 64).reshape(nsb, 256, 2)
    q = bits[:, :, 0] | (bits[:, :, 1] << 1)
    sbits = _bits_le(scales, 4).reshape(nsb, 8, 4)
    s = (sbits[:, :, 0] | (sbits[:, :, 1] << 1) | (sbits[:, :, 2] << 2) |
         (sbits[:, :, 3] << 3))                                      # [nsb,8]
    d = fp16_to_f64(dbits)                                           # [nsb]
    sub = np.repeat(2.0 * s.astype(np.float64) + 1.0, 32, axis=1)    # [nsb,256]
    c = 2.0 * q.astype(np.float64) - 3.0
    w = d[:, None] * sub * c / 4.0
    return w.reshape(rows, cols)


def _nibbles(codes: np.ndarray) -> np.ndarray:
    """Codes plane -> one 4-bit code per weight (low nibble first)."""
    b = np.asarray(codes, dtype=np.uint8)
    out = np.empty(b.size * 2, dtype=np.int64)
    out[0::2] = b & 0x0F
    out[1::2] = b >> 4
    return out


def dequant_b32(fmt: int, raw: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """32-weight block formats -> float64 [rows, cols].

    Q4_B32:  w = d * (q - 8)
    NL4_B32: w = d * cb[q]
    with one fp16 scale d per 32 consecutive weights of a row.
    """
    n_codes, n_d = tensor_plane_sizes(fmt, rows, cols)
    raw = np.asarray(raw, dtype=np.uint8)
    q = _nibbles(raw[:n_codes]).reshape(rows * cols // 32, 32)
    d = fp16_to_f64(raw[n_codes:n_codes + n_d])
    if fmt == Q4_B32:
        v = (q - 8).astype(np.float64)
    elif fmt == NL4_B32:
        v = NL4_CODEBOOK[q]
    else:
        raise ValueError(fmt)
    return (d[:, None] * v).reshape(rows, cols)


def dequant(fmt: int, raw: np.ndarray, rows: int, cols: int) -> np.ndarray:
    if fmt == SB3_256:
        return dequant_sb3(raw, rows, cols)
    if fmt == NL3_256:
        return dequant_nl3(raw, rows, cols)
    if fmt == SB2_256:
        return dequant_sb2(raw, rows, cols)
    return dequant_b32(fmt, raw, rows, cols)


# ---------------------------------------------------------------- routing ---
def router_logits(x: np.ndarray, wr: np.ndarray,
                  bias: Optional[np.ndarray] = None) -> np.ndarray:
    """l[t,e] = sum_h x[t,h] Wr[e,h] + bias[e]; x [T,H], Wr [E,H] (float64)."""
    l = np.asarray(x, np.float64) @ np.asarray(wr, np.float64).T
    if bias is not None:
        l = l + np.asarray(bias, np.float64)[None, :]
    return l


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (max subtracted)."""
    z = l - l.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores per row, in descending order; equal
    scores are ordered by ascending index.  A full stable sort per row."""
    scores = np.asarray(scores)
    T, E = scores.shape
    out = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        order = np.lexsort((idx, -scores[t].astype(np.float64)))
        out[t] = order[:k]
    return out


def route(logits: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax over all experts, top-k, renormalise: (idx [T,k], w [T,k]).

    The selection is taken on the logits: softmax is strictly increasing, so
    the order of probabilities and logits is the same.
    """
    p = softmax(np.asarray(logits, np.float64))
    idx = topk_select(logits, k)
    ps = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    w = ps / ps.sum(axis=1, keepdims=True)
    return idx, w


def group_pairs(topk_idx: np.ndarray, E: int
                ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Group pairs p = t*k + j by expert, stable in pair order.

    Returns expert_offsets [E+1], pair_ids [T*k] (pairs of expert e are
    pair_ids[offsets[e]:offsets[e+1]], ascending), active experts (ascending).
    """
    flat = np.asarray(topk_idx, np.int64).reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    active = np.nonzero(counts)[0].astype(np.int32)
    return offsets, order.astype(np.int32), active


# -------------------------------------------------------------------- FFN ---
def silu(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(x_rows: np.ndarray, wu: np.ndarray, wg: np.ndarray,
               wd: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """One expert on its token rows: h = silu(Wg x) * (Wu x), y = Wd h.

    x_rows [n,H], wu/wg [F,H], wd [H,F]; returns (h [n,F], y [n,H]).
    """
    u = x_rows @ wu.T
    g = x_rows @ wg.T
    h = silu(g) * u
    return h, h @ wd.T


def combine(y_pairs: np.ndarray, w: np.ndarray,
            residual: Optional[np.ndarray] = None) -> np.ndarray:
    """out[t] = sum_j w[t,j] * y[t*k+j] (+ residual[t])."""
    T, k = w.shape
    y = np.asarray(y_pairs, np.float64).reshape(T, k, -1)
    out = np.einsum("tj,tjh->th", np.asarray(w, np.float64), y)
    if residual is not None:
        out = out + np.asarray(residual, np.float64)
    return out


def rmsnorm(r: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    r = np.asarray(r, np.float64)
    return r / np.sqrt(np.mean(r * r, axis=-1, keepdims=True) + eps)


# ---------------------------------------------------------- whole layer ---
class ExpertSource:
    """Dequantised weights of one layer's experts, built on demand from the
    natural-layout bytes that ``blob_fn(e)`` returns."""

    def __init__(self, H: int, F: int, fmt_up_gate: int, fmt_down: int,
                 blob_fn: Callable[[int], np.ndarray]):
        self.H, self.F = H, F
        self.fug, self.fd = fmt_up_gate, fmt_down
        self.blob_fn = blob_fn
        self.cache: Dict[int, Tuple[np.ndarray, np.ndarray, np.ndarray]] = {}
        n = sum(tensor_plane_sizes(fmt_up_gate, F, H))
        self.off = (0, n, 2 * n)
        self.down_n = sum(tensor_plane_sizes(fmt_down, H, F))

    def weights(self, e: int):
        if e not in self.cache:
            b = np.asarray(self.blob_fn(e), np.uint8)
            n = self.off[1]
            wu = dequant(self.fug, b[0:n], self.F, self.H)
            wg = dequant(self.fug, b[n:2 * n], self.F, self.H)
            wd = dequant(self.fd, b[2 * n:2 * n + self.down_n], self.H, self.F)
            self.cache[e] = (wu, wg, wd)
        return self.cache[e]


def moe_layer(x: np.ndarray, wr: np.ndarray, bias: Optional[np.ndarray],
              k: int, experts: ExpertSource,
              residual: Optional[np.ndarray] = None,
              topk_idx: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """The whole layer in float64.

    x [T,H] and wr [E,H] are float64 (already widened from bf16).  If
    ``topk_idx`` is given, it replaces the oracle's own selection (used when
    the caller wants the expert FFN and combine checked on a given routing);
    the weights are still the renormalised softmax of the logits.
    """
    logits = router_logits(x, wr, bias)
    if topk_idx is None:
        idx, w = route(logits, k)
    else:
        idx = np.asarray(topk_idx, np.int32)
        p = softmax(logits)
        ps = np.take_along_axis(p, idx.astype(np.int64), axis=1)
        w = ps / ps.sum(axis=1, keepdims=True)
    E = wr.shape[0]
    offsets, pair_ids, active = group_pairs(idx, E)
    T = x.shape[0]
    y_pairs = np.zeros((T * k, experts.H))
    h_pairs = np.zeros((T * k, experts.F))
    for e in active:
        pairs = pair_ids[offsets[e]:offsets[e + 1]]
        toks = pairs // k
        wu, wg, wd = experts.weights(int(e))
        h, y = expert_ffn(x[toks], wu, wg, wd)
        y_pairs[pairs] = y
        h_pairs[pairs] = h
    out = combine(y_pairs, w, residual)
    return dict(logits=logits, topk_idx=idx, topk_w=w, offsets=offsets,
                pair_ids=pair_ids, active=active, h_pairs=h_pairs,
                y_pairs=y_pairs, out=out)


# ------------------------------------------------------------- slot cache ---
class SlotCache:
    """Replay of the per-layer expert slot pool (one layer's partition).

    State: ``table[e]`` = slot holding expert e or -1; ``owner[s]`` = expert
    in slot s or -1; ``stamp[s]`` = last step that used or filled slot s.
    A resolve for one (step, layer) with the layer's chosen experts:
      * a chosen expert already in a slot is a hit and uses that slot;
      * the chosen experts not in a slot are the misses, in ascending id;
      * each miss, in that order, takes the slot with the smallest stamp
        among the slots this resolve has not used or filled yet (ties go to
        the lowest slot), whose previous expert leaves the table;
      * every used or filled slot gets the stamp of this step.
    Slot ids are local to the partition (0..capacity-1).
    """

    def __init__(self, E: int, capacity: int, initial: Sequence[int]):
        self.E, self.cap = E, capacity
        self.table = -np.ones(E, np.int32)
        self.owner = -np.ones(capacity, np.int32)
        self.stamp = np.zeros(capacity, np.int64)
        for s, e in enumerate(list(initial)[:capacity]):
            self.table[e] = s
            self.owner[s] = e

    def resolve(self, chosen: np.ndarray, step_stamp: int):
        uniq = sorted(set(int(e) for e in np.asarray(chosen).reshape(-1)))
        used = np.zeros(self.cap, bool)
        slot_of = {}
        misses = []
        for e in uniq:
            if self.table[e] >= 0:
                slot_of[e] = int(self.table[e])
                used[self.table[e]] = True
            else:
                misses.append(e)
        victims = []
        for e in misses:
            free = np.nonzero(~used)[0]
            if free.size == 0:
                raise RuntimeError("slot pool capacity exceeded")
            # smallest stamp, ties to the lowest slot
            s = int(free[np.lexsort((free, self.stamp[free]))[0]])
            old = self.owner[s]
            if old >= 0:
                self.table[old] = -1
            self.owner[s] = e
            self.table[e] = s
            used[s] = True
            slot_of[e] = s
            victims.append(s)
        for s in np.nonzero(used)[0]:
            self.stamp[s] = step_stamp
        return slot_of, misses, victims
