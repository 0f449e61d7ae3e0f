"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws inputs.  It holds none of the layer's arithmetic
(no routing, no dequantisation, no FFN); the oracle and the CUDA path both
take their inputs from here and share nothing else.

Everything is keyed by integers, so any piece can be regenerated alone:

* activations ``x`` and router rows ``Wr``: normal draws from NumPy's PCG64,
  rounded to bfloat16 (returned as raw uint16 bit patterns);
* the per-layer Zipf popularity bias added to the router logits;
* expert weights: raw bytes of each quantised tensor in its *natural* byte
  layout (see ``tensor_planes``), drawn from a counter-based SplitMix64
  stream (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014).  Code and sub-scale bytes are uniform random
  bytes; the fp16 block scales are ``lo + (hi - lo) * u`` in float64 with
  ``u = (word >> 11) * 2**-53``, rounded to fp16 (round to nearest even).
  ``synth/csrc/synth.cu`` implements the same stream on the device and must
  produce identical bytes (checked by a GPU test).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Tuple

import numpy as np

# ---------------------------------------------------------------- formats ---
# Format ids (same numbering as the C ABI's moe_qfmt).
Q4_B32 = 1    # 4-bit codes, 32 weights per block, fp16 scale: w = d*(q-8)
SB3_256 = 2   # 3-bit codes, 256-weight super-block, 8 4-bit sub-scales
NL4_B32 = 3   # 4-bit codes into a 16-entry int8 codebook, fp16 scale
NL3_256 = 4   # 3-bit codes into an 8-entry codebook, 256-weight super-block
SB2_256 = 5   # 2-bit codes, 256-weight super-block, 8 4-bit sub-scales

FMT_NAMES = {Q4_B32: "q4_b32", SB3_256: "sb3_256", NL4_B32: "nl4_b32",
             NL3_256: "nl3_256", SB2_256: "sb2_256"}

BLOB_ALIGN = 4096  # expert blobs start on 4 KiB boundaries


def tensor_planes(fmt: int, rows: int, cols: int) -> List[Tuple[str, int]]:
    """Byte planes of one quantised [rows x cols] tensor, in storage order.

    Natural layout (row-major blocks along each row, planar per tensor):
      SB3_256: codes   rows*cols*3/8 B (256 codes of a super-block = 96 B,
                       a little-endian bit stream, code i at bit 3*i),
               scales  rows*(cols/256)*4 B (sub-scale j at bit 4*j of a
                       little-endian 32-bit word),
               d       rows*(cols/256) fp16.
      NL3_256: the three SB3 planes, then
               extra   rows*(cols/256) B (bit j = codebook shift of 32-block j).
      SB2_256: codes   rows*cols/4 B (64 B per super-block, code i at bits
                       2*(i%4) of byte i/4), then scales and d as SB3.
      Q4_B32 / NL4_B32: codes rows*cols/2 B (weight i of a row in byte i/2,
                       low nibble for even i), d rows*(cols/32) fp16.
    """
    if fmt in (SB3_256, NL3_256, SB2_256):
        if cols % 256:
            raise ValueError("super-block formats need cols % 256 == 0")
        nsb = rows * (cols // 256)
        cb = 64 if fmt == SB2_256 else 96
        planes = [("codes", nsb * cb), ("scales", nsb * 4), ("d", nsb * 2)]
        if fmt == NL3_256:
            planes.append(("extra", nsb))
        return planes
    if fmt in (Q4_B32, NL4_B32):
        if cols % 32:
            raise ValueError("32-weight block formats need cols % 32 == 0")
        nb = rows * (cols // 32)
        return [("codes", nb * 16), ("d", nb * 2)]
    raise ValueError(f"unknown format {fmt}")


def tensor_bytes(fmt: int, rows: int, cols: int) -> int:
    return sum(n for _, n in tensor_planes(fmt, rows, cols))


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shapes and formats of one MoE layer's experts."""
    H: int            # hidden size (model dim)
    F: int            # expert FFN width
    E: int            # number of routed experts
    k: int            # experts per token
    fmt_up_gate: int
    fmt_down: int
    d_up_gate: Tuple[float, float]   # U[lo, hi] of the fp16 block scales
    d_down: Tuple[float, float]

    @property
    def up_bytes(self) -> int:
        return tensor_bytes(self.fmt_up_gate, self.F, self.H)

    @property
    def down_bytes(self) -> int:
        return tensor_bytes(self.fmt_down, self.H, self.F)

    @property
    def blob_bytes(self) -> int:
        """Bytes of one packed expert: up | gate | down."""
        return 2 * self.up_bytes + self.down_bytes

    @property
    def blob_stride(self) -> int:
        return (self.blob_bytes + BLOB_ALIGN - 1) // BLOB_ALIGN * BLOB_ALIGN

    def tensor_offsets(self) -> Dict[str, int]:
        return {"up": 0, "gate": self.up_bytes, "down": 2 * self.up_bytes}


# The two layer shapes of the workloads.  The tiny one is the 8-token parity
# case; the large one is the 512-expert, top-10 layer of the pages' model
# (hidden 3072, expert FFN 1024).
TINY = LayerShape(H=256, F=128, E=16, k=2, fmt_up_gate=Q4_B32, fmt_down=Q4_B32,
                  d_up_gate=(0.005, 0.02), d_down=(0.005, 0.02))
BIG = LayerShape(H=3072, F=1024, E=512, k=10, fmt_up_gate=SB3_256,
                 fmt_down=NL4_B32, d_up_gate=(0.002, 0.01),
                 d_down=(0.002, 0.01))

# The decode layer shape with up/gate in the 3-bit non-uniform-codebook
# format (64 experts, top-8: a smaller pool for the format's parity tests).
NL3_SHAPE = LayerShape(H=3072, F=1024, E=64, k=8, fmt_up_gate=NL3_256,
                       fmt_down=NL4_B32, d_up_gate=(0.002, 0.01),
                       d_down=(0.002, 0.01))

# The same decode shape with up/gate in the 2-bit super-block format.
SB2_SHAPE = LayerShape(H=3072, F=1024, E=64, k=8, fmt_up_gate=SB2_256,
                       fmt_down=NL4_B32, d_up_gate=(0.002, 0.01),
                       d_down=(0.002, 0.01))

ZIPF_S = 1.1
ROUTER_STD = 0.02

# ------------------------------------------------------------- SplitMix64 ---
_M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_MUL1 = 0xBF58476D1CE4E5B9
_MUL2 = 0x94D049BB133111EB
_KEY0 = 0x243F6A8885A308D3


def _mix64_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * _MUL1) & _M64
    z = ((z ^ (z >> 27)) * _MUL2) & _M64
    return z ^ (z >> 31)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_MUL1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_MUL2)
    return z ^ (z >> np.uint64(31))


def stream_key(*fields: int) -> int:
    """Key of one counter stream: a SplitMix64 hash chain over the fields."""
    k = _KEY0
    for f in fields:
        k = _mix64_int(((k ^ (f & _M64)) + GAMMA) & _M64)
    return k


def stream_words(key: int, start: int, n: int) -> np.ndarray:
    """Words start..start+n-1 of the stream: mix64(key + (i+1)*GAMMA)."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + i * np.uint64(GAMMA)
        return _mix64(z)


# Stream ids of the three tensors and their planes.
TENSOR_ID = {"up": 0, "gate": 1, "down": 2}
PLANE_ID = {"codes": 0, "scales": 1, "d": 2, "extra": 3}


def _random_bytes(key: int, n: int) -> np.ndarray:
    w = stream_words(key, 0, (n + 7) // 8)
    return w.astype("<u8").view(np.uint8)[:n].copy()


def _scale_plane(key: int, n: int, lo: float, hi: float) -> np.ndarray:
    w = stream_words(key, 0, n)
    u = (w >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    d = np.float64(lo) + np.float64(hi - lo) * u
    return d.astype(np.float16).view(np.uint8)


def gen_tensor(seed: int, layer: int, expert: int, name: str, fmt: int,
               rows: int, cols: int, d_range: Tuple[float, float]) -> np.ndarray:
    """Natural-layout bytes of one quantised tensor (uint8 array)."""
    out = []
    tid = TENSOR_ID[name]
    for plane, n in tensor_planes(fmt, rows, cols):
        key = stream_key(seed, layer, expert, tid, PLANE_ID[plane])
        if plane == "d":
            out.append(_scale_plane(key, n // 2, *d_range))
        else:
            out.append(_random_bytes(key, n))
    return np.concatenate(out)


def gen_expert_blob(shape: LayerShape, seed: int, layer: int, expert: int,
                    pad: bool = True) -> np.ndarray:
    """Natural-layout bytes of one expert: up | gate | down (+ zero pad)."""
    parts = [
        gen_tensor(seed, layer, expert, "up", shape.fmt_up_gate, shape.F,
                   shape.H, shape.d_up_gate),
        gen_tensor(seed, layer, expert, "gate", shape.fmt_up_gate, shape.F,
                   shape.H, shape.d_up_gate),
        gen_tensor(seed, layer, expert, "down", shape.fmt_down, shape.H,
                   shape.F, shape.d_down),
    ]
    blob = np.concatenate(parts)
    if pad and blob.size < shape.blob_stride:
        blob = np.concatenate([blob, np.zeros(shape.blob_stride - blob.size,
                                              np.uint8)])
    return blob


def split_blob(shape: LayerShape, blob: np.ndarray) -> Dict[str, np.ndarray]:
    off = shape.tensor_offsets()
    return {
        "up": blob[off["up"]:off["up"] + shape.up_bytes],
        "gate": blob[off["gate"]:off["gate"] + shape.up_bytes],
        "down": blob[off["down"]:off["down"] + shape.down_bytes],
    }


# ------------------------------------------------- activations and router ---
TAG_X, TAG_ROUTER, TAG_ZIPF, TAG_STEP = 11, 12, 13, 14


def _rng(*entropy: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        [int(e) for e in entropy])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def gen_x(seed: int, T: int, H: int, step: int = 0) -> np.ndarray:
    """Token activations ~N(0,1) as bf16 bits, [T, H]."""
    v = _rng(seed, TAG_X, step, T).standard_normal((T, H))
    return f32_to_bf16_bits(v.astype(np.float32))


def gen_router(seed: int, layer: int, E: int, H: int) -> np.ndarray:
    """Router weight ~N(0, 0.02^2) as bf16 bits, [E, H] row-major."""
    v = _rng(seed, TAG_ROUTER, layer).standard_normal((E, H)) * ROUTER_STD
    return f32_to_bf16_bits(v.astype(np.float32))


def zipf_popularity(E: int, s: float = ZIPF_S) -> np.ndarray:
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    return p / p.sum()


def gen_zipf_bias(seed: int, layer: int, E: int, s: float = ZIPF_S
                  ) -> Tuple[np.ndarray, np.ndarray]:
    """Per-layer router-logit bias ln(p[rank(e)]) (fp32) and the ranks.

    rank[e] is expert e's popularity rank (0 = hottest), a seeded random
    permutation per layer; p is a Zipf(s) distribution over the ranks.
    """
    rank = _rng(seed, TAG_ZIPF, layer).permutation(E)
    p = zipf_popularity(E, s)
    bias = np.log(p[rank]).astype(np.float32)
    return bias, rank.astype(np.int64)


def hottest_experts(rank: np.ndarray, n: int) -> np.ndarray:
    """Experts ordered by popularity, hottest first (first n)."""
    return np.argsort(rank, kind="stable")[:n]


# ------------------------------------------------------------- workloads ---
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    T: int
    layers: int = 1
    zipf: bool = False
    seed: int = 0
    description: str = ""


WORKLOADS = {
    "tiny": Workload("tiny", TINY, T=8, description=(
        "8 tokens, hidden 256, expert FFN 128, 16 experts, top-2, 4-bit "
        "block experts")),
    "decode_t1": Workload("decode_t1", BIG, T=1, description=(
        "decode, one layer, 1 token, 512 experts top-10, SB3 up/gate, NL4 "
        "down")),
    "decode_t3": Workload("decode_t3", BIG, T=3, description=(
        "decode, one layer, 3 tokens (1 + 2 MTP drafts)")),
    "decode_stack": Workload("decode_stack", BIG, T=3, layers=48, zipf=True,
                             description="48-layer decode stack, Zipf(1.1)"
                             " routing, all experts resident"),
    "prefill": Workload("prefill", BIG, T=9536, zipf=True, description=(
        "prefill chunk, one layer, 9536 tokens, Zipf(1.1) routing")),
    "slot_cache": Workload("slot_cache", BIG, T=3, layers=48, zipf=True,
                           description="48-layer decode with a device expert"
                           " slot pool and LRU refills"),
}

# Per-layer slot capacity of the slot-pool workload.
def slot_capacity(layer: int) -> int:
    if layer < 5:
        return 240
    if layer < 32:
        return 92
    return 60


def slot_layout(layers: int = 48) -> Tuple[np.ndarray, int]:
    """First slot of each layer's partition and the total slot count."""
    caps = np.array([slot_capacity(l) for l in range(layers)], np.int64)
    begin = np.concatenate([[0], np.cumsum(caps)[:-1]])
    return begin, int(caps.sum())


__all__ = [n for n in dir() if not n.startswith("_")]
