"""GPU: the decoders that the hot path actually runs, bit for bit against the
oracle's closed forms.

moe_dequant_path exports the weights as (a) the int8 tensor-core tile
decoders of the decode kernels produce them (fed one-hot activations, so the
exact int32 block sum times the fp32 scale product is one weight), and (b)
the fp16 operand tiles that the prefill GEMM's dequantising warps write to
shared memory.  (a) must equal the closed form exactly (every weight of
these formats is exact in fp32); (b) must equal the round-to-nearest-even
fp16 of the closed form (numpy's float64 -> float16 conversion is the
reference rounding).  Every (sub-scale, code) pair of the 3-bit super-block
format and every code of the 4-bit formats is covered."""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import quantized_moe_expert_02_b200 as moe
from helpers import dev, pack_natural

pytestmark = pytest.mark.gpu

DEC, PF = moe.MOE_DQ_DECODE, moe.MOE_DQ_PREFILL


def export(fmt, path, nat, rows, cols):
    packed = pack_natural(fmt, dev(nat), rows, cols)
    if path == DEC:
        out = torch.full((rows, cols), float("nan"), device="cuda")
    else:
        out = torch.full((rows, cols), -1, dtype=torch.int16, device="cuda")
    moe.moe_dequant_path(fmt, path, packed, rows, cols, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def check(fmt, path, nat, rows, cols):
    ref = o.dequant(fmt, nat, rows, cols)
    got = export(fmt, path, nat, rows, cols)
    if path == DEC:
        assert np.array_equal(got.astype(np.float64), ref)
    else:
        want = ref.astype(np.float16).view(np.uint16)
        assert np.array_equal(got.view(np.uint16), want)


@pytest.mark.parametrize("path", [DEC, PF])
@pytest.mark.parametrize("fmt,rows,cols", [
    (synth.SB3_256, 128, 256), (synth.SB3_256, 256, 768),
    (synth.SB3_256, 1024, 3072),
    (synth.NL4_B32, 128, 64), (synth.NL4_B32, 128, 192),
    (synth.NL4_B32, 3072, 1024),
    (synth.Q4_B32, 128, 128), (synth.Q4_B32, 256, 256),
    (synth.NL3_256, 128, 256), (synth.NL3_256, 1024, 3072),
    (synth.SB2_256, 128, 256), (synth.SB2_256, 256, 768),
    (synth.SB2_256, 1024, 3072),
])
def test_hot_path_decoders_random(fmt, rows, cols, path):
    nat = synth.gen_tensor(13, 1, rows + cols, "up", fmt, rows, cols,
                           (0.002, 0.01))
    check(fmt, path, nat, rows, cols)


@pytest.mark.parametrize("fmt,rows,cols", [
    (synth.SB3_256, 16, 256), (synth.SB3_256, 48, 512),
    (synth.NL4_B32, 16, 64), (synth.Q4_B32, 48, 192),
    (synth.SB2_256, 16, 256), (synth.NL3_256, 48, 512),
])
def test_decode_decoders_small_tiles(fmt, rows, cols):
    """The decode path's 16-row tiles (no 128-row blocks needed)."""
    nat = synth.gen_tensor(17, 0, rows, "down", fmt, rows, cols,
                           (0.002, 0.01))
    check(fmt, DEC, nat, rows, cols)


def sb3_every_pair(rows=128, dmin=0.001, dmax=0.03):
    """Natural SB3 tensor [rows x 256] whose super-blocks cover every
    (sub-scale, code) pair at every position class: row r has sub-scales
    (r//8 + j) % 16 and codes (r + i) % 8."""
    codes, scales = bytearray(), bytearray()
    for r in range(rows):
        s, q = (r // 8) % 16, r % 8
        acc = 0
        for i in range(256):
            acc |= ((q + i) % 8) << (3 * i)
        codes += acc.to_bytes(96, "little")
        acc = 0
        for j in range(8):
            acc |= ((s + j) % 16) << (4 * j)
        scales += acc.to_bytes(4, "little")
    d = np.linspace(dmin, dmax, rows).astype(np.float16).tobytes()
    return np.frombuffer(bytes(codes) + bytes(scales) + d, np.uint8)


def nl3_every_triple(rows=256, dmin=0.001, dmax=0.03):
    """Natural NL3 tensor [rows x 256]: row r has sub-scales
    (r//16 + j) % 16, codes (r + i) % 8 and shift byte 0x55 or 0xAA
    (alternate blocks shifted, both phases), so every (s, q, e) occurs."""
    codes, scales, extra = bytearray(), bytearray(), bytearray()
    for r in range(rows):
        s, q = (r // 16) % 16, r % 8
        acc = 0
        for i in range(256):
            acc |= ((q + i) % 8) << (3 * i)
        codes += acc.to_bytes(96, "little")
        acc = 0
        for j in range(8):
            acc |= ((s + j) % 16) << (4 * j)
        scales += acc.to_bytes(4, "little")
        extra.append(0x55 if (r // 8) % 2 == 0 else 0xAA)
    d = np.linspace(dmin, dmax, rows).astype(np.float16).tobytes()
    return np.frombuffer(bytes(codes) + bytes(scales) + d + bytes(extra),
                         np.uint8)


@pytest.mark.parametrize("path", [DEC, PF])
def test_nl3_every_subscale_code_and_shift(path):
    nat = nl3_every_triple()
    trip = {(((r // 16) + i // 32) % 16, (r + i) % 8,
             ((0x55 if (r // 8) % 2 == 0 else 0xAA) >> (i // 32)) & 1)
            for r in range(256) for i in range(256)}
    assert len(trip) == 16 * 8 * 2
    check(synth.NL3_256, path, nat, 256, 256)


def sb2_every_pair(rows=128, dmin=0.001, dmax=0.03):
    """Natural SB2 tensor [rows x 256]: row r has sub-scales (r//8 + j) % 16
    and codes (r + i) % 4, so every (sub-scale, code) pair occurs at every
    position class."""
    codes, scales = bytearray(), bytearray()
    for r in range(rows):
        s, q = (r // 8) % 16, r % 4
        acc = 0
        for i in range(256):
            acc |= ((q + i) % 4) << (2 * i)
        codes += acc.to_bytes(64, "little")
        acc = 0
        for j in range(8):
            acc |= ((s + j) % 16) << (4 * j)
        scales += acc.to_bytes(4, "little")
    d = np.linspace(dmin, dmax, rows).astype(np.float16).tobytes()
    return np.frombuffer(bytes(codes) + bytes(scales) + d, np.uint8)


@pytest.mark.parametrize("path", [DEC, PF])
def test_sb2_every_subscale_and_code(path):
    nat = sb2_every_pair()
    pairs = {(((r // 8) + i // 32) % 16, (r + i) % 4)
             for r in range(128) for i in range(256)}
    assert len(pairs) == 16 * 4
    check(synth.SB2_256, path, nat, 128, 256)


def b32_every_code(rows=128, cols=128, dmin=0.001, dmax=0.03):
    """Natural Q4/NL4 tensor: weight (r, i) has code (r + i) % 16."""
    q = (np.arange(rows)[:, None] + np.arange(cols)[None, :]) % 16
    q = q.reshape(-1)
    codes = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)
    d = np.linspace(dmin, dmax, rows * cols // 32).astype(np.float16)
    return np.concatenate([codes, d.view(np.uint8)])


@pytest.mark.parametrize("path", [DEC, PF])
def test_sb3_every_subscale_and_code(path):
    nat = sb3_every_pair()
    # every (s, q) pair occurs in the fixture
    pairs = {(((r // 8) + i // 32) % 16, (r + i) % 8)
             for r in range(128) for i in range(256)}
    assert len(pairs) == 16 * 8
    check(synth.SB3_256, path, nat, 128, 256)


@pytest.mark.parametrize("path", [DEC, PF])
@pytest.mark.parametrize("fmt", [synth.NL4_B32, synth.Q4_B32])
def test_b32_every_code(fmt, path):
    nat = b32_every_code()
    ref = o.dequant(fmt, nat, 128, 128)
    cb = o.NL4_CODEBOOK if fmt == synth.NL4_B32 else np.arange(16) - 8.0
    d = o.fp16_to_f64(nat[128 * 128 // 2:]).reshape(128, 4)
    # all 16 code values appear in every row (the layout of the fixture)
    assert set(np.round(ref[0, :16] / d[0, 0]).tolist()) == set(cb.tolist())
    check(fmt, path, nat, 128, 128)


@pytest.mark.parametrize("path", [DEC, PF])
def test_small_scales(path):
    """Scales near the bottom of the fp16 range: the decode products stay
    exact in fp32; the prefill fp16 products round into fp16 subnormals."""
    check(synth.SB3_256, path, sb3_every_pair(dmin=2e-6, dmax=4e-4),
          128, 256)
    check(synth.NL4_B32, path, b32_every_code(dmin=2e-7, dmax=1e-5),
          128, 128)


def test_dequant_path_argument_errors():
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_dequant_path(synth.SB3_256, 7, buf, 128, 256, buf)
    assert ei.value.code == moe.MOE_ERR_INVALID
    with pytest.raises(moe.MoeError) as ei:     # prefill tiles: 128 rows
        moe.moe_dequant_path(synth.SB3_256, PF, buf, 16, 256, buf)
    assert ei.value.code == moe.MOE_ERR_SHAPE
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_dequant_path(synth.NL4_B32, DEC, buf, 16, 48, buf)
    assert ei.value.code == moe.MOE_ERR_SHAPE
