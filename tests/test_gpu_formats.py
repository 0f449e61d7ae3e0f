"""GPU: seeded generator twin, pack + dequantisation export (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle as o
import synth
import synth.device as sdev
import quantized_moe_expert_02_b200 as moe
from helpers import dev, pack_natural, stream

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,layer,experts", [
    (synth.TINY, 0, list(range(16))),
    (synth.BIG, 3, [0, 257, 511]),
    (synth.NL3_SHAPE, 1, [0, 5, 63]),
    (synth.SB2_SHAPE, 2, [0, 9, 63]),
])
def test_device_generator_matches_host(shape, layer, experts):
    stride = shape.blob_stride
    buf = torch.zeros(len(experts) * stride, dtype=torch.uint8, device="cuda")
    for i, e in enumerate(experts):
        sdev.fill_experts(buf.data_ptr() + i * stride, stride, shape, 5, layer,
                          e, 1, stream())
    got = buf.cpu().numpy().reshape(len(experts), stride)
    for i, e in enumerate(experts):
        ref = synth.gen_expert_blob(shape, 5, layer, e)
        assert np.array_equal(got[i, :shape.blob_bytes],
                              ref[:shape.blob_bytes]), e


@pytest.mark.parametrize("fmt,rows,cols", [
    (synth.SB3_256, 16, 256), (synth.SB3_256, 48, 768),
    (synth.SB3_256, 1024, 3072),
    (synth.NL4_B32, 16, 64), (synth.NL4_B32, 48, 192),
    (synth.NL4_B32, 3072, 1024),
    (synth.Q4_B32, 32, 128), (synth.Q4_B32, 128, 256),
    (synth.NL3_256, 16, 256), (synth.NL3_256, 48, 768),
    (synth.NL3_256, 1024, 3072),
    (synth.SB2_256, 16, 256), (synth.SB2_256, 48, 768),
    (synth.SB2_256, 1024, 3072),
])
def test_pack_dequant_bit_exact(fmt, rows, cols):
    nat = synth.gen_tensor(11, 2, rows + cols, "up", fmt, rows, cols,
                           (0.002, 0.01))
    packed = pack_natural(fmt, dev(nat), rows, cols)
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    moe.moe_dequant(fmt, packed, rows, cols, out)
    torch.cuda.synchronize()
    ref = o.dequant(fmt, nat, rows, cols)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), ref)


def test_dequant_every_code_and_subscale():
    # natural SB3 tensor whose super-blocks cover every (s, q) pair
    rows, cols = 128, 256
    codes, scales = bytearray(), bytearray()
    for r in range(rows):
        s, q = r // 8, r % 8
        acc = 0
        for i in range(256):
            acc |= ((q + i) % 8) << (3 * i)
        codes += acc.to_bytes(96, "little")
        acc = 0
        for j in range(8):
            acc |= ((s + j) % 16) << (4 * j)
        scales += acc.to_bytes(4, "little")
    d = np.linspace(0.001, 0.03, rows).astype(np.float16).tobytes()
    nat = np.frombuffer(bytes(codes) + bytes(scales) + d, np.uint8)
    packed = pack_natural(synth.SB3_256, dev(nat), rows, cols)
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    moe.moe_dequant(synth.SB3_256, packed, rows, cols, out)
    assert np.array_equal(out.cpu().numpy().astype(np.float64),
                          o.dequant_sb3(nat, rows, cols))


def test_format_argument_errors():
    buf = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_pack_tensor(synth.SB3_256, buf, 16, 100, buf)
    assert ei.value.code == moe.MOE_ERR_SHAPE
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_dequant(9, buf, 16, 64, buf)
    assert ei.value.code == moe.MOE_ERR_INVALID
    assert moe.moe_tensor_bytes(synth.NL4_B32, 15, 64) == 0
