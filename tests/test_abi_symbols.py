"""CPU: the C-ABI library loads, exports every function include/moe.h
declares, and the Python binding wraps each of them under the same name."""
import ctypes
import os
import re

import quantized_moe_expert_02_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(
        r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["moe_route_topk", "moe_group_tokens", "moe_slot_resolve",
              "moe_expert_ffn_q", "moe_combine", "moe_pack_tensor",
              "moe_dequant", "moe_layer_forward"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_binding_wraps_every_symbol():
    for n in declared_functions():
        if n == "moe_status_string":
            continue
        assert callable(getattr(moe, n)), n


def test_host_side_queries_without_gpu():
    assert moe.moe_tensor_bytes(moe.MOE_SB3_256, 1024, 3072) == 1253376
    assert moe.moe_tensor_bytes(moe.MOE_NL4_B32, 3072, 1024) == 1769472
    assert moe.moe_blob_bytes(moe.MOE_SB3_256, moe.MOE_NL4_B32, 3072,
                              1024) == 4276224
    assert moe.moe_tensor_bytes(moe.MOE_SB3_256, 16, 100) == 0
    # 16 x 256 tiles: SB3 1632 B, NL3 1648 B, SB2 1120 B
    assert moe.moe_tensor_bytes(moe.MOE_NL3_256, 1024, 3072) == 64 * 12 * 1648
    assert moe.moe_tensor_bytes(moe.MOE_SB2_256, 1024, 3072) == 64 * 12 * 1120
    assert moe.moe_tensor_bytes(moe.MOE_SB2_256, 8, 256) == 0
    assert moe.moe_tensor_bytes(6, 1024, 3072) == 0
    assert moe.moe_ffn_workspace_bytes(3, 10, 3072, 1024) > 0
    assert moe.status_string(moe.MOE_ERR_CAPACITY).startswith("slot")


def test_stage_argument_errors_without_gpu():
    """The in-stream staging calls reject bad arguments on the host, before
    any CUDA call (fake non-null addresses are never dereferenced)."""
    f = 4096   # a 16-byte aligned stand-in address
    lib = moe.lib

    def stage(**kw):
        a = dict(n_miss=f, miss_expert=f, miss_slot=f, P=30, layer=0, L=48,
                 E=512, table=f, pool=f, slot_base=0, n_slots=240,
                 pool_slots=4644,
                 blob_stride=4276224, blob_bytes=4276224, err=f, stream=None)
        a.update(kw)
        return lib.moe_stage_misses(
            a["n_miss"], a["miss_expert"], a["miss_slot"], a["P"],
            a["layer"], a["L"], a["E"], a["table"], a["pool"],
            a["slot_base"], a["n_slots"], a["pool_slots"], a["blob_stride"],
            a["blob_bytes"], a["err"], a["stream"])

    assert stage(n_miss=None) == moe.MOE_ERR_INVALID
    assert stage(table=None) == moe.MOE_ERR_INVALID
    assert stage(pool=None) == moe.MOE_ERR_INVALID
    assert stage(P=0) == moe.MOE_ERR_SHAPE
    assert stage(layer=48) == moe.MOE_ERR_SHAPE           # layer >= L
    assert stage(layer=-1) == moe.MOE_ERR_SHAPE
    assert stage(blob_bytes=4276224 + 8) == moe.MOE_ERR_SHAPE   # not 16n
    assert stage(blob_stride=4276224 - 16) == moe.MOE_ERR_SHAPE  # < blob
    assert stage(pool=f + 8) == moe.MOE_ERR_SHAPE           # misaligned
    assert stage(pool_slots=0) == moe.MOE_ERR_SHAPE
    assert stage(n_slots=0) == moe.MOE_ERR_SHAPE
    # the layer's partition must lie inside the pool
    assert stage(slot_base=4644 - 59, n_slots=60) == moe.MOE_ERR_SHAPE
    assert lib.moe_slot_resolve_dev(f, 3, 10, 512, f, f, f, 60, 0, None, f,
                                    f, f, f, f, None) == moe.MOE_ERR_INVALID
    table = (ctypes.c_void_p * 1)(None)
    assert lib.moe_stage_table(table, 0, f, None) == moe.MOE_ERR_INVALID
    assert lib.moe_stage_table(None, 1, f, None) == moe.MOE_ERR_INVALID
    # an unaligned host address is refused before it is looked up
    table[0] = f + 4
    assert lib.moe_stage_table(table, 1, f, None) == moe.MOE_ERR_INVALID


def test_staged_ffn_argument_errors_without_gpu():
    """moe_layer_ffn_residual_staged rejects bad arguments on the host."""
    f = 4096
    lib = moe.lib
    desc = moe.moe_layer_desc(H=3072, F=1024, E=512,
                              fmt_up_gate=moe.MOE_SB3_256,
                              fmt_down=moe.MOE_NL4_B32, pool=f,
                              blob_stride=4276224)
    ws_b = moe.moe_layer_workspace_bytes(3, 10, 512, 3072, 1024)

    def call(**kw):
        a = dict(n_miss=f, table=f, layer=0, L=48, slot_base=0, n_slots=60,
                 pool_slots=4644, ws=f, ws_bytes=ws_b)
        a.update(kw)
        return lib.moe_layer_ffn_residual_staged(
            ctypes.addressof(desc), f, 3, 10, f, f, f, f, None, a["n_miss"],
            f, f, a["layer"], a["L"], a["table"], a["slot_base"],
            a["n_slots"], a["pool_slots"], a["ws"], a["ws_bytes"], None)

    assert call(n_miss=None) == moe.MOE_ERR_INVALID
    assert call(table=None) == moe.MOE_ERR_INVALID
    assert call(layer=48) == moe.MOE_ERR_SHAPE
    assert call(slot_base=4600, n_slots=60) == moe.MOE_ERR_SHAPE
    assert call(ws_bytes=16) == moe.MOE_ERR_WORKSPACE
