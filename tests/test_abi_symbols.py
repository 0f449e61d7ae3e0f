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
    assert moe.moe_ffn_workspace_bytes(3, 10, 3072, 1024) > 0
    assert moe.status_string(moe.MOE_ERR_CAPACITY).startswith("slot")
