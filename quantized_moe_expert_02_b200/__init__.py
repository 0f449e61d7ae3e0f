"""Python binding of libmoe.so, the CUDA library declared in include/moe.h.

Argument marshalling only: every entry point keeps its C name and argument
order; tensors are passed by device pointer (``tensor.data_ptr()``), None
becomes NULL, and the stream defaults to torch's current CUDA stream.  A
non-zero status raises ``MoeError``.  Every step of the layer runs in the
library's kernels; there is no Python or CPU fallback, and importing this
package fails if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_double, c_int, c_int64, c_size_t, c_uint32, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID = 1
MOE_ERR_SHAPE = 2
MOE_ERR_UNSUPPORTED = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE = 5
MOE_ERR_CAPACITY = 6
MOE_ERR_TIMEOUT = 7
MOE_ERR_WORKSPACE = 8

MOE_Q4_B32 = 1
MOE_SB3_256 = 2
MOE_NL4_B32 = 3
MOE_NL3_256 = 4
MOE_SB2_256 = 5

MOE_DQ_DECODE = 1
MOE_DQ_PREFILL = 2


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")


class moe_layer_desc(ctypes.Structure):
    _fields_ = [("H", c_int), ("F", c_int), ("E", c_int),
                ("fmt_up_gate", c_int), ("fmt_down", c_int),
                ("pool", c_void_p), ("blob_stride", c_int64)]


_P = c_void_p
_SIGS = {
    "moe_tensor_bytes": (c_size_t, [c_int, c_int, c_int]),
    "moe_blob_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "moe_pack_tensor": (c_int, [c_int, _P, c_int, c_int, _P, _P]),
    "moe_dequant": (c_int, [c_int, _P, c_int, c_int, _P, _P]),
    "moe_dequant_path": (c_int, [c_int, c_int, _P, c_int, c_int, _P, _P]),
    "moe_route_topk": (c_int, [_P, c_int, c_int, _P, c_int, _P, c_int, _P,
                               _P, _P, _P]),
    "moe_group_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "moe_group_tokens": (c_int, [_P, c_int, c_int, c_int, _P, _P, _P, _P,
                                 _P, c_size_t, _P]),
    "moe_group_tokens_static": (c_int, [_P, c_int, c_int, c_int, _P, _P,
                                        _P, _P, _P, _P]),
    "moe_group_subset": (c_int, [_P, _P, c_int, _P, c_int, _P, _P, _P, _P,
                                 _P, _P]),
    "moe_slot_resolve": (c_int, [_P, c_int, c_int, c_int, _P, _P, _P, c_int,
                                 c_int, c_uint32, _P, _P, _P, _P, _P, _P]),
    "moe_ffn_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "moe_workspace_init": (c_int, [_P, c_size_t, _P]),
    "moe_expert_ffn_q": (c_int, [_P, _P, c_int, c_int, _P, _P, _P, _P, _P,
                                 _P, _P, c_size_t, _P]),
    "moe_expert_up_q": (c_int, [_P, _P, c_int, c_int, _P, _P, _P, _P, _P,
                                _P, c_size_t, _P]),
    "moe_expert_up_gemm_q": (c_int, [_P, c_int, c_int, _P, _P, _P, _P, _P,
                                     _P, c_size_t, _P]),
    "moe_expert_down_q": (c_int, [_P, c_int, c_int, _P, _P, _P, _P, _P, _P,
                                  _P, _P, _P, _P, _P, c_size_t, _P]),
    "moe_combine": (c_int, [_P, _P, c_int, c_int, c_int, _P, _P, _P, _P]),
    "moe_expert_ffn_combine_q": (c_int, [_P, _P, c_int, c_int, _P, _P, _P,
                                         _P, _P, _P, _P, _P, _P, _P,
                                         c_size_t, _P]),
    "moe_rmsnorm_bf16": (c_int, [_P, c_int, c_int, _P, _P]),
    "moe_layer_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int,
                                             c_int]),
    "moe_layer_forward": (c_int, [_P, _P, c_int, c_int, _P, _P, _P, _P, _P,
                                  _P, _P, _P, _P, _P, c_size_t, _P]),
    "moe_layer_forward_residual": (c_int, [_P, _P, c_int, c_int, _P, _P, _P,
                                           _P, _P, _P, _P, _P, _P, c_size_t,
                                           _P]),
    "moe_layer_route_residual": (c_int, [_P, _P, c_int, c_int, _P, _P, _P,
                                         _P, _P, _P, c_size_t, _P]),
    "moe_layer_ffn_residual": (c_int, [_P, _P, c_int, c_int, _P, _P, _P, _P,
                                       _P, _P, c_size_t, _P]),
    "moe_stage_table": (c_int, [_P, c_int, _P, _P]),
    "moe_layer_ffn_residual_staged": (c_int, [_P, _P, c_int, c_int, _P, _P,
                                              _P, _P, _P, _P, _P, _P, c_int,
                                              c_int, _P, c_int, c_int,
                                              c_int64, _P, c_size_t, _P]),
    "moe_stage_misses": (c_int, [_P, _P, _P, c_int, c_int, c_int, c_int, _P,
                                 _P, c_int, c_int, c_int64, c_int64, c_int64,
                                 _P, _P]),
    "moe_slot_resolve_dev": (c_int, [_P, c_int, c_int, c_int, _P, _P, _P,
                                     c_int, c_int, _P, _P, _P, _P, _P, _P,
                                     _P]),
    "moe_get_device_status": (c_int, [_P, _P, _P]),
    "moe_status_string": (ctypes.c_char_p, [c_int]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python quantized_moe_expert_02_b200/_build.py` or "
            "`python -c 'import __graft_entry__; __graft_entry__.build()'`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if isinstance(a, ctypes.Structure):
        return ctypes.addressof(a)
    return a.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(name: str, st: int) -> None:
    if st != MOE_OK:
        raise MoeError(name, st)


def status_string(code: int) -> str:
    return lib.moe_status_string(code).decode()


def moe_tensor_bytes(fmt, rows, cols) -> int:
    return lib.moe_tensor_bytes(fmt, rows, cols)


def moe_blob_bytes(fmt_up_gate, fmt_down, H, F) -> int:
    return lib.moe_blob_bytes(fmt_up_gate, fmt_down, H, F)


def moe_pack_tensor(fmt, natural, rows, cols, packed, stream=None):
    _check("moe_pack_tensor", lib.moe_pack_tensor(
        fmt, _ptr(natural), rows, cols, _ptr(packed), _stream(stream)))


def moe_dequant(fmt, packed, rows, cols, out, stream=None):
    _check("moe_dequant", lib.moe_dequant(
        fmt, _ptr(packed), rows, cols, _ptr(out), _stream(stream)))


def moe_dequant_path(fmt, path, packed, rows, cols, out, stream=None):
    _check("moe_dequant_path", lib.moe_dequant_path(
        fmt, path, _ptr(packed), rows, cols, _ptr(out), _stream(stream)))


def moe_route_topk(x, T, H, w_router, E, bias, k, topk_idx, topk_w,
                   logits_out, stream=None):
    _check("moe_route_topk", lib.moe_route_topk(
        _ptr(x), T, H, _ptr(w_router), E, _ptr(bias), k, _ptr(topk_idx),
        _ptr(topk_w), _ptr(logits_out), _stream(stream)))


def moe_group_workspace_bytes(T, k, E) -> int:
    return lib.moe_group_workspace_bytes(T, k, E)


def moe_group_tokens(topk_idx, T, k, E, expert_offsets, pair_ids, active,
                     n_active, ws, ws_bytes, stream=None):
    _check("moe_group_tokens", lib.moe_group_tokens(
        _ptr(topk_idx), T, k, E, _ptr(expert_offsets), _ptr(pair_ids),
        _ptr(active), _ptr(n_active), _ptr(ws), ws_bytes, _stream(stream)))


def moe_group_tokens_static(topk_idx, T, k, E, expert_offsets, pair_ids,
                            active, n_active, err, stream=None):
    _check("moe_group_tokens_static", lib.moe_group_tokens_static(
        _ptr(topk_idx), T, k, E, _ptr(expert_offsets), _ptr(pair_ids),
        _ptr(active), _ptr(n_active), _ptr(err), _stream(stream)))


def moe_group_subset(expert_offsets, pair_ids, E, experts, n, sub_offsets,
                     sub_pairs, sub_active, sub_n_active, err, stream=None):
    _check("moe_group_subset", lib.moe_group_subset(
        _ptr(expert_offsets), _ptr(pair_ids), E, _ptr(experts), n,
        _ptr(sub_offsets), _ptr(sub_pairs), _ptr(sub_active),
        _ptr(sub_n_active), _ptr(err), _stream(stream)))


def moe_slot_resolve(topk_idx, T, k, E, slot_table, slot_owner, last_use,
                     n_slots, slot_base, stamp, blob_index, miss_expert,
                     miss_slot, n_miss, err, stream=None):
    _check("moe_slot_resolve", lib.moe_slot_resolve(
        _ptr(topk_idx), T, k, E, _ptr(slot_table), _ptr(slot_owner),
        _ptr(last_use), n_slots, slot_base, stamp, _ptr(blob_index),
        _ptr(miss_expert), _ptr(miss_slot), _ptr(n_miss), _ptr(err),
        _stream(stream)))


def moe_slot_resolve_dev(topk_idx, T, k, E, slot_table, slot_owner,
                         last_use, n_slots, slot_base, stamp, blob_index,
                         miss_expert, miss_slot, n_miss, err, stream=None):
    _check("moe_slot_resolve_dev", lib.moe_slot_resolve_dev(
        _ptr(topk_idx), T, k, E, _ptr(slot_table), _ptr(slot_owner),
        _ptr(last_use), n_slots, slot_base, _ptr(stamp), _ptr(blob_index),
        _ptr(miss_expert), _ptr(miss_slot), _ptr(n_miss), _ptr(err),
        _stream(stream)))


def moe_ffn_workspace_bytes(T, k, H, F) -> int:
    return lib.moe_ffn_workspace_bytes(T, k, H, F)


def moe_layer_workspace_bytes(T, k, E, H, F) -> int:
    return lib.moe_layer_workspace_bytes(T, k, E, H, F)


def moe_workspace_init(ws, ws_bytes, stream=None):
    _check("moe_workspace_init", lib.moe_workspace_init(
        _ptr(ws), ws_bytes, _stream(stream)))


def moe_expert_ffn_q(desc, x, T, k, expert_offsets, pair_ids, active,
                     n_active, blob_index, y_pairs, ws, ws_bytes,
                     stream=None):
    _check("moe_expert_ffn_q", lib.moe_expert_ffn_q(
        _ptr(desc), _ptr(x), T, k, _ptr(expert_offsets), _ptr(pair_ids),
        _ptr(active), _ptr(n_active), _ptr(blob_index), _ptr(y_pairs),
        _ptr(ws), ws_bytes, _stream(stream)))


def moe_expert_up_q(desc, x, T, k, expert_offsets, pair_ids, active,
                    n_active, blob_index, ws, ws_bytes, stream=None):
    _check("moe_expert_up_q", lib.moe_expert_up_q(
        _ptr(desc), _ptr(x), T, k, _ptr(expert_offsets), _ptr(pair_ids),
        _ptr(active), _ptr(n_active), _ptr(blob_index), _ptr(ws), ws_bytes,
        _stream(stream)))


def moe_expert_up_gemm_q(desc, T, k, expert_offsets, pair_ids, active,
                         n_active, blob_index, ws, ws_bytes, stream=None):
    _check("moe_expert_up_gemm_q", lib.moe_expert_up_gemm_q(
        _ptr(desc), T, k, _ptr(expert_offsets), _ptr(pair_ids), _ptr(active),
        _ptr(n_active), _ptr(blob_index), _ptr(ws), ws_bytes,
        _stream(stream)))


def moe_expert_down_q(desc, T, k, expert_offsets, pair_ids, active, n_active,
                      blob_index, y_pairs, topk_w, residual, out, out_bf16,
                      ws, ws_bytes, stream=None):
    _check("moe_expert_down_q", lib.moe_expert_down_q(
        _ptr(desc), T, k, _ptr(expert_offsets), _ptr(pair_ids), _ptr(active),
        _ptr(n_active), _ptr(blob_index), _ptr(y_pairs), _ptr(topk_w),
        _ptr(residual), _ptr(out), _ptr(out_bf16), _ptr(ws), ws_bytes,
        _stream(stream)))


def moe_combine(y_pairs, topk_w, T, k, H, residual, out, out_bf16,
                stream=None):
    _check("moe_combine", lib.moe_combine(
        _ptr(y_pairs), _ptr(topk_w), T, k, H, _ptr(residual), _ptr(out),
        _ptr(out_bf16), _stream(stream)))


def moe_expert_ffn_combine_q(desc, x, T, k, expert_offsets, pair_ids, active,
                             n_active, blob_index, topk_w, residual, out,
                             out_bf16, ws, ws_bytes, stream=None):
    _check("moe_expert_ffn_combine_q", lib.moe_expert_ffn_combine_q(
        _ptr(desc), _ptr(x), T, k, _ptr(expert_offsets), _ptr(pair_ids),
        _ptr(active), _ptr(n_active), _ptr(blob_index), _ptr(topk_w),
        _ptr(residual), _ptr(out), _ptr(out_bf16), _ptr(ws), ws_bytes,
        _stream(stream)))


def moe_rmsnorm_bf16(r, T, H, x_out, stream=None):
    _check("moe_rmsnorm_bf16", lib.moe_rmsnorm_bf16(
        _ptr(r), T, H, _ptr(x_out), _stream(stream)))


def moe_layer_forward(desc, x, T, k, w_router, bias, blob_index, residual,
                      out, out_bf16, topk_idx, topk_w, logits_out, ws,
                      ws_bytes, stream=None):
    _check("moe_layer_forward", lib.moe_layer_forward(
        _ptr(desc), _ptr(x), T, k, _ptr(w_router), _ptr(bias),
        _ptr(blob_index), _ptr(residual), _ptr(out), _ptr(out_bf16),
        _ptr(topk_idx), _ptr(topk_w), _ptr(logits_out), _ptr(ws), ws_bytes,
        _stream(stream)))


def moe_layer_forward_residual(desc, r, T, k, w_router, bias, blob_index,
                               r_out, out_bf16, topk_idx, topk_w, logits_out,
                               ws, ws_bytes, stream=None):
    _check("moe_layer_forward_residual", lib.moe_layer_forward_residual(
        _ptr(desc), _ptr(r), T, k, _ptr(w_router), _ptr(bias),
        _ptr(blob_index), _ptr(r_out), _ptr(out_bf16), _ptr(topk_idx),
        _ptr(topk_w), _ptr(logits_out), _ptr(ws), ws_bytes, _stream(stream)))


def moe_layer_route_residual(desc, r, T, k, w_router, bias, topk_idx, topk_w,
                             logits_out, ws, ws_bytes, stream=None):
    _check("moe_layer_route_residual", lib.moe_layer_route_residual(
        _ptr(desc), _ptr(r), T, k, _ptr(w_router), _ptr(bias),
        _ptr(topk_idx), _ptr(topk_w), _ptr(logits_out), _ptr(ws), ws_bytes,
        _stream(stream)))


def moe_layer_ffn_residual(desc, r, T, k, topk_idx, topk_w, blob_index,
                           r_out, out_bf16, ws, ws_bytes, stream=None):
    _check("moe_layer_ffn_residual", lib.moe_layer_ffn_residual(
        _ptr(desc), _ptr(r), T, k, _ptr(topk_idx), _ptr(topk_w),
        _ptr(blob_index), _ptr(r_out), _ptr(out_bf16), _ptr(ws), ws_bytes,
        _stream(stream)))


def moe_layer_ffn_residual_staged(desc, r, T, k, topk_idx, topk_w,
                                  blob_index, r_out, out_bf16, n_miss,
                                  miss_expert, miss_slot, layer, L, table,
                                  slot_base, n_slots, pool_slots, ws,
                                  ws_bytes, stream=None):
    _check("moe_layer_ffn_residual_staged",
           lib.moe_layer_ffn_residual_staged(
               _ptr(desc), _ptr(r), T, k, _ptr(topk_idx), _ptr(topk_w),
               _ptr(blob_index), _ptr(r_out), _ptr(out_bf16), _ptr(n_miss),
               _ptr(miss_expert), _ptr(miss_slot), layer, L, _ptr(table),
               slot_base, n_slots, pool_slots, _ptr(ws), ws_bytes,
               _stream(stream)))


def moe_stage_table(host_blob, table, stream=None):
    """host_blob: host addresses (0 = not stored), one per table entry."""
    n = len(host_blob)
    arr = (c_void_p * n)(*[int(a) or None for a in host_blob])
    _check("moe_stage_table", lib.moe_stage_table(
        arr, n, _ptr(table), _stream(stream)))


def moe_stage_misses(n_miss, miss_expert, miss_slot, P, layer, L, E, table,
                     pool, slot_base, n_slots, pool_slots, blob_stride,
                     blob_bytes, err, stream=None):
    _check("moe_stage_misses", lib.moe_stage_misses(
        _ptr(n_miss), _ptr(miss_expert), _ptr(miss_slot), P, layer, L, E,
        _ptr(table), _ptr(pool), slot_base, n_slots, pool_slots, blob_stride,
        blob_bytes, _ptr(err), _stream(stream)))


def moe_get_device_status(ws, stream=None) -> int:
    """Synchronises the stream; returns the device error word (0 = none)
    and clears it."""
    err = ctypes.c_int32(0)
    lib.moe_get_device_status(_ptr(ws), ctypes.byref(err), _stream(stream))
    return err.value
