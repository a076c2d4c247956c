"""ctypes view of libq4kv.so: structs and signatures of include/q4kv.h.

Loading never falls back to anything: if the library cannot be built or
loaded, the error propagates.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

from . import build as _build

c_int32, c_int64, c_size_t, c_void_p, c_float = (ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                                  ctypes.c_void_p, ctypes.c_float)

HEADER = os.path.join(_build.INCLUDE, "q4kv.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_DEVICE = range(6)
F16, BF16, F32 = 0, 1, 2
DEVERR_BLOCK_ID, DEVERR_SEQ_LEN, DEVERR_SLOT_ID, DEVERR_TIMEOUT, DEVERR_IMAGE, DEVERR_WIDTH = 1, 2, 4, 8, 16, 32


class PoolDesc(ctypes.Structure):
    _fields_ = [("head_dim", c_int32), ("n_kv_heads", c_int32), ("k_rotated", c_int32),
                ("n_q4_blocks", c_int32), ("n_q8_blocks", c_int32), ("value_format", c_int32),
                ("k_codes4", c_void_p), ("v_codes4", c_void_p),
                ("k_params4", c_void_p), ("v_params4", c_void_p),
                ("k_codes8", c_void_p), ("v_codes8", c_void_p),
                ("k_params8", c_void_p), ("v_params8", c_void_p),
                ("remap_mask", c_void_p), ("error_word", c_void_p),
                ("n_q2_blocks", c_int32), ("reserved", c_int32),
                ("k_codes2", c_void_p), ("v_codes2", c_void_p),
                ("k_params2", c_void_p), ("v_params2", c_void_p)]


class DecodePlan(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("n_q_heads", c_int32), ("n_kv_heads", c_int32),
                ("head_dim", c_int32), ("max_blocks_per_seq", c_int32), ("n_splits", c_int32),
                ("tokens_per_split", c_int32), ("kernel", c_int32), ("workspace_bytes", c_size_t)]


P = ctypes.POINTER
_SIGNATURES = {
    "q4kv_status_string": (ctypes.c_char_p, [c_int32]),
    "q4kv_abi_version": (c_int32, []),
    "q4kv_pool_array_bytes": (c_int32, [c_int32, c_int32, c_int64, c_int32, P(c_size_t), P(c_size_t)]),
    "q4kv_quantize_blocks": (c_int32, [P(PoolDesc), c_void_p, c_void_p, c_int32, c_int64, c_int64,
                                       c_void_p, c_void_p]),
    "q4kv_append_tokens": (c_int32, [P(PoolDesc), c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                     c_void_p, c_int64, c_int64, c_void_p, c_int32, c_void_p, c_void_p]),
    "q4kv_selftest_bounded_wait": (c_int32, [c_void_p, c_int32, c_void_p]),
    "q4kv_block_image_stride": (c_int32, [P(PoolDesc), P(c_size_t)]),
    "q4kv_export_blocks": (c_int32, [P(PoolDesc), c_void_p, c_int32, c_void_p, c_void_p]),
    "q4kv_import_blocks": (c_int32, [P(PoolDesc), c_void_p, c_void_p, c_int32, c_void_p]),
    "q4kv_card_max_bytes": (c_int32, [c_int32, c_int32, c_int64, P(c_size_t)]),
    "q4kv_card_encode": (c_int32, [c_int32, c_int32, c_int32, c_void_p, c_void_p, c_int32, c_int64, c_int64,
                                   c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "q4kv_card_decode": (c_int32, [c_void_p, c_size_t, c_int32, c_int32, c_int64, c_void_p, c_void_p, c_int32,
                                   c_void_p, c_void_p]),
    "q4kv_export_blocks_host_ids": (c_int32, [P(PoolDesc), c_void_p, c_int32, c_void_p, c_void_p]),
    "q4kv_import_blocks_host_ids": (c_int32, [P(PoolDesc), c_void_p, c_void_p, c_int32, c_void_p]),
    "q4kv_dequantize": (c_int32, [P(PoolDesc), c_void_p, c_int32, c_void_p, c_void_p, c_int32,
                                  c_int32, c_void_p]),
    "q4kv_invalidate_slots": (c_int32, [P(PoolDesc), c_void_p, c_int64, c_void_p]),
    "q4kv_block_absmean": (c_int32, [c_void_p, c_int32, c_int64, c_int64, c_int32, c_int32,
                                     c_void_p, c_void_p]),
    "q4kv_mixed_block_ids": (c_int32, [c_void_p, c_int32, c_int32, c_int32, c_int32, c_void_p,
                                       c_void_p]),
    "q4kv_decode_plan_make": (c_int32, [c_int32, c_int32, c_int32, c_int32, c_int32, c_int32,
                                        c_int32, P(DecodePlan)]),
    "q4kv_decode_attention": (c_int32, [P(PoolDesc), P(DecodePlan), c_void_p, c_int32, c_void_p,
                                        c_void_p, c_float, c_void_p, c_int32, c_void_p, c_size_t,
                                        c_void_p]),
    "q4kv_append_decode": (c_int32, [P(PoolDesc), P(DecodePlan), c_void_p, c_void_p, c_int32, c_int32,
                                     c_void_p, c_int64, c_int64, c_void_p, c_int32, c_void_p, c_void_p,
                                     c_float, c_void_p, c_int32, c_void_p, c_size_t, c_void_p]),
    "q4kv_read_device_error": (c_int32, [P(PoolDesc), P(ctypes.c_uint32), c_int32, c_void_p]),
    "q4kv_decode_attention_static_scratch": (c_int32, [P(PoolDesc), P(DecodePlan), c_void_p, c_int32,
                                                       c_void_p, c_void_p, c_float, c_void_p,
                                                       c_int32, c_void_p]),
}

_lib = None
_lock = threading.Lock()


def header_functions():
    """Names of the functions include/q4kv.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(q4kv_\w+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """The loaded library, building it first when missing or older than its sources."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            dll = ctypes.CDLL(path)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(dll, name)
                fn.restype = res
                fn.argtypes = args
            _lib = dll
    return _lib


class Q4KVError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib().q4kv_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != OK:
        raise Q4KVError(status, where)
