"""ctypes binding to libswattn.so: argument marshalling only.

Every step of the attention runs in the library's CUDA kernels.  If the library is missing
this module raises at first use; there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libswattn.so")

SW_OK, SW_EINVAL, SW_ESHAPE, SW_EALIGN, SW_ESTATE, SW_ECUDA = 0, -1, -2, -3, -4, -5
SW_STATUS_TIMEOUT, SW_STATUS_BAD_SLOT, SW_STATUS_OVERFLOW = 0x1, 0x2, 0x4
SW_OUT_BF16, SW_OUT_F32 = 0, 1
SW_SCHED_PERSISTENT, SW_SCHED_GRID, SW_SCHED_TRI, SW_SCHED_AUTO, SW_SCHED_PAIR = 0, 1, 2, 3, 4
SW_COMMIT_AUTO, SW_COMMIT_COPY, SW_COMMIT_TMA = 0, 1, 2

# every symbol include/swattn.h declares
EXPORTS = (
    "sw_attn_create", "sw_attn_create_ex", "sw_attn_workspace_bytes", "sw_attn_bind_workspace",
    "sw_attn_set_cond", "sw_attn_append_chunk", "sw_attn_forward", "sw_attn_forward_joint",
    "sw_attn_forward_commit", "sw_attn_append_chunk_batched",
    "sw_attn_table_ints",
    "sw_attn_get_table", "sw_attn_get_status", "sw_attn_reset", "sw_attn_destroy",
    "sw_attn_last_error", "sw_attn_cache_offsets", "sw_attn_forward_short_noalloc", "sw_attn_schedule_pieces",
    "sw_attn_table_host",
    "sw_attn_selftest_timeout", "sw_attn_schedule_for", "sw_attn_commit_kind",
)


class SwAttnConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("tokens_per_chunk", ctypes.c_int), ("W", ctypes.c_int), ("n_cond", ctypes.c_int),
                ("sink", ctypes.c_int), ("out_dtype", ctypes.c_int), ("scale", ctypes.c_float),
                ("max_short_q", ctypes.c_int), ("schedule", ctypes.c_int), ("commit_in_forward", ctypes.c_int),
                ("qk_fp8", ctypes.c_int), ("q_scale", ctypes.c_float), ("k_scale", ctypes.c_float),
                ("commit_path", ctypes.c_int), ("pv_fp8", ctypes.c_int), ("v_scale", ctypes.c_float)]


class SwAttnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libswattn error {code}: {msg}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libswattn.so not built at {LIB_PATH}; run __graft_entry__.build() "
                          "or python -m block_causal_attention_sliding_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.sw_attn_create.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(vp)]
    L.sw_attn_create.restype = i32
    L.sw_attn_create_ex.argtypes = [ctypes.POINTER(SwAttnConfig), ctypes.POINTER(vp)]
    L.sw_attn_create_ex.restype = i32
    L.sw_attn_workspace_bytes.argtypes = [vp]
    L.sw_attn_workspace_bytes.restype = sz
    L.sw_attn_bind_workspace.argtypes = [vp, vp, sz, vp]
    L.sw_attn_bind_workspace.restype = i32
    L.sw_attn_set_cond.argtypes = [vp, vp, vp, vp]
    L.sw_attn_set_cond.restype = i32
    L.sw_attn_append_chunk.argtypes = [vp, vp, vp, vp]
    L.sw_attn_append_chunk.restype = i32
    L.sw_attn_forward.argtypes = [vp, vp, vp, vp, vp, i32, vp]
    L.sw_attn_forward.restype = i32
    L.sw_attn_forward_joint.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    L.sw_attn_forward_joint.restype = i32
    L.sw_attn_forward_commit.argtypes = [vp, vp, vp, vp, vp, vp]
    L.sw_attn_forward_commit.restype = i32
    L.sw_attn_append_chunk_batched.argtypes = [vp, i32, vp, vp, vp]
    L.sw_attn_append_chunk_batched.restype = i32
    L.sw_attn_forward_short_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, vp]
    L.sw_attn_forward_short_noalloc.restype = i32
    L.sw_attn_selftest_timeout.argtypes = [vp, ctypes.c_int64, vp]
    L.sw_attn_selftest_timeout.restype = i32
    L.sw_attn_schedule_for.argtypes = [vp, i32]
    L.sw_attn_schedule_for.restype = i32
    L.sw_attn_commit_kind.argtypes = [vp]
    L.sw_attn_commit_kind.restype = i32
    L.sw_attn_table_ints.argtypes = [vp]
    L.sw_attn_table_ints.restype = i32
    L.sw_attn_get_table.argtypes = [vp, vp, vp]
    L.sw_attn_get_table.restype = i32
    L.sw_attn_get_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    L.sw_attn_get_status.restype = i32
    L.sw_attn_reset.argtypes = [vp, vp]
    L.sw_attn_reset.restype = i32
    L.sw_attn_destroy.argtypes = [vp]
    L.sw_attn_destroy.restype = None
    L.sw_attn_cache_offsets.argtypes = [vp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.sw_attn_cache_offsets.restype = i32
    L.sw_attn_schedule_pieces.argtypes = [i32, i32, i32, i32, i32, vp, i32]
    L.sw_attn_schedule_pieces.restype = i32
    L.sw_attn_table_host.argtypes = [i32] * 7 + [vp, i32]
    L.sw_attn_table_host.restype = i32
    L.sw_attn_last_error.argtypes = []
    L.sw_attn_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def check(rc: int) -> None:
    if rc != SW_OK:
        raise SwAttnError(rc, lib().sw_attn_last_error().decode(errors="replace"))
