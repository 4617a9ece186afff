"""ctypes declarations of the C ABI in include/moe_rt.h and the library loader.

The shared library is built in-tree (``python -m combine_moe_route_tokens_b200.build``).
There is no fallback: if the library is missing or fails to load, every call
raises.
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
LIB_PATH = os.path.join(PKG_DIR, "libmoert.so")
HEADER_PATH = os.path.join(ROOT, "include", "moe_rt.h")

MOE_OK = 0
MOE_ERR_INVALID = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_SCRATCH_LIMIT = -4
MOE_NOALLOC_MAX_E_LOG = 512
MOE_MAX_TP = 8
MOE_MAX_DEDUP_RANKS = 32

MOE_DEV_EXPERT_RANGE = 0x1
MOE_DEV_TIMEOUT = 0x2
MOE_DEV_ROW_RANGE = 0x4

MOE_FLAG_NONE = 0
MOE_FLAG_TEST_WAIT_TIMEOUT = 0x80000000
MOE_FLAG_DISPATCH_BULK_COPY = 0x1

ABI_VERSION = 6


class MoeProblem(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int64),
        ("H", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("E_log", ctypes.c_int32),
        ("num_replicas", ctypes.c_int32),
        ("R", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("row_align", ctypes.c_int32),
        ("tp_size", ctypes.c_int32),
        ("tp_rank", ctypes.c_int32),
    ]


LAYOUT_FIELDS = (
    "phys_idx",
    "ordinal",
    "dest_row",
    "drop_mask",
    "counts_logical",
    "placement",
    "counts_raw",
    "tokens_per_expert",
    "expert_offsets",
    "input_splits",
    "output_splits",
    "rank_offsets",
    "counters",
    "num_rows",
    "status",
    "row_token",
    "row_slot",
    "row_local_expert",
    "row_prob",
    "pad_mask",
    "local_topk",
)


class MoeLayout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in LAYOUT_FIELDS]


DEDUP_FIELDS = (
    "num_tokens_per_rank",
    "recv_rank_offsets",
    "num_recv",
    "is_token_in_rank",
    "token_rank_row",
    "recv_src_token",
    "recv_topk_idx",
    "recv_topk_weights",
    "recv_routing_map",
    "recv_probs",
    "recv_pad_mask",
    "status",
)


class MoeDedup(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in DEDUP_FIELDS]


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn} failed: {code} ({text})")
        self.code = code


_lib: Optional[ctypes.CDLL] = None

_VP = ctypes.c_void_p
_PP = ctypes.POINTER(MoeProblem)
_PL = ctypes.POINTER(MoeLayout)
_PD = ctypes.POINTER(MoeDedup)

class MoeIpcBuffer(ctypes.Structure):
    _fields_ = [
        ("handle", ctypes.c_ubyte * 64),
        ("offset", ctypes.c_uint64),
        ("bytes", ctypes.c_uint64),
        ("device", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


_SIGNATURES = {
    "moe_abi_version": (ctypes.c_int, []),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_rows_max": (ctypes.c_int64, [_PP]),
    "moe_layout_workspace_bytes": (ctypes.c_int, [_PP, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_route_topk": (ctypes.c_int, [_VP, _VP, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP]),
    "moe_dispatch_layout": (ctypes.c_int, [_PP, _VP, _VP, _PL, _VP, ctypes.c_size_t, _VP]),
    "moe_dispatch_layout_noalloc": (ctypes.c_int, [_PP, _VP, _VP, _PL, _VP]),
    "moe_dispatch": (ctypes.c_int, [_PP, _VP, _VP, _PL, _VP, ctypes.c_size_t, _VP, _VP, _VP]),
    "moe_ep_publish_offsets": (ctypes.c_int, [_PP, _VP, ctypes.c_int32, _VP, _VP]),
    "moe_ipc_export": (ctypes.c_int, [_VP, ctypes.c_size_t, ctypes.POINTER(MoeIpcBuffer)]),
    "moe_ipc_open": (ctypes.c_int, [ctypes.POINTER(MoeIpcBuffer), ctypes.POINTER(ctypes.c_void_p),
                                    ctypes.POINTER(ctypes.c_void_p)]),
    "moe_ipc_close": (ctypes.c_int, [_VP]),
    "moe_permute": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP]),
    "moe_combine": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP, _VP]),
    "moe_restore_combined": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP, _VP]),
    "moe_permute_backward": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP]),
    "moe_combine_backward": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_ep_recv_rows_max": (ctypes.c_int64, [_PP]),
    "moe_ep_plan": (ctypes.c_int, [_PP, _VP, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP]),
    "moe_ep_dispatch": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP, _VP]),
    "moe_ep_combine": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP, _VP, _VP]),
    "moe_ep_combine_backward": (ctypes.c_int, [_PP, _PL, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_dedup_rows_max": (ctypes.c_int64, [_PP]),
    "moe_dedup_workspace_bytes": (ctypes.c_int, [_PP, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_dedup_layout": (ctypes.c_int, [_PP, _PL, _VP, _PD, _VP, ctypes.c_size_t, _VP]),
    "moe_dedup_dispatch": (ctypes.c_int, [_PP, _PD, _VP, _VP, _VP]),
    "moe_dedup_combine_local": (ctypes.c_int, [_PP, _PL, _PD, _VP, _VP, _VP, _VP]),
    "moe_dedup_combine": (ctypes.c_int, [_PP, _PD, _VP, _VP, _VP]),
}


def declared_functions(header: str = HEADER_PATH) -> list:
    """Names of the functions include/moe_rt.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """The loaded libmoert.so (loaded once)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m combine_moe_route_tokens_b200.build` "
                "(there is no fallback implementation)"
            )
        handle = ctypes.CDLL(LIB_PATH)
        for name, (restype, argtypes) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = restype
            fn.argtypes = argtypes
        version = handle.moe_abi_version()
        if version != ABI_VERSION:
            raise RuntimeError(f"libmoert.so ABI version {version}, binding expects {ABI_VERSION}")
        _lib = handle
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def check(fn: str, code: int) -> None:
    if code != MOE_OK:
        raise MoeError(fn, code, status_string(code))
