"""ctypes wrapper over the plain-C oracle (moe_oracle.c) — TEST INFRASTRUCTURE.

numpy arrays in, numpy arrays out. bf16 tensors travel as uint16 bit patterns.
The C library is built by :func:`build` with ``-O2 -ffp-contract=off`` and no
fast-math, single-threaded.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_HDR = os.path.join(_HERE, "moe_oracle.h")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_OMP_SRC = os.path.join(_HERE, "moe_oracle_omp.c")
_OMP_LIB = os.path.join(_HERE, "libmoe_oracle_omp.so")
# MOE_ORACLE_LIB names a prebuilt variant of the library to load instead; the
# mutation tests build copies of moe_oracle.c with one planted mistake each and
# check that the pins reject every one of them.
_LIB_OVERRIDE = os.environ.get("MOE_ORACLE_LIB") or None

COUNTER_NAMES = (
    "assignments_total",
    "kept",
    "dropped",
    "padded",
    "split_sum_in",
    "split_sum_out",
    "num_rows",
    "error",
)


def library_path() -> str:
    return _LIB_OVERRIDE or _LIB


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmoe_oracle.so`` (gcc, no fast-math, no FP contraction)."""
    if _LIB_OVERRIDE:  # a prebuilt variant: nothing to compile
        return _LIB_OVERRIDE
    stale = (
        not os.path.exists(_LIB)
        or os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    )
    if force or stale:
        cmd = [
            os.environ.get("CC", "gcc"),
            "-O2",
            "-std=c11",
            "-ffp-contract=off",
            "-fno-fast-math",
            "-fPIC",
            "-shared",
            "-Wall",
            "-o",
            _LIB + ".tmp",
            _SRC,
            "-lm",
        ]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def build_omp(force: bool = False) -> str:
    """Compile the all-cores variant ``oracle/libmoe_oracle_omp.so``: moe_oracle_omp.c (OpenMP over
    tokens for route, permute and combine, calling the unchanged oracle functions) linked with its
    own copy of moe_oracle.c, built with the same flags as the oracle plus -fopenmp."""
    srcs = (_SRC, _HDR, _OMP_SRC)
    stale = not os.path.exists(_OMP_LIB) or os.path.getmtime(_OMP_LIB) < max(os.path.getmtime(x) for x in srcs)
    if force or stale:
        # the first compiler that has an OpenMP runtime ($CC may be a toolchain without libgomp)
        last = None
        for cc in dict.fromkeys([os.environ.get("CC", "gcc"), "gcc", "/usr/bin/gcc"]):
            cmd = [cc, "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
                   "-Wall", "-o", _OMP_LIB + ".tmp", _OMP_SRC, _SRC, "-lm"]
            last = subprocess.run(cmd, capture_output=True, text=True)
            if last.returncode == 0:
                break
        if last.returncode != 0:
            raise RuntimeError("no C compiler with OpenMP found: " + last.stderr[-500:])
        os.replace(_OMP_LIB + ".tmp", _OMP_LIB)
    return _OMP_LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int64),
        ("k", ctypes.c_int32),
        ("E_log", ctypes.c_int32),
        ("num_replicas", ctypes.c_int32),
        ("R", ctypes.c_int32),
        ("C", ctypes.c_int32),
        ("align", ctypes.c_int32),
        ("tp_size", ctypes.c_int32),
        ("tp_rank", ctypes.c_int32),
    ]


_P = ctypes.c_void_p


class _LayoutOut(ctypes.Structure):
    _fields_ = [
        ("phys_idx", _P),
        ("ordinal", _P),
        ("logical_ordinal", _P),
        ("dest_row", _P),
        ("drop_mask", _P),
        ("counts_logical", _P),
        ("placement", _P),
        ("counts_raw", _P),
        ("tokens_per_expert", _P),
        ("expert_offsets", _P),
        ("input_splits", _P),
        ("output_splits", _P),
        ("rank_offsets", _P),
        ("counters", _P),
        ("num_rows", _P),
        ("row_token", _P),
        ("row_slot", _P),
        ("row_local_expert", _P),
        ("row_prob", _P),
        ("pad_mask", _P),
        ("local_topk", _P),
    ]


class _DedupOut(ctypes.Structure):
    _fields_ = [
        ("num_tokens_per_rank", _P),
        ("recv_rank_offsets", _P),
        ("num_recv", _P),
        ("is_token_in_rank", _P),
        ("token_rank_row", _P),
        ("recv_src_token", _P),
        ("recv_topk_idx", _P),
        ("recv_topk_weights", _P),
        ("recv_routing_map", _P),
        ("recv_probs", _P),
        ("recv_pad_mask", _P),
    ]


_lib_handle: Optional[ctypes.CDLL] = None


def _lib() -> ctypes.CDLL:
    global _lib_handle
    if _lib_handle is None:
        build()
        lib = ctypes.CDLL(library_path())
        lib.oracle_problem_valid.restype = ctypes.c_int
        lib.oracle_problem_valid.argtypes = [ctypes.POINTER(_Problem)]
        lib.oracle_rows_max.restype = ctypes.c_int64
        lib.oracle_rows_max.argtypes = [ctypes.POINTER(_Problem)]
        lib.oracle_num_experts.restype = ctypes.c_int32
        lib.oracle_num_experts.argtypes = [ctypes.POINTER(_Problem)]
        lib.oracle_route_topk.restype = None
        lib.oracle_route_topk.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P]
        lib.oracle_layout.restype = ctypes.c_int
        lib.oracle_layout.argtypes = [ctypes.POINTER(_Problem), _P, _P, ctypes.POINTER(_LayoutOut)]
        lib.oracle_permute.restype = None
        lib.oracle_permute.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, _P, ctypes.c_int64, _P, _P]
        lib.oracle_combine.restype = None
        lib.oracle_combine.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, _P, _P, _P, _P]
        lib.oracle_restore_combined.restype = None
        lib.oracle_restore_combined.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, ctypes.c_int32, _P, _P, _P,
                                                _P]
        lib.oracle_permute_backward.restype = None
        lib.oracle_permute_backward.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, _P, _P, _P]
        lib.oracle_combine_backward.restype = None
        lib.oracle_combine_backward.argtypes = [
            ctypes.POINTER(_Problem),
            ctypes.c_int32,
            ctypes.c_int64,
            _P,
            _P,
            _P,
            _P,
            _P,
            _P,
            _P,
        ]
        lib.oracle_dedup_rows_max.restype = ctypes.c_int64
        lib.oracle_dedup_rows_max.argtypes = [ctypes.POINTER(_Problem)]
        lib.oracle_dedup_layout.restype = ctypes.c_int
        lib.oracle_dedup_layout.argtypes = [ctypes.POINTER(_Problem), _P, _P, _P, ctypes.POINTER(_DedupOut)]
        lib.oracle_dedup_combine_local.restype = None
        lib.oracle_dedup_combine_local.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, ctypes.c_int64, _P, _P,
                                                   _P, _P, _P, _P, _P]
        lib.oracle_bf16_from_f32.restype = ctypes.c_uint16
        lib.oracle_bf16_from_f32.argtypes = [ctypes.c_float]
        _lib_handle = lib
    return _lib_handle


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _problem(N, k, E_log, R, C=0, num_replicas=0, align=0, tp_size=0, tp_rank=0) -> _Problem:
    p = _Problem(N=int(N), k=int(k), E_log=int(E_log), num_replicas=int(num_replicas), R=int(R), C=int(C),
                 align=int(align), tp_size=int(tp_size), tp_rank=int(tp_rank))
    if not _lib().oracle_problem_valid(ctypes.byref(p)):
        raise ValueError(f"invalid problem N={N} k={k} E_log={E_log} R={R} C={C} replicas={num_replicas} "
                         f"align={align} tp={tp_rank}/{tp_size}")
    return p


def rows_max(N, k, E_log, R, C=0, num_replicas=0, align=0, tp_size=0, tp_rank=0) -> int:
    p = _problem(N, k, E_log, R, C, num_replicas, align, tp_size, tp_rank)
    return int(_lib().oracle_rows_max(ctypes.byref(p)))


def num_experts(E_log, num_replicas=0) -> int:
    return int(E_log + num_replicas)


def bf16_from_f32(x: float) -> int:
    return int(_lib().oracle_bf16_from_f32(float(x)))


def route_topk(logits: np.ndarray, k: int, token_mask: Optional[np.ndarray] = None):
    """Softmax over E in double, top-k by descending logit (ties: lower id). Returns (idx int32, probs f32)."""
    logits = _c(logits, np.float32)
    N, E = logits.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    mask = None if token_mask is None else _c(token_mask, np.uint8)
    idx = np.empty((N, k), dtype=np.int32)
    probs = np.empty((N, k), dtype=np.float32)
    _lib().oracle_route_topk(_ptr(logits), _ptr(mask), N, E, k, _ptr(idx), _ptr(probs))
    return idx, probs


def layout(topk_idx: np.ndarray, topk_probs: Optional[np.ndarray], *, E_log: int, R: int, C: int = 0,
           num_replicas: int = 0, align: int = 0, tp_size: int = 0, tp_rank: int = 0,
           local_topk: bool = True) -> dict:
    """Every dispatch-layout output as a dict of numpy arrays (see moe_oracle.c)."""
    topk_idx = _c(topk_idx, np.int32)
    N, k = topk_idx.shape
    p = _problem(N, k, E_log, R, C, num_replicas, align, tp_size, tp_rank)
    lib = _lib()
    E = E_log + num_replicas
    NK = N * k
    RM = int(lib.oracle_rows_max(ctypes.byref(p)))
    probs = None if topk_probs is None else _c(topk_probs, np.float32)
    out = {
        "phys_idx": np.empty(NK, np.int32),
        "ordinal": np.empty(NK, np.int32),
        "logical_ordinal": np.empty(NK, np.int32),
        "dest_row": np.empty(NK, np.int32),
        "drop_mask": np.empty(NK, np.uint8),
        "counts_logical": np.empty(E_log, np.int32),
        "placement": np.empty(E_log, np.int32),
        "counts_raw": np.empty(E, np.int32),
        "tokens_per_expert": np.empty(E, np.int32),
        "expert_offsets": np.empty(E + 1, np.int32),
        "input_splits": np.empty(R, np.int32),
        "output_splits": np.empty(R, np.int32),
        "rank_offsets": np.empty(R + 1, np.int32),
        "counters": np.empty(8, np.int32),
        "num_rows": np.empty(1, np.int32),
        "row_token": np.empty(RM, np.int32),
        "row_slot": np.empty(RM, np.int32),
        "row_local_expert": np.empty(RM, np.int32),
        "row_prob": np.empty(RM, np.float32),
        "pad_mask": np.empty(RM, np.uint8),
        "local_topk": np.empty(R * NK, np.int32) if local_topk else None,
    }
    o = _LayoutOut(**{name: _ptr(arr) for name, arr in out.items()})
    rc = lib.oracle_layout(ctypes.byref(p), _ptr(topk_idx), _ptr(probs), ctypes.byref(o))
    if rc != 0:
        raise ValueError("oracle_layout rejected the problem")
    for name in ("phys_idx", "ordinal", "logical_ordinal", "dest_row", "drop_mask"):
        out[name] = out[name].reshape(N, k)
    if out["local_topk"] is not None:
        out["local_topk"] = out["local_topk"].reshape(R, N, k)
    else:
        del out["local_topk"]
    out["rows_max"] = RM
    out["E"] = E
    return out


def dedup_layout(L: dict, topk_probs: Optional[np.ndarray], *, E_log: int, R: int, num_replicas: int = 0) -> dict:
    """DeepEP-style one-row-per-(token, rank) view of a layout (see moe_oracle.c)."""
    phys = _c(L["phys_idx"], np.int32)
    dest = _c(L["dest_row"], np.int32)
    N, k = phys.shape
    p = _Problem(N=N, k=k, E_log=E_log, num_replicas=num_replicas, R=R, C=0)
    lib = _lib()
    RM = int(lib.oracle_dedup_rows_max(ctypes.byref(p)))
    E_loc = (E_log + num_replicas) // R
    probs = None if topk_probs is None else _c(topk_probs, np.float32)
    out = {
        "num_tokens_per_rank": np.empty(R, np.int32),
        "recv_rank_offsets": np.empty(R + 1, np.int32),
        "num_recv": np.empty(1, np.int32),
        "is_token_in_rank": np.empty(N * R, np.uint8),
        "token_rank_row": np.empty(N * R, np.int32),
        "recv_src_token": np.empty(RM, np.int32),
        "recv_topk_idx": np.empty(RM * k, np.int32),
        "recv_topk_weights": np.empty(RM * k, np.float32),
        "recv_routing_map": np.empty(RM * E_loc, np.uint8),
        "recv_probs": np.empty(RM * E_loc, np.float32),
        "recv_pad_mask": np.empty(RM, np.uint8),
    }
    o = _DedupOut(**{name: _ptr(arr) for name, arr in out.items()})
    if lib.oracle_dedup_layout(ctypes.byref(p), _ptr(phys), _ptr(dest), _ptr(probs), ctypes.byref(o)) != 0:
        raise ValueError("oracle_dedup_layout rejected the problem")
    out["is_token_in_rank"] = out["is_token_in_rank"].reshape(N, R)
    out["token_rank_row"] = out["token_rank_row"].reshape(N, R)
    out["recv_topk_idx"] = out["recv_topk_idx"].reshape(RM, k)
    out["recv_topk_weights"] = out["recv_topk_weights"].reshape(RM, k)
    out["recv_routing_map"] = out["recv_routing_map"].reshape(RM, E_loc)
    out["recv_probs"] = out["recv_probs"].reshape(RM, E_loc)
    out["recv_max"] = RM
    return out


def dedup_combine_local(expert_out: np.ndarray, L: dict, D: dict, topk_probs: Optional[np.ndarray], R: int) -> np.ndarray:
    """Receiver-side partial per (token, rank) row (see moe_oracle.c)."""
    expert_out = _c(expert_out, np.uint16)
    dest = _c(L["dest_row"], np.int32)
    N, k = dest.shape
    H = expert_out.shape[1]
    RM = D["recv_max"]
    probs = None if topk_probs is None else _c(topk_probs, np.float32)
    p = _Problem(N=N, k=k, E_log=R, num_replicas=0, R=R, C=0)
    partial = np.empty((RM, H), np.uint16)
    _lib().oracle_dedup_combine_local(ctypes.byref(p), H, RM, _ptr(dest), _ptr(_c(L["rank_offsets"], np.int32)),
                                      _ptr(_c(D["recv_src_token"], np.int32)),
                                      _ptr(_c(D["recv_rank_offsets"], np.int32)), _ptr(expert_out), _ptr(probs),
                                      _ptr(partial))
    return partial


def permute(hidden: np.ndarray, dest_row: np.ndarray, rows_max: int) -> np.ndarray:
    hidden = _c(hidden, np.uint16)
    dest_row = _c(dest_row, np.int32)
    N, H = hidden.shape
    k = dest_row.shape[1]
    p = _Problem(N=N, k=k, E_log=1, num_replicas=0, R=1, C=0)
    send = np.empty((rows_max, H), np.uint16)
    _lib().oracle_permute(ctypes.byref(p), H, _ptr(dest_row), rows_max, _ptr(hidden), _ptr(send))
    return send


def combine(expert_out: np.ndarray, dest_row: np.ndarray, topk_probs: Optional[np.ndarray]) -> np.ndarray:
    expert_out = _c(expert_out, np.uint16)
    dest_row = _c(dest_row, np.int32)
    N, k = dest_row.shape
    H = expert_out.shape[1]
    probs = None if topk_probs is None else _c(topk_probs, np.float32)
    p = _Problem(N=N, k=k, E_log=1, num_replicas=0, R=1, C=0)
    out = np.empty((N, H), np.uint16)
    _lib().oracle_combine(ctypes.byref(p), H, _ptr(dest_row), _ptr(expert_out), _ptr(probs), _ptr(out))
    return out


def restore_combined(expert_outs, dest_rows, topk_probs: Optional[np.ndarray]) -> np.ndarray:
    """Slot-ordered combine over the TP peers' buffers (one row map and expert output per peer)."""
    expert_outs = [_c(y, np.uint16) for y in expert_outs]
    dest_rows = [_c(d, np.int32) for d in dest_rows]
    T = len(dest_rows)
    N, k = dest_rows[0].shape
    H = expert_outs[0].shape[1]
    probs = None if topk_probs is None else _c(topk_probs, np.float32)
    p = _Problem(N=N, k=k, E_log=1, num_replicas=0, R=1, C=0)
    d_arr = (ctypes.c_void_p * T)(*[d.ctypes.data for d in dest_rows])
    y_arr = (ctypes.c_void_p * T)(*[y.ctypes.data for y in expert_outs])
    out = np.empty((N, H), np.uint16)
    _lib().oracle_restore_combined(ctypes.byref(p), H, T, d_arr, y_arr, _ptr(probs), _ptr(out))
    return out


def ep_exchange(layouts, sends, R: int):
    """The expert-parallel exchange between R ranks ([Megatron MoE] all-to-all token
    dispatcher: each rank's permuted rows go to the rank owning their expert, which
    then sorts what it received by local expert; [Megatron MORI] dispatch into the
    receivers' buffers, combine reading the expert outputs back).

    ``layouts[s]`` / ``sends[s]``: source rank s's layout (``expert_offsets``,
    ``tokens_per_expert``) and send buffer. Rank r receives, for each of its experts
    q in ascending order and within q for each source s in ascending order, the rows
    that s holds for q (its padding rows included, as zeros).

    Returns ``recv`` (per rank: [rows, H]), ``recv_expert_offsets`` (per rank:
    [E_loc + 1], where each local expert's rows start) and ``base`` (per source:
    [E], the receive row on q's owner where source s's rows for q start).
    """
    S = len(layouts)
    E = len(layouts[0]["expert_offsets"]) - 1
    E_loc = E // R
    H = sends[0].shape[1]
    recv, recv_off = [], []
    base = [np.zeros(E, np.int64) for _ in range(S)]
    for r in range(R):
        blocks, offs, pos = [], [], 0
        for q in range(r * E_loc, (r + 1) * E_loc):
            offs.append(pos)
            for s in range(S):
                lo, hi = int(layouts[s]["expert_offsets"][q]), int(layouts[s]["expert_offsets"][q + 1])
                base[s][q] = pos
                blocks.append(sends[s][lo:hi])
                pos += hi - lo
        offs.append(pos)
        recv.append(np.concatenate(blocks, axis=0) if blocks else np.zeros((0, H), np.uint16))
        recv_off.append(np.asarray(offs, np.int64))
    return recv, recv_off, base


def permute_backward(grad_send: np.ndarray, dest_row: np.ndarray) -> np.ndarray:
    grad_send = _c(grad_send, np.uint16)
    dest_row = _c(dest_row, np.int32)
    N, k = dest_row.shape
    H = grad_send.shape[1]
    p = _Problem(N=N, k=k, E_log=1, num_replicas=0, R=1, C=0)
    out = np.empty((N, H), np.uint16)
    _lib().oracle_permute_backward(ctypes.byref(p), H, _ptr(dest_row), _ptr(grad_send), _ptr(out))
    return out


def combine_backward(grad_out: np.ndarray, expert_out: np.ndarray, dest_row: np.ndarray,
                     row_token: np.ndarray, row_prob: np.ndarray):
    """Returns (grad_expert_out [rows_max,H] bf16 bits, grad_probs [N,k] f32)."""
    grad_out = _c(grad_out, np.uint16)
    expert_out = _c(expert_out, np.uint16)
    dest_row = _c(dest_row, np.int32)
    row_token = _c(row_token, np.int32)
    row_prob = _c(row_prob, np.float32)
    N, k = dest_row.shape
    H = grad_out.shape[1]
    RM = row_token.shape[0]
    p = _Problem(N=N, k=k, E_log=1, num_replicas=0, R=1, C=0)
    gy = np.empty((RM, H), np.uint16)
    gp = np.empty((N, k), np.float32)
    _lib().oracle_combine_backward(ctypes.byref(p), H, RM, _ptr(dest_row), _ptr(row_token), _ptr(row_prob),
                                   _ptr(grad_out), _ptr(expert_out), _ptr(gy), _ptr(gp))
    return gy, gp


# ------------------------------------------------------------ all host cores
# The token-independent steps through libmoe_oracle_omp.so: the same oracle functions, each
# thread on a contiguous chunk of tokens (a timing baseline; results equal the serial calls).

_omp_handle: Optional[ctypes.CDLL] = None


def _omp() -> ctypes.CDLL:
    global _omp_handle
    if _omp_handle is None:
        build_omp()
        lib = ctypes.CDLL(_OMP_LIB)
        lib.oracle_omp_threads.restype = ctypes.c_int
        lib.oracle_omp_threads.argtypes = []
        lib.oracle_omp_route_topk.restype = None
        lib.oracle_omp_route_topk.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P]
        lib.oracle_omp_permute.restype = None
        lib.oracle_omp_permute.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, _P, ctypes.c_int64, _P, _P]
        lib.oracle_omp_combine.restype = None
        lib.oracle_omp_combine.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int32, _P, _P, _P, _P]
        _omp_handle = lib
    return _omp_handle


def omp_threads() -> int:
    """Threads the all-cores variant runs with (OMP_NUM_THREADS, else every host core)."""
    return int(_omp().oracle_omp_threads())


def omp_route_topk(logits: np.ndarray, k: int, token_mask: Optional[np.ndarray] = None):
    logits = _c(logits, np.float32)
    N, E = logits.shape
    idx = np.empty((N, k), np.int32)
    probs = np.empty((N, k), np.float32)
    mask = None if token_mask is None else _c(token_mask, np.uint8)
    _omp().oracle_omp_route_topk(_ptr(logits), _ptr(mask), N, E, k, _ptr(idx), _ptr(probs))
    return idx, probs


def omp_permute(hidden: np.ndarray, dest_row: np.ndarray, rows_max: int) -> np.ndarray:
    hidden = _c(hidden, np.uint16)
    dest_row = _c(dest_row, np.int32)
    N, H = hidden.shape
    p = _Problem(N=N, k=dest_row.shape[1], E_log=1, num_replicas=0, R=1, C=0)
    send = np.empty((rows_max, H), np.uint16)
    _omp().oracle_omp_permute(ctypes.byref(p), H, _ptr(dest_row), rows_max, _ptr(hidden), _ptr(send))
    return send


def omp_combine(expert_out: np.ndarray, dest_row: np.ndarray, topk_probs: Optional[np.ndarray]) -> np.ndarray:
    expert_out = _c(expert_out, np.uint16)
    dest_row = _c(dest_row, np.int32)
    N, k = dest_row.shape
    H = expert_out.shape[1]
    probs = None if topk_probs is None else _c(topk_probs, np.float32)
    p = _Problem(N=N, k=k, E_log=1, num_replicas=0, R=1, C=0)
    out = np.empty((N, H), np.uint16)
    _omp().oracle_omp_combine(ctypes.byref(p), H, _ptr(dest_row), _ptr(expert_out), _ptr(probs), _ptr(out))
    return out
