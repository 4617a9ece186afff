"""MoE token dispatch and combine on one B200 — Python binding of libmoert.so.

Argument marshalling only: every step runs in the CUDA kernels behind the C
ABI of include/moe_rt.h. PyTorch supplies device memory and the stream. The
functions keep the C names:

    moe_route_topk        router softmax + top-k
    moe_dispatch_layout   reroute, histogram, ordinals, capacity, scan, splits, row maps
    moe_dispatch          the layout and the permute in one call (the permute fused into the layout's fill)
    moe_permute           send[dest_row[t, j]] = hidden[t]
    moe_combine           out[t] = bf16(sum_j p[t, j] * y[dest_row[t, j]]), fp32, ascending j
    moe_restore_combined  the same over the buffers of TP peers (after TP folding)
    moe_dedup_*           DeepEP-style view: one receive row per (token, rank), two-level combine
    moe_ep_*              expert-parallel exchange: dispatch into / combine from the ranks' receive buffers
    EpGroup               that exchange between processes (CUDA IPC mappings, offsets all-gather, fences)
    Pipeline              two batches in flight: one's route and layout beside the other's combine
    moe_permute_backward  grad_hidden[t] = bf16(sum_j grad_send[dest_row[t, j]])
    moe_combine_backward  grad_y[row] = bf16(p * grad_out[t]); grad_probs[t, j] = <grad_out[t], y[row]>

All calls are stream-ordered on the current torch stream (or ``stream=``)
and never synchronise with the host.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional

import ctypes

import torch

from . import _native
from ._native import (
    MoeError,
    MOE_DEV_EXPERT_RANGE,
    MOE_DEV_ROW_RANGE,
    MOE_DEV_TIMEOUT,
    MOE_FLAG_NONE,
    MOE_FLAG_TEST_WAIT_TIMEOUT,
    MOE_FLAG_DISPATCH_BULK_COPY,
)

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

__all__ = [
    "Problem",
    "Layout",
    "CountsPrefetch",
    "MoeError",
    "moe_route_topk",
    "moe_dispatch_layout",
    "moe_dispatch_layout_noalloc",
    "moe_dispatch",
    "moe_permute",
    "moe_combine",
    "moe_restore_combined",
    "DedupView",
    "EpPlan",
    "EpGroup",
    "Pipeline",
    "peer_table",
    "moe_ep_recv_rows_max",
    "moe_ep_plan",
    "moe_ep_dispatch",
    "moe_ep_combine",
    "moe_ep_combine_backward",
    "moe_dedup_layout",
    "moe_dedup_dispatch",
    "moe_dedup_combine_local",
    "moe_dedup_combine",
    "moe_permute_backward",
    "moe_combine_backward",
    "load_library",
    "COUNTER_NAMES",
    "MOE_DEV_EXPERT_RANGE",
    "MOE_DEV_ROW_RANGE",
    "MOE_DEV_TIMEOUT",
    "MOE_FLAG_NONE",
    "MOE_FLAG_TEST_WAIT_TIMEOUT",
    "MOE_FLAG_DISPATCH_BULK_COPY",
]


def load_library():
    """Load libmoert.so (raises if it is missing; there is no fallback)."""
    return _native.lib()


@dataclass(frozen=True)
class Problem:
    """The problem statement: hidden [N,H] bf16, top-k ids/probs [N,k], E_log experts on R ranks."""

    N: int
    H: int
    k: int
    E_log: int
    R: int
    capacity: int = 0
    num_replicas: int = 0
    flags: int = MOE_FLAG_NONE
    row_align: int = 0
    tp_size: int = 0
    tp_rank: int = 0

    @property
    def E(self) -> int:
        return self.E_log + self.num_replicas

    @property
    def E_loc(self) -> int:
        return self.E // self.R

    def c_struct(self) -> _native.MoeProblem:
        return _native.MoeProblem(
            N=self.N,
            H=self.H,
            k=self.k,
            E_log=self.E_log,
            num_replicas=self.num_replicas,
            R=self.R,
            capacity=self.capacity,
            flags=self.flags,
            row_align=self.row_align,
            tp_size=self.tp_size,
            tp_rank=self.tp_rank,
        )

    @property
    def rows_max(self) -> int:
        p = self.c_struct()
        v = _native.lib().moe_rows_max(ctypes.byref(p))
        if v < 0:
            _native.check("moe_rows_max", int(v))
        return int(v)

    @property
    def workspace_bytes(self) -> int:
        p = self.c_struct()
        n = ctypes.c_size_t(0)
        _native.check("moe_layout_workspace_bytes",
                      _native.lib().moe_layout_workspace_bytes(ctypes.byref(p), ctypes.byref(n)))
        return int(n.value)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


@dataclass
class CountsPrefetch:
    """Counts on their way to pinned host memory (Layout.prefetch_counts)."""

    host: Dict[str, torch.Tensor]
    event: "torch.cuda.Event"

    def ready(self) -> bool:
        return self.event.query()

    def get(self) -> Dict[str, torch.Tensor]:
        """The host tensors, waiting for the copies if they have not landed yet."""
        self.event.synchronize()
        return self.host


@dataclass
class Layout:
    """Device buffers of every dispatch-layout output plus the layout workspace."""

    problem: Problem
    tensors: Dict[str, torch.Tensor] = field(default_factory=dict)
    workspace: Optional[torch.Tensor] = None
    _pinned: Optional[Dict[str, torch.Tensor]] = field(default=None, repr=False)
    _pinned_done: Optional["torch.cuda.Event"] = field(default=None, repr=False)

    @classmethod
    def allocate(cls, problem: Problem, device=None, local_topk: bool = True) -> "Layout":
        device = torch.device("cuda") if device is None else torch.device(device)
        N, k, E, R, E_log = problem.N, problem.k, problem.E, problem.R, problem.E_log
        NK = N * k
        RM = problem.rows_max
        i32, f32, u8 = torch.int32, torch.float32, torch.uint8
        t = {
            "phys_idx": torch.empty((N, k), dtype=i32, device=device),
            "ordinal": torch.empty((N, k), dtype=i32, device=device),
            "dest_row": torch.empty((N, k), dtype=i32, device=device),
            "drop_mask": torch.empty((N, k), dtype=u8, device=device),
            "counts_logical": torch.empty(E_log, dtype=i32, device=device),
            "placement": torch.empty(E_log, dtype=i32, device=device),
            "counts_raw": torch.empty(E, dtype=i32, device=device),
            "tokens_per_expert": torch.empty(E, dtype=i32, device=device),
            "expert_offsets": torch.empty(E + 1, dtype=i32, device=device),
            "input_splits": torch.empty(R, dtype=i32, device=device),
            "output_splits": torch.empty(R, dtype=i32, device=device),
            "rank_offsets": torch.empty(R + 1, dtype=i32, device=device),
            "counters": torch.empty(8, dtype=i32, device=device),
            "num_rows": torch.empty(1, dtype=i32, device=device),
            "status": torch.zeros(1, dtype=torch.int32, device=device),
            "row_token": torch.empty(RM, dtype=i32, device=device),
            "row_slot": torch.empty(RM, dtype=i32, device=device),
            "row_local_expert": torch.empty(RM, dtype=i32, device=device),
            "row_prob": torch.empty(RM, dtype=f32, device=device),
            "pad_mask": torch.empty(RM, dtype=u8, device=device),
        }
        if local_topk:
            t["local_topk"] = torch.empty((R, N, k), dtype=i32, device=device)
        ws = torch.zeros(problem.workspace_bytes, dtype=u8, device=device)
        assert NK >= 0
        return cls(problem=problem, tensors=t, workspace=ws)

    def __getitem__(self, name: str) -> torch.Tensor:
        return self.tensors[name]

    def c_struct(self) -> _native.MoeLayout:
        return _native.MoeLayout(**{name: (self.tensors[name].data_ptr() if name in self.tensors else None)
                                    for name in _native.LAYOUT_FIELDS})

    @property
    def device(self) -> torch.device:
        return self.tensors["dest_row"].device

    def status(self) -> int:
        """Device status bits (MOE_DEV_*) OR-ed by every call on this layout. Synchronises."""
        return int(self.tensors["status"].item()) & 0xFFFFFFFF

    def clear_status(self) -> None:
        self.tensors["status"].zero_()

    def prefetch_counts(self, stream=None) -> "CountsPrefetch":
        """Copy the per-expert and per-rank counts to pinned host memory without waiting.

        The copies are enqueued after the work already on ``stream`` (the layout call),
        so the host can read them later, off the critical path, instead of forcing a
        synchronisation when it needs them (Megatron MORI: deferred count reads). The
        pinned buffers are allocated on the first call and reused by every later one,
        so later calls allocate nothing (a pinned allocation can synchronise the
        device). Each call overwrites what the previous one copied."""
        st = torch.cuda.current_stream(self.device) if stream is None else stream
        keys = ("tokens_per_expert", "expert_offsets", "input_splits", "output_splits", "num_rows", "counters")
        if self._pinned is None:
            self._pinned = {key: torch.empty(self.tensors[key].shape, dtype=self.tensors[key].dtype,
                                             pin_memory=True) for key in keys}
            self._pinned_done = torch.cuda.Event()
        with torch.cuda.stream(st):
            for key in keys:
                self._pinned[key].copy_(self.tensors[key], non_blocking=True)
            self._pinned_done.record(st)
        return CountsPrefetch(host=self._pinned, event=self._pinned_done)

    def counters(self) -> Dict[str, int]:
        """dispatch_counters as a dict. Synchronises."""
        return dict(zip(COUNTER_NAMES, (int(v) for v in self.tensors["counters"].tolist())))


@dataclass
class DedupView:
    """Device buffers of the DeepEP-style token-dedup view plus its workspace."""

    problem: Problem
    tensors: Dict[str, torch.Tensor] = field(default_factory=dict)
    workspace: Optional[torch.Tensor] = None

    @property
    def recv_max(self) -> int:
        p = self.problem.c_struct()
        v = _native.lib().moe_dedup_rows_max(ctypes.byref(p))
        if v < 0:
            _native.check("moe_dedup_rows_max", int(v))
        return int(v)

    @classmethod
    def allocate(cls, problem: Problem, device=None) -> "DedupView":
        device = torch.device("cuda") if device is None else torch.device(device)
        view = cls(problem=problem)
        N, k, R = problem.N, problem.k, problem.R
        E_loc = problem.E_loc
        RM = view.recv_max
        i32, f32, u8 = torch.int32, torch.float32, torch.uint8
        view.tensors = {
            "num_tokens_per_rank": torch.empty(R, dtype=i32, device=device),
            "recv_rank_offsets": torch.empty(R + 1, dtype=i32, device=device),
            "num_recv": torch.empty(1, dtype=i32, device=device),
            "is_token_in_rank": torch.empty((N, R), dtype=u8, device=device),
            "token_rank_row": torch.empty((N, R), dtype=i32, device=device),
            "recv_src_token": torch.empty(RM, dtype=i32, device=device),
            "recv_topk_idx": torch.empty((RM, k), dtype=i32, device=device),
            "recv_topk_weights": torch.empty((RM, k), dtype=f32, device=device),
            "recv_routing_map": torch.empty((RM, E_loc), dtype=u8, device=device),
            "recv_probs": torch.empty((RM, E_loc), dtype=f32, device=device),
            "recv_pad_mask": torch.empty(RM, dtype=u8, device=device),
            "status": torch.zeros(1, dtype=i32, device=device),
        }
        n = ctypes.c_size_t(0)
        pc = problem.c_struct()
        _native.check("moe_dedup_workspace_bytes",
                      _native.lib().moe_dedup_workspace_bytes(ctypes.byref(pc), ctypes.byref(n)))
        view.workspace = torch.zeros(int(n.value), dtype=u8, device=device)
        return view

    def __getitem__(self, name: str) -> torch.Tensor:
        return self.tensors[name]

    def c_struct(self) -> _native.MoeDedup:
        return _native.MoeDedup(**{name: self.tensors[name].data_ptr() for name in _native.DEDUP_FIELDS})

    def status(self) -> int:
        return int(self.tensors["status"].item()) & 0xFFFFFFFF


def moe_dedup_layout(problem: Problem, layout: Layout, topk_probs: Optional[torch.Tensor],
                     dedup: Optional[DedupView] = None, stream=None) -> DedupView:
    """DeepEP-style view (one receive row per (token, rank)) of a dispatch layout."""
    if dedup is None:
        dedup = DedupView.allocate(problem, layout.device)
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    D = dedup.c_struct()
    _native.check("moe_dedup_layout",
                  _native.lib().moe_dedup_layout(ctypes.byref(p), ctypes.byref(L), _ptr(topk_probs), ctypes.byref(D),
                                                 _ptr(dedup.workspace), dedup.workspace.numel(), _stream(stream)))
    return dedup


def moe_dedup_dispatch(problem: Problem, dedup: DedupView, hidden: torch.Tensor,
                       recv_x: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """recv_x[token_rank_row[t, r]] = hidden[t]; tail rows zero."""
    _need(hidden, "hidden", torch.bfloat16, (problem.N, problem.H))
    if recv_x is None:
        recv_x = torch.empty((dedup.recv_max, problem.H), dtype=torch.bfloat16, device=hidden.device)
    _need(recv_x, "recv_x", torch.bfloat16, (dedup.recv_max, problem.H), hidden.device)
    p = problem.c_struct()
    D = dedup.c_struct()
    _native.check("moe_dedup_dispatch",
                  _native.lib().moe_dedup_dispatch(ctypes.byref(p), ctypes.byref(D), _ptr(hidden), _ptr(recv_x),
                                                   _stream(stream)))
    return recv_x


def moe_dedup_combine_local(problem: Problem, layout: Layout, dedup: DedupView, expert_out: torch.Tensor,
                            topk_probs: Optional[torch.Tensor], partial: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """Receiver-side partial per receive row (fp32 chain over the row's local slots, one bf16 rounding)."""
    _need(expert_out, "expert_out", torch.bfloat16, (problem.rows_max, problem.H), layout.device)
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), layout.device)
    if partial is None:
        partial = torch.empty((dedup.recv_max, problem.H), dtype=torch.bfloat16, device=layout.device)
    _need(partial, "partial", torch.bfloat16, (dedup.recv_max, problem.H), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    D = dedup.c_struct()
    _native.check("moe_dedup_combine_local",
                  _native.lib().moe_dedup_combine_local(ctypes.byref(p), ctypes.byref(L), ctypes.byref(D),
                                                        _ptr(expert_out), _ptr(topk_probs), _ptr(partial),
                                                        _stream(stream)))
    return partial


def moe_dedup_combine(problem: Problem, dedup: DedupView, partial: torch.Tensor, out: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """out[t] = bf16(fp32 sum over ascending r of partial[token_rank_row[t, r]])."""
    _need(partial, "partial", torch.bfloat16, (dedup.recv_max, problem.H))
    if out is None:
        out = torch.empty((problem.N, problem.H), dtype=torch.bfloat16, device=partial.device)
    _need(out, "out", torch.bfloat16, (problem.N, problem.H), partial.device)
    p = problem.c_struct()
    D = dedup.c_struct()
    _native.check("moe_dedup_combine",
                  _native.lib().moe_dedup_combine(ctypes.byref(p), ctypes.byref(D), _ptr(partial), _ptr(out),
                                                  _stream(stream)))
    return out


def moe_route_topk(logits: torch.Tensor, k: int, token_mask: Optional[torch.Tensor] = None,
                   topk_idx: Optional[torch.Tensor] = None, topk_probs: Optional[torch.Tensor] = None,
                   stream=None):
    """Softmax over E + top-k. Returns (topk_idx [N,k] int32, topk_probs [N,k] fp32)."""
    _need(logits, "logits", torch.float32)
    if logits.dim() != 2:
        raise ValueError("logits must be [N, E]")
    N, E = logits.shape
    if token_mask is not None:
        _need(token_mask, "token_mask", torch.uint8, (N,), logits.device)
    if topk_idx is None:
        topk_idx = torch.empty((N, k), dtype=torch.int32, device=logits.device)
    if topk_probs is None:
        topk_probs = torch.empty((N, k), dtype=torch.float32, device=logits.device)
    _need(topk_idx, "topk_idx", torch.int32, (N, k), logits.device)
    _need(topk_probs, "topk_probs", torch.float32, (N, k), logits.device)
    rc = _native.lib().moe_route_topk(_ptr(logits), _ptr(token_mask), N, E, k, _ptr(topk_idx), _ptr(topk_probs),
                                      _stream(stream))
    _native.check("moe_route_topk", rc)
    return topk_idx, topk_probs


def moe_dispatch_layout(problem: Problem, topk_idx: torch.Tensor, topk_probs: Optional[torch.Tensor],
                        layout: Optional[Layout] = None, stream=None) -> Layout:
    """Every dispatch-layout output (a count pass and a fill pass); returns the (reusable) Layout."""
    _need(topk_idx, "topk_idx", torch.int32, (problem.N, problem.k))
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), topk_idx.device)
    if layout is None:
        layout = Layout.allocate(problem, topk_idx.device)
    elif layout.problem != problem:
        raise ValueError("layout was allocated for a different problem")
    p = problem.c_struct()
    L = layout.c_struct()
    rc = _native.lib().moe_dispatch_layout(ctypes.byref(p), _ptr(topk_idx), _ptr(topk_probs), ctypes.byref(L),
                                           _ptr(layout.workspace), layout.workspace.numel(), _stream(stream))
    _native.check("moe_dispatch_layout", rc)
    return layout


def moe_dispatch(problem: Problem, topk_idx: torch.Tensor, topk_probs: Optional[torch.Tensor], hidden: torch.Tensor,
                 layout: Optional[Layout] = None, send: Optional[torch.Tensor] = None, stream=None):
    """Dispatch layout and permute in one call; returns (layout, send).

    Equals moe_dispatch_layout followed by moe_permute, bit for bit."""
    _need(topk_idx, "topk_idx", torch.int32, (problem.N, problem.k))
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), topk_idx.device)
    _need(hidden, "hidden", torch.bfloat16, (problem.N, problem.H), topk_idx.device)
    if layout is None:
        layout = Layout.allocate(problem, topk_idx.device)
    elif layout.problem != problem:
        raise ValueError("layout was allocated for a different problem")
    if send is None:
        send = torch.empty((problem.rows_max, problem.H), dtype=torch.bfloat16, device=topk_idx.device)
    _need(send, "send", torch.bfloat16, (problem.rows_max, problem.H), topk_idx.device)
    p = problem.c_struct()
    L = layout.c_struct()
    rc = _native.lib().moe_dispatch(ctypes.byref(p), _ptr(topk_idx), _ptr(topk_probs), ctypes.byref(L),
                                    _ptr(layout.workspace), layout.workspace.numel(), _ptr(hidden), _ptr(send),
                                    _stream(stream))
    _native.check("moe_dispatch", rc)
    return layout, send


def moe_dispatch_layout_noalloc(problem: Problem, topk_idx: torch.Tensor, topk_probs: Optional[torch.Tensor],
                                layout: Layout, stream=None) -> Layout:
    """moe_dispatch_layout for callers that cannot allocate device scratch.

    The library keeps the scratch in a fixed device array (E_log up to
    MOE_NOALLOC_MAX_E_LOG); ``layout.workspace`` is not used. Calls share that
    array, so calls running at the same time on different streams race; keep
    them on one stream. The first call on a device must not happen during
    stream capture.
    """
    _need(topk_idx, "topk_idx", torch.int32, (problem.N, problem.k))
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), topk_idx.device)
    if layout.problem != problem:
        raise ValueError("layout was allocated for a different problem")
    p = problem.c_struct()
    L = layout.c_struct()
    rc = _native.lib().moe_dispatch_layout_noalloc(ctypes.byref(p), _ptr(topk_idx), _ptr(topk_probs),
                                                   ctypes.byref(L), _stream(stream))
    _native.check("moe_dispatch_layout_noalloc", rc)
    return layout


def moe_permute(problem: Problem, layout: Layout, hidden: torch.Tensor, send: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """send[dest_row[t,j]] = hidden[t]; pad rows zero. Returns send [rows_max, H] bf16."""
    _need(hidden, "hidden", torch.bfloat16, (problem.N, problem.H), layout.device)
    if send is None:
        send = torch.empty((problem.rows_max, problem.H), dtype=torch.bfloat16, device=hidden.device)
    _need(send, "send", torch.bfloat16, (problem.rows_max, problem.H), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    _native.check("moe_permute",
                  _native.lib().moe_permute(ctypes.byref(p), ctypes.byref(L), _ptr(hidden), _ptr(send),
                                            _stream(stream)))
    return send


def moe_combine(problem: Problem, layout: Layout, expert_out: torch.Tensor, topk_probs: Optional[torch.Tensor],
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[t] = bf16(fp32 fma chain over ascending kept j of p[t,j] * expert_out[dest_row[t,j]])."""
    _need(expert_out, "expert_out", torch.bfloat16, (problem.rows_max, problem.H), layout.device)
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), layout.device)
    if out is None:
        out = torch.empty((problem.N, problem.H), dtype=torch.bfloat16, device=expert_out.device)
    _need(out, "out", torch.bfloat16, (problem.N, problem.H), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    _native.check("moe_combine",
                  _native.lib().moe_combine(ctypes.byref(p), ctypes.byref(L), _ptr(expert_out), _ptr(topk_probs),
                                            _ptr(out), _stream(stream)))
    return out


def moe_restore_combined(problem: Problem, layouts, expert_outs, topk_probs: Optional[torch.Tensor],
                         out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Slot-ordered combine over the TP peers' buffers (layouts[q], expert_outs[q] of peer q)."""
    T = max(problem.tp_size, 1)
    if len(layouts) != T or len(expert_outs) != T:
        raise ValueError(f"need {T} peer layouts and expert outputs")
    for q in range(T):
        _need(expert_outs[q], f"expert_outs[{q}]", torch.bfloat16, (problem.rows_max, problem.H), layouts[0].device)
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), layouts[0].device)
    if out is None:
        out = torch.empty((problem.N, problem.H), dtype=torch.bfloat16, device=layouts[0].device)
    _need(out, "out", torch.bfloat16, (problem.N, problem.H), layouts[0].device)
    p = problem.c_struct()
    Ls = (_native.MoeLayout * T)(*[L.c_struct() for L in layouts])
    ys = (ctypes.c_void_p * T)(*[y.data_ptr() for y in expert_outs])
    _native.check("moe_restore_combined",
                  _native.lib().moe_restore_combined(ctypes.byref(p), Ls, ys, _ptr(topk_probs), _ptr(out),
                                                     _stream(stream)))
    return out


# ------------------------------------------------- expert-parallel exchange


def moe_ep_recv_rows_max(problem: Problem) -> int:
    """Rows of one rank's receive buffer for the exchange (an upper bound, fixed per problem)."""
    p = problem.c_struct()
    v = int(_native.lib().moe_ep_recv_rows_max(ctypes.byref(p)))
    if v < 0:
        _native.check("moe_ep_recv_rows_max", v)
    return v


@dataclass
class EpPlan:
    """moe_ep_plan outputs for one source rank (device tensors)."""

    base: torch.Tensor                 # [E] int32
    recv_expert_offsets: torch.Tensor  # [E_loc + 1] int32
    num_recv: torch.Tensor             # [1] int32
    status: torch.Tensor               # [1] int32 (MOE_DEV_* bits)

    @classmethod
    def allocate(cls, problem: Problem, device=None) -> "EpPlan":
        device = torch.device("cuda") if device is None else torch.device(device)
        i32 = torch.int32
        return cls(base=torch.empty(problem.E, dtype=i32, device=device),
                   recv_expert_offsets=torch.empty(problem.E_loc + 1, dtype=i32, device=device),
                   num_recv=torch.empty(1, dtype=i32, device=device),
                   status=torch.zeros(1, dtype=i32, device=device))


def peer_table(buffers, device=None) -> torch.Tensor:
    """A device array of the buffers' device addresses (rank order), for the exchange calls."""
    device = buffers[0].device if device is None else torch.device(device)
    return torch.tensor([b.data_ptr() for b in buffers], dtype=torch.int64, device=device)


def moe_ep_plan(problem: Problem, offsets_all: torch.Tensor, src_rank: int, plan: Optional[EpPlan] = None,
                stream=None) -> EpPlan:
    """Where this rank's rows go on the owners, and this rank's receive layout.

    ``offsets_all``: [R, E+1] int32, every rank's layout ``expert_offsets`` (gathered by the caller).
    """
    _need(offsets_all, "offsets_all", torch.int32, (problem.R, problem.E + 1))
    if plan is None:
        plan = EpPlan.allocate(problem, offsets_all.device)
    p = problem.c_struct()
    _native.check("moe_ep_plan", _native.lib().moe_ep_plan(
        ctypes.byref(p), _ptr(offsets_all), int(src_rank), _ptr(plan.base), _ptr(plan.recv_expert_offsets),
        _ptr(plan.num_recv), _ptr(plan.status), _stream(stream)))
    return plan


def _table(peers, device, problem: Optional[Problem] = None) -> torch.Tensor:
    """A peer table as given (int64 device addresses), or built from R buffers after checking
    that each is a [moe_ep_recv_rows_max, H] bf16 tensor."""
    if isinstance(peers, torch.Tensor) and peers.dtype == torch.int64:
        return peers
    peers = list(peers)
    if problem is not None:
        rows = moe_ep_recv_rows_max(problem)
        for r, b in enumerate(peers):
            _need(b, f"buffer of rank {r}", torch.bfloat16, (rows, problem.H))
    return peer_table(peers, device)


def moe_ep_dispatch(problem: Problem, layout: Layout, plan: EpPlan, hidden: torch.Tensor, peer_recv,
                    stream=None) -> None:
    """Write this rank's kept rows into the owners' receive buffers (and its padding rows as zeros).

    ``peer_recv``: the R receive buffers ([moe_ep_recv_rows_max, H] bf16 each), or
    their ``peer_table``.
    """
    _need(hidden, "hidden", torch.bfloat16, (problem.N, problem.H), layout.device)
    table = _table(peer_recv, layout.device, problem)
    if table.numel() != problem.R:
        raise ValueError("peer_recv needs one buffer per rank")
    p = problem.c_struct()
    L = layout.c_struct()
    _native.check("moe_ep_dispatch", _native.lib().moe_ep_dispatch(
        ctypes.byref(p), ctypes.byref(L), _ptr(plan.base), _ptr(hidden), _ptr(table), _stream(stream)))


def moe_ep_combine(problem: Problem, layout: Layout, plan: EpPlan, peer_expert_out, topk_probs: Optional[torch.Tensor],
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[t] = bf16(fp32 sum over ascending kept j of p[t,j] * (row of slot j on its expert's owner))."""
    table = _table(peer_expert_out, layout.device, problem)
    if table.numel() != problem.R:
        raise ValueError("peer_expert_out needs one buffer per rank")
    if topk_probs is not None:
        _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), layout.device)
    if out is None:
        out = torch.empty((problem.N, problem.H), dtype=torch.bfloat16, device=layout.device)
    _need(out, "out", torch.bfloat16, (problem.N, problem.H), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    _native.check("moe_ep_combine", _native.lib().moe_ep_combine(
        ctypes.byref(p), ctypes.byref(L), _ptr(plan.base), _ptr(table), _ptr(topk_probs), _ptr(out),
        _stream(stream)))
    return out


def moe_ep_combine_backward(problem: Problem, layout: Layout, plan: EpPlan, grad_out: torch.Tensor,
                            peer_expert_out, topk_probs: torch.Tensor, peer_grad_expert_out,
                            grad_probs: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grad_y rows written into the owners' gradient buffers; returns grad_probs [N, k] fp32.

    The backward of moe_ep_dispatch is moe_ep_combine(..., topk_probs=None) over the
    gradient buffers.
    """
    _need(grad_out, "grad_out", torch.bfloat16, (problem.N, problem.H), layout.device)
    _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), layout.device)
    ty = _table(peer_expert_out, layout.device, problem)
    tg = _table(peer_grad_expert_out, layout.device, problem)
    if ty.numel() != problem.R or tg.numel() != problem.R:
        raise ValueError("one expert-output and one gradient buffer per rank")
    if grad_probs is None:
        grad_probs = torch.empty((problem.N, problem.k), dtype=torch.float32, device=layout.device)
    _need(grad_probs, "grad_probs", torch.float32, (problem.N, problem.k), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    _native.check("moe_ep_combine_backward", _native.lib().moe_ep_combine_backward(
        ctypes.byref(p), ctypes.byref(L), _ptr(plan.base), _ptr(grad_out), _ptr(ty), _ptr(topk_probs), _ptr(tg),
        _ptr(grad_probs), _stream(stream)))
    return grad_probs


def moe_permute_backward(problem: Problem, layout: Layout, grad_send: torch.Tensor,
                         grad_hidden: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grad_hidden[t] = bf16(fp32 sum over ascending kept j of grad_send[dest_row[t,j]])."""
    _need(grad_send, "grad_send", torch.bfloat16, (problem.rows_max, problem.H), layout.device)
    if grad_hidden is None:
        grad_hidden = torch.empty((problem.N, problem.H), dtype=torch.bfloat16, device=grad_send.device)
    _need(grad_hidden, "grad_hidden", torch.bfloat16, (problem.N, problem.H), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    _native.check("moe_permute_backward",
                  _native.lib().moe_permute_backward(ctypes.byref(p), ctypes.byref(L), _ptr(grad_send),
                                                     _ptr(grad_hidden), _stream(stream)))
    return grad_hidden


def moe_combine_backward(problem: Problem, layout: Layout, grad_out: torch.Tensor, expert_out: torch.Tensor,
                         topk_probs: torch.Tensor, grad_expert_out: Optional[torch.Tensor] = None,
                         grad_probs: Optional[torch.Tensor] = None, stream=None):
    """Returns (grad_expert_out [rows_max,H] bf16, grad_probs [N,k] fp32)."""
    _need(grad_out, "grad_out", torch.bfloat16, (problem.N, problem.H), layout.device)
    _need(expert_out, "expert_out", torch.bfloat16, (problem.rows_max, problem.H), layout.device)
    _need(topk_probs, "topk_probs", torch.float32, (problem.N, problem.k), layout.device)
    if grad_expert_out is None:
        grad_expert_out = torch.empty((problem.rows_max, problem.H), dtype=torch.bfloat16, device=grad_out.device)
    if grad_probs is None:
        grad_probs = torch.empty((problem.N, problem.k), dtype=torch.float32, device=grad_out.device)
    _need(grad_expert_out, "grad_expert_out", torch.bfloat16, (problem.rows_max, problem.H), layout.device)
    _need(grad_probs, "grad_probs", torch.float32, (problem.N, problem.k), layout.device)
    p = problem.c_struct()
    L = layout.c_struct()
    _native.check("moe_combine_backward",
                  _native.lib().moe_combine_backward(ctypes.byref(p), ctypes.byref(L), _ptr(grad_out),
                                                     _ptr(expert_out), _ptr(topk_probs), _ptr(grad_expert_out),
                                                     _ptr(grad_probs), _stream(stream)))
    return grad_expert_out, grad_probs


from .ep_group import EpGroup  # noqa: E402  (the exchange between processes; host plumbing only)
from .pipeline import Pipeline  # noqa: E402  (two batches in flight; host scheduling only)
