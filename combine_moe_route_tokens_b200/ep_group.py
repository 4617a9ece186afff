"""The expert-parallel exchange between processes, one rank per process.

Megatron MoE page, the all-to-all token dispatcher: every rank's permuted rows go
to the rank that owns their expert and come back after the experts; Megatron MORI
page: the dispatch writes straight into the receivers' buffers (the permute fused
in) and the combine reads the expert outputs back. The kernels are the C ABI's
``moe_ep_*`` calls, which take device arrays of peer pointers; this module only
wires the processes together:

* every rank allocates its receive buffer, its gradient buffer and its ``[R, E+1]``
  table of every rank's expert offsets, exports them with CUDA IPC
  (``moe_ipc_export``) and all-gathers the handles over the process group;
* every rank maps the others' buffers (``moe_ipc_open``) and builds the device
  tables of R pointers the kernels take (its own buffers at its own index);
* ``fence()`` orders the steps across processes: each rank records an
  interprocess CUDA event on its stream, a host barrier follows, then each
  stream waits for every peer's event. Nothing on the device waits for another
  process.

One step (forward, then backward) per rank, given its own layout:
``publish_offsets`` (the all-gather of expert offsets, written into every rank's
table over peer memory) -> ``fence`` -> ``plan`` -> ``dispatch`` (rows into the
owners' receive buffers) -> ``fence`` -> experts on ``recv`` -> ``fence`` ->
``combine``; backward: ``combine_backward`` (gradient rows into the owners'
gradient buffers) -> ``fence`` -> ``dispatch_backward``. A ``fence`` before the
next step's dispatch keeps a rank from overwriting rows that a peer is still
reading.

With every rank on its own GPU the mappings are peer memory over NVLink; with
several ranks on one GPU they are the same GPU's memory seen from another
process. Plain peer loads and stores only (no TMA, no multicast).
"""

from __future__ import annotations

import ctypes
from typing import Callable, Dict, List, Optional, Sequence

import numpy as np
import torch

from . import _native

BUFFERS = ("recv", "grad", "offsets_all")


def export_buffer(t: torch.Tensor) -> bytes:
    """The CUDA IPC description of a device tensor's memory (plain bytes, to send to peers)."""
    buf = _native.MoeIpcBuffer()
    _native.check("moe_ipc_export",
                  _native.lib().moe_ipc_export(ctypes.c_void_p(t.data_ptr()), t.numel() * t.element_size(),
                                               ctypes.byref(buf)))
    return bytes(ctypes.string_at(ctypes.addressof(buf), ctypes.sizeof(buf)))


def open_buffer(blob: bytes):
    """Map a peer's exported buffer into this process: (device address, mapping)."""
    buf = _native.MoeIpcBuffer.from_buffer_copy(blob)
    ptr, mapping = ctypes.c_void_p(), ctypes.c_void_p()
    _native.check("moe_ipc_open", _native.lib().moe_ipc_open(ctypes.byref(buf), ctypes.byref(ptr),
                                                            ctypes.byref(mapping)))
    return int(ptr.value), int(mapping.value)


def close_buffer(mapping: int) -> None:
    _native.check("moe_ipc_close", _native.lib().moe_ipc_close(ctypes.c_void_p(mapping)))


def exchange(group, obj) -> List:
    """Every rank's ``obj`` in rank order (all_gather_object over the process group)."""
    import torch.distributed as dist

    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, obj, group=group)
    return out


def peer_pointers(rank: int, own: Dict[str, int], blobs: Sequence[Dict[str, bytes]],
                  open_fn: Callable[[bytes], tuple]):
    """Per buffer kind, the R device addresses in rank order (this rank's own at its index),
    and the mappings opened (to close later). ``blobs[r]`` holds rank r's exported buffers."""
    tables = {name: [] for name in own}
    mappings = []
    for r, theirs in enumerate(blobs):
        for name in own:
            if r == rank:
                tables[name].append(own[name])
            else:
                ptr, mapping = open_fn(theirs[name])
                tables[name].append(ptr)
                mappings.append(mapping)
    return tables, mappings


def gather_offsets_host(group, offsets: np.ndarray) -> np.ndarray:
    """The [R, E+1] table of every rank's expert offsets gathered on the host (rank order).

    The device path (``EpGroup.publish_offsets``) writes the table over peer memory
    without a host round trip; this host form serves callers whose ranks cannot map
    each other's memory (it needs the offsets on the host, so it waits for the layout)."""
    import torch.distributed as dist

    mine = torch.from_numpy(np.ascontiguousarray(offsets, dtype=np.int32))
    out = [torch.empty_like(mine) for _ in range(dist.get_world_size(group))]
    dist.all_gather(out, mine, group=group)
    return np.stack([t.numpy() for t in out])


class EpGroup:
    """This process's rank of the exchange: its buffers, the peers' mapped buffers, the fences."""

    def __init__(self, problem, rank: int, group=None, device=None):
        from . import EpPlan, moe_ep_recv_rows_max  # the binding's calls (argument marshalling only)

        if problem.tp_size > 1:
            raise ValueError("the exchange takes tp_size 1")
        self.problem = problem
        self.rank = rank
        self.group = group
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        R, E, H = problem.R, problem.E, problem.H
        rows = moe_ep_recv_rows_max(problem)
        self.recv = torch.zeros((rows, H), dtype=torch.bfloat16, device=self.device)
        self.grad = torch.zeros((rows, H), dtype=torch.bfloat16, device=self.device)
        self.offsets_all = torch.zeros((R, E + 1), dtype=torch.int32, device=self.device)
        self.plan = EpPlan.allocate(problem, self.device)
        self.event = torch.cuda.Event(interprocess=True)
        torch.cuda.synchronize(self.device)  # the buffers exist before peers map them
        mine = {name: export_buffer(getattr(self, name)) for name in BUFFERS}
        blobs = exchange(group, {"buffers": mine, "event": self.event.ipc_handle()})
        if len(blobs) != R:
            raise ValueError(f"the process group has {len(blobs)} ranks, the problem {R}")
        own = {name: getattr(self, name).data_ptr() for name in BUFFERS}
        tables, self._mappings = peer_pointers(rank, own, [b["buffers"] for b in blobs], open_buffer)
        self.tables = {name: torch.tensor(ptrs, dtype=torch.int64, device=self.device)
                       for name, ptrs in tables.items()}
        self.peer_events = [None if r == rank else torch.cuda.Event.from_ipc_handle(self.device, b["event"])
                            for r, b in enumerate(blobs)]

    # ------------------------------------------------------------ ordering
    def fence(self, stream=None) -> None:
        """Every rank's work enqueued so far on its stream completes before anything this
        rank enqueues next on ``stream``: record, host barrier, wait for every peer."""
        import torch.distributed as dist

        stream = torch.cuda.current_stream(self.device) if stream is None else stream
        self.event.record(stream)
        dist.barrier(group=self.group)
        for ev in self.peer_events:
            if ev is not None:
                stream.wait_event(ev)

    # --------------------------------------------------------------- steps
    def publish_offsets(self, layout, stream=None) -> None:
        """This rank's expert offsets into row ``rank`` of every rank's table (peer stores)."""
        from . import _stream

        p = self.problem.c_struct()
        _native.check("moe_ep_publish_offsets", _native.lib().moe_ep_publish_offsets(
            ctypes.byref(p), ctypes.c_void_p(layout["expert_offsets"].data_ptr()), int(self.rank),
            ctypes.c_void_p(self.tables["offsets_all"].data_ptr()), _stream(stream)))

    def plan_exchange(self, stream=None):
        from . import moe_ep_plan

        return moe_ep_plan(self.problem, self.offsets_all, self.rank, plan=self.plan, stream=stream)

    def dispatch(self, layout, hidden: torch.Tensor, stream=None) -> None:
        from . import moe_ep_dispatch

        moe_ep_dispatch(self.problem, layout, self.plan, hidden, self.tables["recv"], stream=stream)

    def combine(self, layout, topk_probs: Optional[torch.Tensor], expert_table: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """The combine over the owners' expert outputs (by default the receive buffers:
        identity experts, or experts that write their output in place)."""
        from . import moe_ep_combine

        table = self.tables["recv"] if expert_table is None else expert_table
        return moe_ep_combine(self.problem, layout, self.plan, table, topk_probs, out=out, stream=stream)

    def combine_backward(self, layout, grad_out: torch.Tensor, topk_probs: torch.Tensor,
                         expert_table: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Gradient rows into the owners' gradient buffers; returns grad_probs."""
        from . import moe_ep_combine_backward

        table = self.tables["recv"] if expert_table is None else expert_table
        return moe_ep_combine_backward(self.problem, layout, self.plan, grad_out, table, topk_probs,
                                       self.tables["grad"], stream=stream)

    def dispatch_backward(self, layout, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """The backward of dispatch: the unit-weight combine over the owners' gradient buffers."""
        from . import moe_ep_combine

        return moe_ep_combine(self.problem, layout, self.plan, self.tables["grad"], None, out=out, stream=stream)

    def close(self) -> None:
        """Unmap the peers' buffers (after a barrier, so that no rank still uses them)."""
        import torch.distributed as dist

        torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)
        for m in self._mappings:
            close_buffer(m)
        self._mappings = []
        dist.barrier(group=self.group)
