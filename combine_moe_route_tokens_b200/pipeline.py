"""Two batches in flight through route -> layout -> permute -> experts -> combine.

The router and the dispatch layout of a batch are latency-bound (a few µs each, with HBM
mostly idle); the permute and the combine are HBM-bound. ``Pipeline`` runs batch j's
route and layout on a side stream while batch j-1 is combined on the main stream, and
keeps every permute and combine in batch order on the main stream, so the two
bandwidth-bound passes never share HBM with each other and the latency-bound calls are
hidden beside them (Megatron MoE page: router_and_preprocess, dispatch_preprocess, then
token_dispatch / experts / token_combine per batch; the overlap of one micro-batch's
routing with another's combine is this module's scheduling, not the pages').

Two lanes of intermediate buffers (ids, probs, layout, send buffer, output) alternate;
a lane is reused only after its previous batch has been combined. Host-side scheduling
only: every call is the library's own, issued through the binding on the streams below.

    pipe = Pipeline(problem)
    ready = torch.cuda.Event(); ready.record()  # the inputs below are on the device by now
    for logits, hidden in batches:
        out = pipe.submit(logits, hidden, ready=ready)  # the batch's combine output (main stream)
        consume(out)                                    # before the lane comes round again
    pipe.join()
"""

from __future__ import annotations

from typing import Callable, List, Optional

import torch


class _Lane:
    def __init__(self, problem, device, side_priority: int):
        from . import Layout

        N, H, k = problem.N, problem.H, problem.k
        self.layout = Layout.allocate(problem, device)
        self.idx = torch.empty((N, k), dtype=torch.int32, device=device)
        self.probs = torch.empty((N, k), dtype=torch.float32, device=device)
        self.send = torch.empty((problem.rows_max, H), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((N, H), dtype=torch.bfloat16, device=device)
        self.stream = torch.cuda.Stream(device, priority=side_priority)
        self.laid_out = torch.cuda.Event()
        self.combined: Optional[torch.cuda.Event] = None  # this lane's last batch has been combined


class Pipeline:
    """Two batches in flight (see the module docstring).

    ``submit`` enqueues one batch and returns that batch's combine output, a buffer of the
    lane it ran on: it holds the result once the main stream has reached it, and is
    overwritten by the batch after next. ``experts(send, lane)``, if given, runs on the
    main stream between the permute and the combine and returns the expert output
    ``[rows_max, H]`` (default: the send buffer itself, identity experts)."""

    def __init__(self, problem, device=None, stream: Optional[torch.cuda.Stream] = None,
                 experts: Optional[Callable] = None):
        if problem.tp_size > 1:
            raise ValueError("the pipeline takes tp_size 1")
        self.problem = problem
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.main = torch.cuda.current_stream(self.device) if stream is None else stream
        # the side streams' blocks go first when SMs free up (a lower number is a higher priority)
        self.lanes: List[_Lane] = [_Lane(problem, self.device, -1) for _ in range(2)]
        self.experts = experts
        self._next = 0

    def submit(self, logits: torch.Tensor, hidden: torch.Tensor, token_mask: Optional[torch.Tensor] = None,
               ready: Optional[torch.cuda.Event] = None) -> torch.Tensor:
        """Enqueue one batch. ``ready``: an event after which ``logits`` and ``hidden`` hold the
        batch. The default, an event recorded on the main stream now, is always safe but
        orders this batch's routing after the previous batch's combine (no overlap); inputs
        that are already on the device, or produced elsewhere, should come with their own
        event so that the routing can run beside that combine."""
        from . import moe_combine, moe_dispatch_layout, moe_permute, moe_route_topk

        p = self.problem
        lane = self.lanes[self._next]
        self._next ^= 1
        if ready is None:
            ready = torch.cuda.Event()
            ready.record(self.main)
        side = lane.stream
        side.wait_event(ready)
        if lane.combined is not None:  # the lane's buffers are free once its last batch is combined
            side.wait_event(lane.combined)
        moe_route_topk(logits, p.k, token_mask=token_mask, topk_idx=lane.idx, topk_probs=lane.probs, stream=side)
        moe_dispatch_layout(p, lane.idx, lane.probs, layout=lane.layout, stream=side)
        lane.laid_out.record(side)
        self.main.wait_event(ready)  # the permute reads `hidden` (a no-op if `ready` is on this stream)
        self.main.wait_event(lane.laid_out)
        moe_permute(p, lane.layout, hidden, send=lane.send, stream=self.main)
        y = lane.send if self.experts is None else self.experts(lane.send, lane)
        moe_combine(p, lane.layout, y, lane.probs, out=lane.out, stream=self.main)
        done = torch.cuda.Event()
        done.record(self.main)
        lane.combined = done
        return lane.out

    def reset(self) -> None:
        """Forget the earlier batches' events; call it with their work complete (for example
        after a synchronise, before a graph capture: a capture waits only for events
        recorded inside it). The next batch takes lane 0."""
        for lane in self.lanes:
            lane.combined = None
        self._next = 0

    def join(self) -> None:
        """The main stream waits for both side streams (needed before a graph capture ends)."""
        for lane in self.lanes:
            ev = torch.cuda.Event()
            ev.record(lane.stream)
            self.main.wait_event(ev)

    def status(self) -> int:
        st = 0
        for lane in self.lanes:
            st |= lane.layout.status()
        return st

    def clear_status(self) -> None:
        for lane in self.lanes:
            lane.layout.clear_status()
