#!/usr/bin/env python3
"""Benchmark: MoE dispatch + combine on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ht] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
router top-k -> dispatch (the layout and the permute) -> (identity experts) ->
combine, plus combine-backward and permute-backward for workloads that train
(``ultraep``). Inputs are resident in HBM when the timed region starts and
rotate over several buffer sets whose total size exceeds the 126 MB L2, so no
step reads inputs that a previous step left in L2.

Headline schedule (``--schedule pipelined``, the default where the step is route,
layout, permute and combine on one rank): two batches in flight
(combine_moe_route_tokens_b200.Pipeline) — batch i's route and layout run on a side
stream beside batch i-1's combine, the permutes and combines stay in batch order —
the K batches captured as one CUDA graph and replayed once. Beside it (``serial``):
the same K batches one at a time through the fused dispatch call (moe_dispatch), each
round of buffer sets captured as one CUDA graph of the same C-ABI calls and replayed
(``--schedule serial`` makes that the headline; ``--eager``: the calls themselves).
Per-call times come from an eager pass with CUDA events around every call, and from
the step's own replays (a round minus the round without the call).
N > 1 (torchrun, one process per GPU): each rank processes its own batch
(data-parallel, independent seeds, no collective on the data path); timing is
the max over ranks; ``value`` counts the tokens of all ranks.

``--impl reference`` times the plain CPU oracle on this machine's host cores
on a bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synthetic import get_workload, make_inputs  # noqa: E402

METRIC = "dispatch+combine tokens/s and effective HBM GB/s (% of B200 peak), 1 GPU"
L2_BYTES = 126 * 1024 * 1024
E2E_DEPTH = 3  # device buffer sets the end-to-end pipeline rotates over
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------- helpers


# C-ABI calls that enqueue more than one kernel (the dispatch layout: count + look-back,
# then the row-map fill; the fused dispatch: count + look-back, then fill + row copy; the
# dedup layout: placement, then the per-row fill); every other call is one kernel
KERNELS_PER_CALL = {"layout": 2, "dispatch": 2, "dedup_layout": 2}


def kernels_per_call(name: str) -> int:
    """Kernels one call enqueues; per-peer names such as 'layout.1' count as their base call."""
    return KERNELS_PER_CALL.get(name.split(".")[0], 1)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank value over all ranks (the value itself without a process group)."""
    import torch
    import torch.distributed as tdist

    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(w, rank: int) -> dict:
    """Each data-parallel rank processes its own batch: the workload's recipe with seed + rank."""
    return make_inputs(w, grad=w.backward, seed_offset=rank)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments and whitespace (what the compiler sees as code)."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return "".join(text.split())


def source_digest():
    """Digest of the kernel sources' code (comments and layout ignored), to tell whether a
    stored ncu capture still applies."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "combine_moe_route_tokens_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from a committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload][kernel]
        if e.get("source_digest") == source_digest():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle",
        0x2: "applications_clocks_setting",
        0x4: "sw_power_cap",
        0x8: "hw_slowdown",
        0x10: "sync_boost",
        0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []  # (time.perf_counter(), SM MHz, reason bits)
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
                self.samples.append((time.perf_counter(), mhz, bits))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop.clear()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._thread = None

    @staticmethod
    def mark() -> float:
        return time.perf_counter()

    def summary(self, window=None):
        """Median SM clock and the clock-event reasons over every sample taken while the
        GPU ran the benchmark (warm-up, both timed passes, the other workloads), with the
        sample count; the same for the samples inside the headline's timed region."""
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml_unavailable"]}

        def names(bits):
            return [n for bit, n in self.REASONS.items() if bits & bit]

        allbits = 0
        for _, _, b in self.samples:
            allbits |= b
        out = {
            "sm_mhz": statistics.median([m for _, m, _ in self.samples]) if self.samples else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": names(allbits),
            "samples": len(self.samples),
            "sampled": "NVML every ~1 ms while the GPU ran the benchmark's steps",
        }
        if window is not None:
            inside = [(m, b) for t, m, b in self.samples if window[0] <= t <= window[1]]
            wbits = 0
            for _, b in inside:
                wbits |= b
            out["timed_region"] = {
                "sm_mhz": statistics.median([m for m, _ in inside]) if inside else None,
                "reasons": names(wbits),
                "samples": len(inside),
                "window": f"the timed region, then untimed repetitions of the same steps: ~{CLOCK_WINDOW_MS:.0f} ms",
            }
        return out


# ------------------------------------------------------------- GPU arm


class Step:
    """One step of the hot path with every C-ABI argument marshalled up front.

    With TP folding (workload tp_size = T > 1) the step routes once, builds the
    layout and the send buffer of every peer in turn (all on this GPU), and
    restores with one slot-ordered combine over the peers' buffers."""

    def __init__(self, w, moe, native, torch, sets, device, unfused=False, bulk_copy=False):
        self.w = w
        self.torch = torch
        self.lib = native.lib()
        T = max(w.tp_size, 1)
        self.T = T
        flags = moe.MOE_FLAG_DISPATCH_BULK_COPY if bulk_copy else 0
        self.problems = [moe.Problem(N=w.N, H=w.H, k=w.k, E_log=w.E_log, R=w.R, capacity=w.capacity,
                                     num_replicas=w.num_replicas, row_align=w.row_align,
                                     tp_size=w.tp_size, tp_rank=r, flags=flags) for r in range(T)]
        p = self.problems[0]
        self.problem = p
        self.layouts = [moe.Layout.allocate(q, device) for q in self.problems]
        self.layout = self.layouts[0]
        self.sets = sets
        N, H, k = w.N, w.H, w.k
        RM = p.rows_max
        self.idx = torch.empty((N, k), dtype=torch.int32, device=device)
        self.probs = torch.empty((N, k), dtype=torch.float32, device=device)
        self.sends = [torch.empty((RM, H), dtype=torch.bfloat16, device=device) for _ in range(T)]
        self.send = self.sends[0]
        self.out = torch.empty((N, H), dtype=torch.bfloat16, device=device)
        if w.backward:
            self.gy = torch.empty((RM, H), dtype=torch.bfloat16, device=device)
            self.gp = torch.empty((N, k), dtype=torch.float32, device=device)
            self.gh = torch.empty((N, H), dtype=torch.bfloat16, device=device)
        if w.dedup:
            self.dedup = moe.DedupView.allocate(p, device)
            self._D = self.dedup.c_struct()
            self.recv_x = torch.empty((self.dedup.recv_max, H), dtype=torch.bfloat16, device=device)
            self.partial = torch.empty((self.dedup.recv_max, H), dtype=torch.bfloat16, device=device)
        self._ps = [q.c_struct() for q in self.problems]
        self._Ls = [L.c_struct() for L in self.layouts]
        self._L_arr = (native.MoeLayout * T)(*self._Ls)
        self._y_arr = (ctypes.c_void_p * T)(*[y.data_ptr() for y in self.sends])
        self.stream = torch.cuda.current_stream(device)
        self._s = ctypes.c_void_p(self.stream.cuda_stream)
        vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        P, L = ctypes.byref(self._ps[0]), ctypes.byref(self._Ls[0])
        self.calls = []
        for s in sets:
            c = [("route", self.lib.moe_route_topk,
                  (vp(s["logits"]), None, N, w.E_log, k, vp(self.idx), vp(self.probs), self._s))]
            if T == 1 and w.dedup:
                ws = self.layout.workspace
                D = ctypes.byref(self._D)
                if unfused:
                    c += [("layout", self.lib.moe_dispatch_layout,
                           (P, vp(self.idx), vp(self.probs), L, vp(ws), ws.numel(), self._s))]
                else:  # the layout and the send buffer in one call
                    c += [("dispatch", self.lib.moe_dispatch,
                           (P, vp(self.idx), vp(self.probs), L, vp(ws), ws.numel(), vp(s["hidden"]), vp(self.send),
                            self._s))]
                c += [
                    ("dedup_layout", self.lib.moe_dedup_layout,
                     (P, L, vp(self.probs), D, vp(self.dedup.workspace), self.dedup.workspace.numel(), self._s)),
                    ("dedup_dispatch", self.lib.moe_dedup_dispatch, (P, D, vp(s["hidden"]), vp(self.recv_x), self._s)),
                ]
                if unfused:
                    c += [("permute", self.lib.moe_permute, (P, L, vp(s["hidden"]), vp(self.send), self._s))]
                c += [
                    ("dedup_combine_local", self.lib.moe_dedup_combine_local,
                     (P, L, D, vp(self.send), vp(self.probs), vp(self.partial), self._s)),
                    ("dedup_combine", self.lib.moe_dedup_combine, (P, D, vp(self.partial), vp(self.out), self._s)),
                ]
            elif T == 1 and not unfused:
                ws = self.layout.workspace
                c += [
                    ("dispatch", self.lib.moe_dispatch,
                     (P, vp(self.idx), vp(self.probs), L, vp(ws), ws.numel(), vp(s["hidden"]), vp(self.send),
                      self._s)),
                    ("combine", self.lib.moe_combine, (P, L, vp(self.send), vp(self.probs), vp(self.out), self._s)),
                ]
            elif T == 1:
                ws = self.layout.workspace
                c += [
                    ("layout", self.lib.moe_dispatch_layout,
                     (P, vp(self.idx), vp(self.probs), L, vp(ws), ws.numel(), self._s)),
                    ("permute", self.lib.moe_permute, (P, L, vp(s["hidden"]), vp(self.send), self._s)),
                    ("combine", self.lib.moe_combine, (P, L, vp(self.send), vp(self.probs), vp(self.out), self._s)),
                ]
            else:
                for r in range(T):
                    Pr, Lr = ctypes.byref(self._ps[r]), ctypes.byref(self._Ls[r])
                    ws = self.layouts[r].workspace
                    if unfused:
                        c += [
                            (f"layout.{r}", self.lib.moe_dispatch_layout,
                             (Pr, vp(self.idx), vp(self.probs), Lr, vp(ws), ws.numel(), self._s)),
                            (f"permute.{r}", self.lib.moe_permute,
                             (Pr, Lr, vp(s["hidden"]), vp(self.sends[r]), self._s)),
                        ]
                    else:  # each peer's layout and send buffer in one call
                        c += [(f"dispatch.{r}", self.lib.moe_dispatch,
                               (Pr, vp(self.idx), vp(self.probs), Lr, vp(ws), ws.numel(), vp(s["hidden"]),
                                vp(self.sends[r]), self._s))]
                c += [("restore", self.lib.moe_restore_combined,
                       (P, self._L_arr, self._y_arr, vp(self.probs), vp(self.out), self._s))]
            if w.backward:
                c += [
                    ("combine_backward", self.lib.moe_combine_backward,
                     (P, L, vp(s["grad_out"]), vp(self.send), vp(self.probs), vp(self.gy), vp(self.gp), self._s)),
                    ("permute_backward", self.lib.moe_permute_backward, (P, L, vp(self.gy), vp(self.gh), self._s)),
                ]
            self.calls.append(c)
        self.kernel_names = [name for name, _, _ in self.calls[0]]

    def run(self, i, events=None, skip=()):
        """Enqueue step i (buffer set i mod sets); calls named in `skip` are left out."""
        for n, (name, fn, args) in enumerate(self.calls[i % len(self.calls)]):
            if name in skip:
                continue
            if events is not None:
                events[n][0].record(self.stream)
            rc = fn(*args)
            if rc != 0:
                raise RuntimeError(f"{name} returned {rc}")
            if events is not None:
                events[n][1].record(self.stream)

    def clear_status(self) -> None:
        for L in self.layouts:
            L.clear_status()
        if self.w.dedup:
            self.dedup.tensors["status"].zero_()

    def status(self) -> int:
        st = 0
        for L in self.layouts:
            st |= L.status()
        if self.w.dedup:
            st |= self.dedup.status()
        return st

    def algorithmic_bytes(self) -> dict:
        """Bytes each kernel must move at least once, from the last step's layouts.

        A row of hidden is read only if its token keeps a slot; every send row is
        written (pads as zeros); the combine reads only kept rows."""
        w, T = self.w, self.T
        N, H, k, E = w.N, w.H, w.k, w.E_log
        NK, row, RM = N * k, H * 2, self.problem.rows_max
        kept = [int(L["counters"][1].item()) for L in self.layouts]
        read = [int((L["dest_row"] >= 0).any(dim=1).sum().item()) for L in self.layouts]
        layout_bytes = NK * 8 + NK * (4 + 4 + 4 + 1) + RM * (4 * 4 + 1) + w.R * NK * 4
        out = {"route": N * E * 4 + NK * 8}
        if T == 1:
            out["layout"] = layout_bytes
            out["permute"] = read[0] * row + RM * row + NK * 4 + RM
            # the fused call moves the layout's bytes and the row copy's, without the
            # permute's re-read of the row map
            out["dispatch"] = layout_bytes + read[0] * row + RM * row
            out["combine"] = kept[0] * row + N * row + NK * 8
        else:
            for r in range(T):
                out[f"layout.{r}"] = layout_bytes
                out[f"permute.{r}"] = read[r] * row + RM * row + NK * 4 + RM
                out[f"dispatch.{r}"] = layout_bytes + read[r] * row + RM * row
            out["restore"] = sum(kept) * row + N * row + NK * 4 * (T + 1)
        if w.dedup:
            RR = self.dedup.recv_max
            nrecv = int(self.dedup["num_recv"].item())
            out["dedup_layout"] = NK * 8 + NK * 4 + N * w.R * 5 + RR * (4 + 1 + k * 8 + (w.R and (E // w.R)) * 5)
            out["dedup_dispatch"] = read[0] * row + RR * row + N * w.R * 4 + RR
            out["dedup_combine_local"] = kept[0] * row + RR * row + NK * 8 + RR * 4
            out["dedup_combine"] = nrecv * row + N * row + N * w.R * 4
        out["combine_backward"] = N * row + kept[0] * row + RM * row + NK * 8 + NK * 4
        out["permute_backward"] = kept[0] * row + N * row + NK * 4
        return out


class EpStep:
    """One step of the expert-parallel exchange between R ranks simulated on this GPU.

    The workload's N tokens are split evenly over the R ranks, and each rank's calls
    run on a stream of its own, as the ranks would on GPUs of their own. Every rank
    routes and lays out its own tokens (its layout writes its expert_offsets straight
    into row r of one [R, E+1] table: the stand-in for the all-gather); after all
    layouts every rank plans and dispatches into the owners' receive buffers; after
    all dispatches every rank combines from them (identity experts). The step then
    joins the ranks' streams. Calls of the same kind share a name in the per-call table."""

    PHASES = ("route", "layout", "ep_plan", "ep_dispatch", "ep_combine")

    def __init__(self, w, moe, native, torch, sets, device):
        self.w = w
        self.torch = torch
        self.lib = native.lib()
        R, H, k, E = w.R, w.H, w.k, w.E
        if w.N % R:
            raise ValueError("the EP workload needs N divisible by R")
        n = w.N // R
        self.n = n
        p = moe.Problem(N=n, H=H, k=k, E_log=w.E_log, R=R, capacity=w.capacity, num_replicas=w.num_replicas,
                        row_align=w.row_align)
        self.problem = p
        self.offsets_all = torch.zeros((R, E + 1), dtype=torch.int32, device=device)
        self.layouts = []
        for r in range(R):
            G = moe.Layout.allocate(p, device)
            G.tensors["expert_offsets"] = self.offsets_all[r]  # the layout writes its row of the table
            self.layouts.append(G)
        self.plans = [moe.EpPlan.allocate(p, device) for _ in range(R)]
        RR = moe.moe_ep_recv_rows_max(p)
        self.recv = [torch.empty((RR, H), dtype=torch.bfloat16, device=device) for _ in range(R)]
        self.table = moe.peer_table(self.recv)
        self.sets = sets
        self.idx = torch.empty((w.N, k), dtype=torch.int32, device=device)
        self.probs = torch.empty((w.N, k), dtype=torch.float32, device=device)
        self.out = torch.empty((w.N, H), dtype=torch.bfloat16, device=device)
        self._p = p.c_struct()
        self._Ls = [G.c_struct() for G in self.layouts]
        self.stream = torch.cuda.current_stream(device)
        self.rank_streams = [torch.cuda.Stream(device) for _ in range(R)]
        self._rs = [ctypes.c_void_p(st.cuda_stream) for st in self.rank_streams]
        ev = lambda: torch.cuda.Event()  # noqa: E731
        self._start = ev()
        self._phase_done = [[ev() for _ in range(R)] for _ in self.PHASES]
        vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        P = ctypes.byref(self._p)
        lib = self.lib
        self.calls = []  # per set: {phase: [(name, fn, args) for each rank]}
        for st in sets:
            rows = [slice(r * n, (r + 1) * n) for r in range(R)]
            ph = {
                "route": [("route", lib.moe_route_topk,
                           (vp(st["logits"][rows[r]]), None, n, w.E_log, k, vp(self.idx[rows[r]]),
                            vp(self.probs[rows[r]]), self._rs[r])) for r in range(R)],
                "layout": [("layout", lib.moe_dispatch_layout,
                            (P, vp(self.idx[rows[r]]), vp(self.probs[rows[r]]), ctypes.byref(self._Ls[r]),
                             vp(self.layouts[r].workspace), self.layouts[r].workspace.numel(), self._rs[r]))
                           for r in range(R)],
                "ep_plan": [("ep_plan", lib.moe_ep_plan,
                             (P, vp(self.offsets_all), r, vp(self.plans[r].base),
                              vp(self.plans[r].recv_expert_offsets), vp(self.plans[r].num_recv),
                              vp(self.plans[r].status), self._rs[r])) for r in range(R)],
                "ep_dispatch": [("ep_dispatch", lib.moe_ep_dispatch,
                                 (P, ctypes.byref(self._Ls[r]), vp(self.plans[r].base), vp(st["hidden"][rows[r]]),
                                  vp(self.table), self._rs[r])) for r in range(R)],
                "ep_combine": [("ep_combine", lib.moe_ep_combine,
                                (P, ctypes.byref(self._Ls[r]), vp(self.plans[r].base), vp(self.table),
                                 vp(self.probs[rows[r]]), vp(self.out[rows[r]]), self._rs[r])) for r in range(R)],
            }
            self.calls.append(ph)
        self.kernel_names = [name for phase in self.PHASES for name, _, _ in self.calls[0][phase]]

    def run(self, i, events=None, skip=()):
        """Fork to the ranks' streams; join where a phase needs every rank's previous one.
        Calls named in `skip` are left out (their phase's join events are still recorded)."""
        R = self.w.R
        ph = self.calls[i % len(self.calls)]
        self._start.record(self.stream)
        for st in self.rank_streams:
            st.wait_event(self._start)
        n = 0
        for p_i, phase in enumerate(self.PHASES):
            if phase in ("ep_plan", "ep_combine"):  # needs every rank's layout / dispatch
                for st in self.rank_streams:
                    for e in self._phase_done[p_i - 1]:
                        st.wait_event(e)
            for r, (name, fn, args) in enumerate(ph[phase]):
                if events is not None:
                    events[n][0].record(self.rank_streams[r])
                rc = 0 if name in skip else fn(*args)
                if rc != 0:
                    raise RuntimeError(f"{name} returned {rc}")
                if events is not None:
                    events[n][1].record(self.rank_streams[r])
                self._phase_done[p_i][r].record(self.rank_streams[r])
                n += 1
        for r in range(R):
            self.stream.wait_event(self._phase_done[-1][r])

    def status(self) -> int:
        st = 0
        for G in self.layouts:
            st |= G.status()
        for pl in self.plans:
            st |= int(pl.status.item())
        return st

    def clear_status(self) -> None:
        for G in self.layouts:
            G.clear_status()
        for pl in self.plans:
            pl.status.zero_()

    def algorithmic_bytes(self) -> dict:
        """Bytes per call (the mean over the R ranks), each row moved once."""
        w, R, n = self.w, self.w.R, self.n
        H, k, E = w.H, w.k, w.E
        row, NK, RM = 2 * H, n * k, self.problem.rows_max
        kept = [int(G["counters"][1].item()) for G in self.layouts]
        read = [int((G["dest_row"] >= 0).any(dim=1).sum().item()) for G in self.layouts]
        rows = [int(G["num_rows"].item()) for G in self.layouts]
        mean = lambda v: sum(v) / len(v)  # noqa: E731
        layout_bytes = NK * 8 + NK * (4 + 4 + 4 + 1) + RM * (4 * 4 + 1) + R * NK * 4
        return {
            "route": n * w.E_log * 4 + NK * 8,
            "layout": layout_bytes,
            "ep_plan": R * (E + 1) * 4 + E * 4 + (E // R + 2) * 4,
            "ep_dispatch": round(mean([read[r] * row + rows[r] * row + NK * 8 + E * 12 for r in range(R)])),
            "ep_combine": round(mean([kept[r] * row + n * row + NK * 12 + E * 8 for r in range(R)])),
        }


def device_sets(w, host, torch, device):
    """Input buffer sets resident in HBM: one generated batch plus token-rotated copies
    of it (same distribution, different buffers and token order), together larger than
    twice the 126 MB L2 so that no step reads inputs a previous step left in L2."""
    set_bytes = sum(v.nbytes for v in host.values())
    nsets = max(2, min(8, math.ceil(2 * L2_BYTES / set_bytes)))
    base = {
        "logits": torch.from_numpy(host["logits"]).to(device),
        "hidden": torch.from_numpy(host["hidden"].view(np.int16)).to(device).view(torch.bfloat16),
    }
    if w.backward:
        base["grad_out"] = torch.from_numpy(host["grad_out"].view(np.int16)).to(device).view(torch.bfloat16)
    sets = []
    for s in range(nsets):
        shift = (s * 7919) % max(w.N, 1)
        sets.append({key: torch.roll(v, shifts=shift, dims=0).contiguous() for key, v in base.items()})
    return sets, nsets, set_bytes


def measure(w, host, steps, warmup, eager, hot_l2, ctx):
    """Times `steps` whole steps of workload `w` on this rank's GPU.

    Timed region 1: the K steps back to back between two CUDA events on the launching
    stream (each buffer set's step captured once into a CUDA graph and replayed, unless
    `eager`), barrier and synchronize on both sides, max over ranks. Optionally the same
    K steps on one buffer set (inputs in L2, for comparison). Timed region 2: the same K
    steps launched eagerly with events around every call, for per-call durations."""
    torch, moe, _native, device, barrier = ctx["torch"], ctx["moe"], ctx["native"], ctx["device"], ctx["barrier"]
    sets, nsets, set_bytes = device_sets(w, host, torch, device)
    # a stream of our own (not the legacy default stream), so that steps can be captured
    work_stream = torch.cuda.Stream(device)
    with torch.cuda.stream(work_stream):
        step = EpStep(w, moe, _native, torch, sets, device) if w.ep else \
            Step(w, moe, _native, torch, sets, device, unfused=ctx.get("unfused", False),
                 bulk_copy=ctx.get("bulk_copy", False))
    for i in range(warmup):
        step.run(i)
    torch.cuda.synchronize()
    abytes = step.algorithmic_bytes()

    # The steps captured from the same C-ABI calls into CUDA graphs (the launches keep
    # their programmatic-dependent-launch edges, also from one step's last kernel to the
    # next step's first): one graph per buffer set, and one holding the steps of all sets
    # in order, which the timed region replays whenever a whole round of sets is left.
    nsets_g = len(step.calls)
    run_step = step.run
    launch_mode = "eager C-ABI calls, programmatic dependent launch"
    graphs, rounds = [], {}

    def capture_round(skip=()):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=work_stream):
            for i in range(nsets_g):
                step.run(i, skip=skip)
        return g

    if not eager:
        try:
            for i in range(nsets_g):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=work_stream):
                    step.run(i)
                graphs.append(g)
            rounds[()] = capture_round()
        except Exception as exc:  # a driver without capture support: time the calls themselves
            graphs, rounds = [], {}
            torch.cuda.synchronize()
            launch_mode += f" (graph capture failed: {type(exc).__name__})"
    if graphs:
        launch_mode = (f"CUDA graphs of the captured C-ABI calls (programmatic dependent launch), replayed: one "
                       f"holding the steps of all {nsets_g} buffer sets in order, one per set for the rest")

        def run_step(i, events=None):
            with torch.cuda.stream(work_stream):  # replay where the events are recorded
                graphs[i % nsets_g].replay()

        for i in range(warmup):
            run_step(i)
        torch.cuda.synchronize()

    def run_steps(first, count):
        """Steps first .. first+count-1: whole rounds of buffer sets from the round graph."""
        i = 0
        while i < count:
            if rounds and (first + i) % nsets_g == 0 and count - i >= nsets_g:
                with torch.cuda.stream(work_stream):
                    rounds[()].replay()
                i += nsets_g
            else:
                run_step(first + i)
                i += 1

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    tr0 = ctx["sampler"].mark()
    t0.record(step.stream)
    run_steps(warmup, steps)
    t1.record(step.stream)
    torch.cuda.synchronize()
    for _ in range(clock_tail_reps(t0.elapsed_time(t1))):  # the clock window's tail (see clock_tail_reps)
        run_steps(warmup, steps)
    torch.cuda.synchronize()
    tr1 = ctx["sampler"].mark()
    barrier()
    elapsed_ms = t0.elapsed_time(t1)
    status = step.status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the timed steps of '{w.name}'")
    in_step = in_step_costs(step, rounds, capture_round, work_stream, torch) if rounds else {}
    hot_ms = None
    if hot_l2:
        h0 = torch.cuda.Event(enable_timing=True)
        h1 = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        h0.record(step.stream)
        for i in range(steps):
            run_step(0)
        h1.record(step.stream)
        torch.cuda.synchronize()
        barrier()
        hot_ms = max_over_ranks(h0.elapsed_time(h1), device)
    nk = len(step.kernel_names)
    events = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
              for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        step.run(warmup + i, events[i])
    torch.cuda.synchronize()
    barrier()
    per_kernel_ms = {name: [] for name in step.kernel_names}
    for i in range(steps):
        for n, name in enumerate(step.kernel_names):
            per_kernel_ms[name].append(events[i][n][0].elapsed_time(events[i][n][1]))
    status = step.status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the timed steps of '{w.name}'")
    elapsed_ms = max_over_ranks(elapsed_ms, device)
    del graphs, rounds
    return {
        "step": step, "abytes": abytes, "elapsed_ms": elapsed_ms, "hot_ms": hot_ms, "per_kernel_ms": per_kernel_ms,
        "in_step_us": in_step,
        "launch_mode": launch_mode, "nsets": nsets, "set_bytes": set_bytes, "timed_window": (tr0, tr1),
    }


CLOCK_WINDOW_MS = 30.0


def clock_tail_reps(timed_ms: float) -> int:
    """Untimed repetitions of the timed work that follow it inside the clock record's
    window, so that the window lasts about CLOCK_WINDOW_MS."""
    return max(0, math.ceil((CLOCK_WINDOW_MS - timed_ms) / max(timed_ms, 1e-3)))


def pipelined_eligible(w) -> bool:
    """Workloads whose step is route -> layout -> permute -> combine on one rank."""
    return w.tp_size <= 1 and not w.dedup and not w.ep and not w.backward


def measure_pipelined(w, host, steps, warmup, ctx):
    """The same steps with two batches in flight (combine_moe_route_tokens_b200.Pipeline):
    batch i's route and layout run on a side stream beside batch i-1's combine; the
    permutes and combines stay in batch order on the launching stream. Warm-up: `warmup`
    batches enqueued from the host, then one untimed replay of the timed graph (its
    upload); timed: the K batches captured as one CUDA graph, replayed once between two
    CUDA events on the launching stream, barrier and synchronize on both sides."""
    torch, moe, device, barrier = ctx["torch"], ctx["moe"], ctx["device"], ctx["barrier"]
    sets, nsets, set_bytes = device_sets(w, host, torch, device)
    p = moe.Problem(N=w.N, H=w.H, k=w.k, E_log=w.E_log, R=w.R, capacity=w.capacity,
                    num_replicas=w.num_replicas, row_align=w.row_align)
    work = torch.cuda.Stream(device)
    pipe = moe.Pipeline(p, device=device, stream=work)

    def enqueue(first, count):
        ready = torch.cuda.Event()  # the inputs are resident before the first batch
        ready.record(work)
        for i in range(first, first + count):
            s = sets[i % nsets]
            pipe.submit(s["logits"], s["hidden"], ready=ready)
        pipe.join()

    with torch.cuda.stream(work):
        enqueue(0, warmup)
    torch.cuda.synchronize()
    pipe.reset()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=work):
        enqueue(warmup, steps)
    with torch.cuda.stream(work):
        g.replay()
    torch.cuda.synchronize()
    status = pipe.status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the pipelined warm-up of '{w.name}'")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    tr0 = ctx["sampler"].mark()
    t0.record(work)
    with torch.cuda.stream(work):
        g.replay()
    t1.record(work)
    torch.cuda.synchronize()
    # the clock record's window: the timed replay and, right after it, enough untimed
    # replays of the same graph to give the ~1 ms NVML sampler a few dozen samples
    more = clock_tail_reps(t0.elapsed_time(t1))
    with torch.cuda.stream(work):
        for _ in range(more):
            g.replay()
    torch.cuda.synchronize()
    tr1 = ctx["sampler"].mark()
    barrier()
    status = pipe.status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the pipelined steps of '{w.name}'")
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), device)
    del g, pipe, sets
    torch.cuda.synchronize()
    return {"elapsed_ms": elapsed_ms, "timed_window": (tr0, tr1), "nsets": nsets, "set_bytes": set_bytes,
            "clock_tail_reps": more}


def in_step_costs(step, rounds, capture_round, stream, torch, target_steps=40, trials=3):
    """What each call costs inside the replayed steps: the time of a round of all buffer
    sets' steps, minus the same round captured without that call (the other calls then
    read what earlier steps left, which stays inside their buffers), per call. Rounds are
    replayed back to back, alternating between the variants; the median of `trials`.
    Leaves the device status words cleared (a call left out can make a later one report
    rows of another layout)."""
    names = list(dict.fromkeys(step.kernel_names))
    nsets = len(step.calls)
    reps = max(2, -(-target_steps // nsets))
    variants = {(): rounds[()]}
    for n in names:
        variants[(n,)] = capture_round(skip=(n,))
    times = {key: [] for key in variants}
    for _ in range(trials):
        for key, g in variants.items():
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                g.replay()  # warm
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            torch.cuda.synchronize()
            times[key].append(e0.elapsed_time(e1) * 1e3 / (reps * nsets))  # µs per step
    med = {key: statistics.median(v) for key, v in times.items()}
    del variants
    step.clear_status()
    torch.cuda.synchronize()
    out = {"step_us": round(med[()], 2)}
    for n in names:
        out[n] = round((med[()] - med[(n,)]) / step.kernel_names.count(n), 2)
    return out


def kernel_table(m, peak):
    """Per-call figures of a measurement: mean / median / p10 / p90 µs, algorithmic bytes, GB/s, frac."""
    step = m["step"]
    kernels = {}
    for name in step.kernel_names:
        vals = m["per_kernel_ms"][name]
        avg_ms = statistics.mean(vals)
        qs = statistics.quantiles(vals, n=10) if len(vals) > 1 else [avg_ms] * 9
        gbs = m["abytes"][name] / (avg_ms * 1e-3) / 1e9
        kernels[name] = {
            "calls_per_step": step.kernel_names.count(name),
            "us": round(avg_ms * 1e3, 2),
            "median_us": round(statistics.median(vals) * 1e3, 2),
            "p10_us": round(qs[0] * 1e3, 2),
            "p90_us": round(qs[8] * 1e3, 2),
            "algorithmic_bytes": m["abytes"][name],
            "gbs": round(gbs, 1),
            "frac": round(gbs / peak, 3),
        }
        ins = m.get("in_step_us", {}).get(name)
        if ins is not None and ins > 0:
            kernels[name]["in_step_us"] = ins
            kernels[name]["in_step_frac"] = round(m["abytes"][name] / (ins * 1e-6) / 1e9 / peak, 3)
    return kernels


# Timed beside the headline in the default run: the other surveyed configurations and the
# workloads of the rows built past them (row alignment, TP folding, the DeepEP-style dedup
# view, the exchange between 4 ranks on this GPU); each gets its step time, per-call figures
# and roofline fractions.
EXTRA_WORKLOADS = ("tiny", "qwen3", "capacity", "ultraep", "ht_align16", "ht_tp2", "ht_dedup", "ht_ep4")
EXTRA_STEPS, EXTRA_WARMUP = 20, 3


def run_ours(args, ws, rank, local):
    import torch
    import torch.distributed as tdist

    import combine_moe_route_tokens_b200 as moe
    from combine_moe_route_tokens_b200 import _native
    from combine_moe_route_tokens_b200.build import build

    if ws > 1:
        tdist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if local == 0:  # one build per node; the other ranks wait for it
        build()
    if ws > 1:
        tdist.barrier()
    moe.load_library()

    def barrier():
        if ws > 1:
            tdist.barrier()

    w = get_workload(args.workload)
    if args.tokens:  # a smaller batch of the same workload (profiling captures), named as such
        w = w.scaled(args.tokens)
    host = rank_inputs(w, rank)
    sampler = ClockSampler(local)
    ctx = {"torch": torch, "moe": moe, "native": _native, "device": device, "barrier": barrier, "sampler": sampler,
           "unfused": args.unfused, "bulk_copy": args.bulk_copy}
    # The headline schedule: two batches in flight (the layout as its own call on a side
    # stream, so the per-call figures are those of route, layout, permute and combine), with
    # the one-batch-at-a-time step of the fused dispatch beside it; or that serial step.
    pipelined = (args.schedule == "pipelined" and pipelined_eligible(w) and not args.eager and not args.bulk_copy
                 and not args.unfused)
    mp = m_serial = None
    with sampler:
        if pipelined:
            m = measure(w, host, args.steps, args.warmup, args.eager, True, {**ctx, "unfused": True})
            m_serial = measure(w, host, args.steps, args.warmup, args.eager, False, ctx)
            mp = measure_pipelined(w, host, args.steps, args.warmup, ctx)
        else:
            m = measure(w, host, args.steps, args.warmup, args.eager, True, ctx)
    step, abytes, elapsed_ms, hot_ms = m["step"], m["abytes"], m["elapsed_ms"], m["hot_ms"]
    if mp is not None:
        elapsed_ms = mp["elapsed_ms"]

    # end to end through the public API: every step copies its inputs in from pinned host
    # memory and its combined output back out. E2E_DEPTH sets of device buffers rotate, so
    # step i's copy-out (one copy engine) overlaps the next steps' copy-in (the other) and
    # kernels; each step waits for the copy-in of its own inputs, and a buffer is written
    # again only after its previous copy-out finished.
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(w, host, step, args, ws, ctx)

    # the other surveyed configurations, a short run each (default run only)
    extra = {}
    if not args.workload_given and not args.tokens and not args.no_extra:
        with sampler:
            for name in EXTRA_WORKLOADS:
                wx = get_workload(name)
                hx = rank_inputs(wx, rank)
                mx = measure(wx, hx, EXTRA_STEPS, EXTRA_WARMUP, args.eager, False, ctx)
                if wx.tp_size <= 1 and not wx.dedup and not wx.ep and not args.unfused and not args.bulk_copy:
                    # the same step with the layout and the permute as separate calls (the permute's own figures)
                    mx["separate"] = measure(wx, hx, EXTRA_STEPS, EXTRA_WARMUP, args.eager, False,
                                             {**ctx, "unfused": True})
                if pipelined_eligible(wx) and not args.eager and not args.bulk_copy and not args.unfused:
                    mx["pipelined"] = measure_pipelined(wx, hx, EXTRA_STEPS, EXTRA_WARMUP, ctx)
                extra[name] = mx
                torch.cuda.empty_cache()

    if ws > 1:
        tdist.barrier()
        tdist.destroy_process_group()
    if rank != 0:
        return None

    peak, peak_kind = measured_peaks()
    kernels = kernel_table(m, peak)
    dominant = max(m["step"].kernel_names, key=lambda n: kernels[n]["us"])
    ach = kernels[dominant]["gbs"]
    ms_step = elapsed_ms / args.steps
    path_bytes = sum(abytes[n] for n in m["step"].kernel_names)
    workloads = {}
    for name, mx in extra.items():
        kx = kernel_table(mx, peak)
        msx = mx["elapsed_ms"] / EXTRA_STEPS
        bx = sum(mx["abytes"][n] for n in mx["step"].kernel_names)
        wx = mx["step"].w
        dom = max(mx["step"].kernel_names, key=lambda n: kx[n]["us"])
        workloads[name] = {
            "config": wx.describe(),
            "steps": EXTRA_STEPS,
            "warmup": EXTRA_WARMUP,
            "ms_per_step": round(msx, 4),
            "tokens_per_s": round(wx.N * EXTRA_STEPS * ws / (mx["elapsed_ms"] / 1e3), 1),
            "effective_gbs": round(bx / (msx * 1e-3) / 1e9, 1),
            "effective_hbm_frac": round(bx / (msx * 1e-3) / 1e9 / peak, 3),
            "dominant": dom,
            "kernels": kx,
            "l2": f"inputs rotated over {mx['nsets']} buffer sets ({mx['nsets'] * mx['set_bytes'] / 2**20:.0f} MiB)",
            "launch": mx["launch_mode"],
            "schedule": "one batch at a time",
        }
        if "separate" in mx:
            ms_sep = mx["separate"]
            workloads[name]["separate_calls"] = {
                "ms_per_step": round(ms_sep["elapsed_ms"] / EXTRA_STEPS, 4),
                "kernels": kernel_table(ms_sep, peak),
                "note": "one batch at a time, moe_dispatch_layout then moe_permute",
            }
        if "pipelined" in mx:  # the same calls split (layout, then permute), two batches in flight
            pm = mx["pipelined"]["elapsed_ms"]
            workloads[name]["pipelined"] = {
                "ms_per_step": round(pm / EXTRA_STEPS, 4),
                "tokens_per_s": round(wx.N * EXTRA_STEPS * ws / (pm / 1e3), 1),
                "schedule": "two batches in flight (Pipeline): route and layout beside the previous combine",
            }
    result = {
        "metric": METRIC,
        "value": round(w.N * args.steps * ws / (elapsed_ms / 1e3), 1),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "accumulate": "fp32 (combine and backward)",
        "data": "synthetic",
        "config": {
            **w.describe(),
            "parallelism": f"dp{ws}: independent batch per GPU, no collective on the data path",
            "step": "+".join(dict.fromkeys(
                f"{n}x{m['step'].kernel_names.count(n)}" if m["step"].kernel_names.count(n) > 1 else n
                for n in m["step"].kernel_names)),
            "l2": f"inputs rotated over {m['nsets']} buffer sets ({m['nsets'] * m['set_bytes'] / 2**20:.0f} MiB "
                  f"> 126 MB L2), no flush",
            "dispatch": ("moe_dispatch_layout on a side stream, then moe_permute (two batches in flight)"
                         if mp is not None else
                         "moe_dispatch_layout + moe_permute (separate calls)" if args.unfused else
                         "moe_dispatch (layout + permute fused), rows copied with "
                         + ("bulk (TMA) copies through shared memory" if args.bulk_copy else "16-byte vector copies")),
            "schedule": ("two batches in flight (combine_moe_route_tokens_b200.Pipeline): batch i's route and "
                         "layout on a side stream beside batch i-1's combine; permutes and combines in batch order"
                         if mp is not None else "one batch at a time"),
        },
        "effective_gbs": round(path_bytes / (ms_step * 1e-3) / 1e9, 1),
        "effective_hbm_frac": round(path_bytes / (ms_step * 1e-3) / 1e9 / peak, 3),
        "kernels": kernels,
        "roofline": {
            "kernel": dominant,
            "bound": "hbm",
            "achieved": ach,
            "peak": peak,
            "peak_source": f"{peak_kind} hbm_gbs",
            "unit": "GB/s",
            "frac": round(ach / peak, 3),
            "traffic": stored_traffic(dominant, w.name),
            **({"in_step_achieved": round(m["abytes"][dominant] / (kernels[dominant]["in_step_us"] * 1e-6) / 1e9, 1),
                "in_step_frac": kernels[dominant]["in_step_frac"]} if "in_step_us" in kernels[dominant] else {}),
        },
        "gpu_launches": args.steps * sum(kernels_per_call(n) for n in m["step"].kernel_names),
        "kernel_timing": "per-kernel CUDA events in a second pass of the same K steps (launched eagerly)",
        "in_step_timing": ("in_step_us: a round of replayed steps minus the same round captured without the call, "
                           "per call (CUDA events, median of 3); in_step_frac from it"),
        "launch": ("the K batches captured as one CUDA graph of the binding's calls on two lanes of buffers "
                   "(programmatic dependent launch within each stream), replayed once" if mp is not None
                   else m["launch_mode"]),
        "hot_l2": {
            "ms_per_step": round(hot_ms / args.steps, 4),
            "value": round(w.N * args.steps * ws / (hot_ms / 1e3), 1),
            "note": "the same K steps, one batch at a time, on one input set (inputs resident in L2); not the headline",
        },
        "clocks": sampler.summary(mp["timed_window"] if mp is not None else m["timed_window"]),
        "e2e": e2e,
    }
    if m_serial is not None:  # the same batches one at a time through the fused dispatch call
        ms_ser = m_serial["elapsed_ms"] / args.steps
        result["serial"] = {
            "ms_per_step": round(ms_ser, 4),
            "value": round(w.N * args.steps * ws / (m_serial["elapsed_ms"] / 1e3), 1),
            "step": "+".join(dict.fromkeys(m_serial["step"].kernel_names)),
            "dispatch": "moe_dispatch (layout + permute fused)",
            "note": "one batch at a time, the step's latency; the headline overlaps two batches",
            "in_step_us": m_serial.get("in_step_us", {}),
        }
        result["serial_unfused_ms_per_step"] = round(m["elapsed_ms"] / args.steps, 4)
    if workloads:
        result["workloads"] = workloads
    if not args.no_cpu_baseline and ws == 1:
        result["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    return result


def measure_e2e(w, host, step, args, ws, ctx):
    """The headline metric end to end through the binding, host copies inside the timed region."""
    torch, moe, _native, device, barrier = ctx["torch"], ctx["moe"], ctx["native"], ctx["device"], ctx["barrier"]
    pin = {key: torch.from_numpy(v if v.dtype != np.uint16 else v.view(np.int16)).pin_memory()
           for key, v in host.items()}
    depth = E2E_DEPTH
    outs_host = [torch.empty((w.N, w.H), dtype=torch.int16).pin_memory() for _ in range(depth)]
    h2d_s = torch.cuda.Stream(device)
    d2h_s = torch.cuda.Stream(device)
    comp_s = torch.cuda.Stream(device)
    pipes = []
    with torch.cuda.stream(comp_s):
        for b in range(depth):
            dset = {key: torch.empty_like(step.sets[0][key]) for key in pin}
            pipes.append(EpStep(w, moe, _native, torch, [dset], device) if w.ep else
                         Step(w, moe, _native, torch, [dset], device, unfused=ctx.get("unfused", False),
                              bulk_copy=ctx.get("bulk_copy", False)))
    views = [{key: (q.sets[0][key].view(torch.int16) if q.sets[0][key].dtype == torch.bfloat16
                    else q.sets[0][key]) for key in pin} for q in pipes]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done, comp_done, out_done = ([ev() for _ in range(depth)] for _ in range(3))
    started = [False] * depth

    def e2e_step(i):
        b = i % depth
        if started[b]:
            h2d_s.wait_event(comp_done[b])  # the kernels of step i-depth finished reading these inputs
        with torch.cuda.stream(h2d_s):
            for key in pin:
                views[b][key].copy_(pin[key], non_blocking=True)
        in_done[b].record(h2d_s)
        comp_s.wait_event(in_done[b])
        if started[b]:
            comp_s.wait_event(out_done[b])  # step i-depth's output has left the device
        pipes[b].run(0)
        comp_done[b].record(comp_s)
        d2h_s.wait_event(comp_done[b])
        with torch.cuda.stream(d2h_s):
            outs_host[b].copy_(pipes[b].out.view(torch.int16), non_blocking=True)
        out_done[b].record(d2h_s)
        started[b] = True

    for i in range(max(2, min(args.warmup, 4))):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(h2d_s)
    comp_s.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    for b in range(depth):  # the timed region ends when the last output is on the host
        d2h_s.wait_event(out_done[b])
    e1.record(d2h_s)
    torch.cuda.synchronize()
    barrier()
    e_ms = max_over_ranks(e0.elapsed_time(e1), device)
    st = 0
    for q in pipes:
        st |= q.status()
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after the end-to-end steps")
    return {
        "value": round(w.N * args.steps * ws / (e_ms / 1e3), 1),
        "unit": "tokens/s",
        "h2d_bytes_per_step": h2d,
        "d2h_bytes_per_step": d2h,
        "ms_per_step": round(e_ms / args.steps, 4),
        "pipelining": f"{depth} device buffer sets; copy-in, kernels and copy-out on three streams",
    }


# --------------------------------------------------------- CPU (oracle) arm


def oracle_step(oracle, w, d):
    """The whole path on the CPU oracle for the batch in ``d``."""
    idx, probs = oracle.route_topk(d["logits"], w.k)
    T = max(w.tp_size, 1)
    layouts, sends = [], []
    for r in range(T):
        L = oracle.layout(idx, probs, E_log=w.E_log, R=w.R, C=w.capacity, num_replicas=w.num_replicas,
                          align=w.row_align, tp_size=w.tp_size, tp_rank=r, local_topk=True)
        layouts.append(L)
        sends.append(oracle.permute(d["hidden"], L["dest_row"], L["rows_max"]))
    L, send = layouts[0], sends[0]
    if T == 1 and w.dedup:
        D = oracle.dedup_layout(L, probs, E_log=w.E_log, R=w.R, num_replicas=w.num_replicas)
        oracle.permute(d["hidden"], D["token_rank_row"], D["recv_max"])
        partial = oracle.dedup_combine_local(send, L, D, probs, w.R)
        out = oracle.combine(partial, D["token_rank_row"], None)
    elif T == 1:
        out = oracle.combine(send, L["dest_row"], probs)
    else:
        out = oracle.restore_combined(sends, [x["dest_row"] for x in layouts], probs)
    if w.backward:
        gy, gp = oracle.combine_backward(d["grad_out"], send, L["dest_row"], L["row_token"], L["row_prob"])
        oracle.permute_backward(gy, L["dest_row"])
    return out


def sample_workload(w, target_s, oracle):
    """A token sample of the workload sized to take about ``target_s`` per oracle step."""
    n = max(16, min(w.N, 64))
    ws = w.scaled(n)
    d = make_inputs(ws, grad=w.backward)
    t = time.perf_counter()
    oracle_step(oracle, ws, d)
    dt = max(time.perf_counter() - t, 1e-4)
    n = int(max(16, min(w.N, n * target_s / dt)))
    ws = w.scaled(n)
    return ws, make_inputs(ws, grad=w.backward)


def oracle_step_all_cores(oracle, w, d):
    """The path on every host core: route, permute and combine split over tokens with OpenMP
    (the unchanged oracle functions on each chunk), the layout serial as defined."""
    idx, probs = oracle.omp_route_topk(d["logits"], w.k)
    L = oracle.layout(idx, probs, E_log=w.E_log, R=w.R, C=w.capacity, num_replicas=w.num_replicas,
                      align=w.row_align, local_topk=True)
    send = oracle.omp_permute(d["hidden"], L["dest_row"], L["rows_max"])
    return oracle.omp_combine(send, L["dest_row"], probs)


def _timed_median(fn, budget_s):
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 3:
        t = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t)
    return statistics.median(times), len(times)


def cpu_baseline(w, budget_s=10.0):
    """The oracle timed on this host: single-threaded as it stands (the headline baseline), and the
    all-cores variant (OpenMP over tokens for route, permute and combine; the layout serial)."""
    import oracle

    oracle.build()
    ws, d = sample_workload(w, min(2.0, budget_s / 5), oracle)
    med, runs = _timed_median(lambda: oracle_step(oracle, ws, d), budget_s)
    out = {
        "value": round(ws.N / med, 1),
        "unit": "tokens/s",
        "cores": 1,
        "kind": "oracle",
        "sample": f"first {ws.N} of {w.N} tokens of '{w.name}' (same H/E/k/R), whole path per run, "
                  f"median of {runs} runs, single-threaded C oracle",
        "host_cpus": os.cpu_count(),
    }
    if not w.tp_size > 1 and not w.dedup and not w.ep and not w.backward:
        try:
            oracle.build_omp()
            threads = oracle.omp_threads()
            wa = w if w.N <= 4 * ws.N * threads else w.scaled(min(w.N, 4 * ws.N * threads))
            da = d if wa.N == ws.N else make_inputs(wa)
            med_a, runs_a = _timed_median(lambda: oracle_step_all_cores(oracle, wa, da), budget_s / 2)
            out["all_cores"] = {
                "value": round(wa.N / med_a, 1),
                "unit": "tokens/s",
                "cores": threads,
                "kind": "oracle, OpenMP over tokens (route, permute, combine); layout serial",
                "sample": f"first {wa.N} of {w.N} tokens of '{w.name}', whole path per run, median of {runs_a} runs",
            }
        except Exception as exc:  # no OpenMP toolchain on this host: the single-threaded figure stands
            out["all_cores"] = {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}
    return out


def run_reference(args, ws, rank):
    if rank != 0:
        return None
    import oracle

    oracle.build()
    w = get_workload(args.workload)
    per_step = max(0.02, min(1.0, 120.0 / max(1, args.steps + args.warmup)))
    wsamp, d = sample_workload(w, per_step, oracle)
    for _ in range(args.warmup):
        oracle_step(oracle, wsamp, d)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(oracle, wsamp, d)
    dt = time.perf_counter() - t
    value = wsamp.N * args.steps / dt
    sample = (f"first {wsamp.N} of {w.N} tokens of '{w.name}' per step (same H/E/k/R), "
              f"single-threaded C oracle")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {**w.describe(), "parallelism": "host cores of rank 0"},
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_calibration(args) -> dict:
    """Device copy and fill bandwidth at the permute's write size (L2 evicted before each run)."""
    import torch

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    nbytes = 470 * 2**20
    a = torch.empty(nbytes // 2, dtype=torch.int16, device=dev)
    b = torch.empty(nbytes // 4, dtype=torch.int16, device=dev)
    flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn, reps=10):
        ms = []
        for r in range(reps + 2):
            flush.fill_(r & 0xFF)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if r >= 2:
                ms.append(e0.elapsed_time(e1))
        return statistics.mean(ms)

    half = a[: nbytes // 4]
    copy_ms = timed(lambda: b.copy_(half))  # device-to-device copy: 235 MB read + 235 MB written
    fill_ms = timed(lambda: a.zero_())  # 470 MB written by torch's fill kernel
    # the capacity workload's send buffer (40,960 rows of 4 KB): a short write-only stream
    cap_bytes = 40960 * 4096
    cap = a[: cap_bytes // 2]
    fill_cap_ms = timed(lambda: cap.zero_())
    # host links at the end-to-end step's sizes (ht: 62.9 MB in, 58.7 MB out), pinned host memory
    h_in = torch.empty(62914560 // 2, dtype=torch.int16).pin_memory()
    h_out = torch.empty(58720256 // 2, dtype=torch.int16).pin_memory()
    d_in = torch.empty_like(h_in, device=dev)
    d_out = torch.empty_like(h_out, device=dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def both():
        cur = torch.cuda.current_stream()
        s_in.wait_stream(cur)  # both copies start after the start event
        s_out.wait_stream(cur)
        with torch.cuda.stream(s_in):
            d_in.copy_(h_in, non_blocking=True)
        with torch.cuda.stream(s_out):
            h_out.copy_(d_out, non_blocking=True)
        torch.cuda.current_stream().wait_stream(s_in)
        torch.cuda.current_stream().wait_stream(s_out)

    h2d_ms = timed(lambda: d_in.copy_(h_in, non_blocking=True))
    d2h_ms = timed(lambda: h_out.copy_(d_out, non_blocking=True))
    both_ms = timed(both)
    return {
        "calibration": "device bandwidth at the permute's size; host links at the e2e step's sizes",
        "copy_d2d_gbs": round(nbytes / (copy_ms * 1e-3) / 1e9, 1),
        "torch_zero_gbs": round(nbytes / (fill_ms * 1e-3) / 1e9, 1),
        "bytes": nbytes,
        "torch_zero_capacity_send_gbs": round(cap_bytes / (fill_cap_ms * 1e-3) / 1e9, 1),
        "capacity_send_bytes": cap_bytes,
        "h2d_gbs": round(h_in.numel() * 2 / (h2d_ms * 1e-3) / 1e9, 1),
        "d2h_gbs": round(h_out.numel() * 2 / (d2h_ms * 1e-3) / 1e9, 1),
        "h2d_d2h_together_ms": round(both_ms, 3),
        "measured_peak_hbm_gbs": measured_peaks()[0],
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=None,
                    help="tiny | ht | qwen3 | capacity | ultraep | ht_align16 | ht_tp2 | ht_dedup | ht_ep4 "
                         "(default: ht as the headline, with tiny, qwen3, capacity and ultraep timed beside it)")
    ap.add_argument("--unfused", action="store_true",
                    help="call moe_dispatch_layout and moe_permute separately instead of the fused moe_dispatch")
    ap.add_argument("--bulk-copy", action="store_true",
                    help="stage the dispatch's rows through shared memory with bulk (TMA) copies "
                         "(MOE_FLAG_DISPATCH_BULK_COPY) instead of 16-byte vector copies")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the headline workload (skip the other surveyed configurations)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--schedule", default="pipelined", choices=["pipelined", "serial"],
                    help="headline schedule: two batches in flight (default, for workloads whose step is route, "
                         "layout, permute, combine on one rank) or one batch at a time")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=0, help="run the workload with this many tokens (profiling)")
    ap.add_argument("--eager", action="store_true",
                    help="time eager C-ABI calls instead of replaying one captured CUDA graph per buffer set")
    ap.add_argument("--calibrate", action="store_true",
                    help="print the device's copy and fill bandwidth at the permute's size, then exit")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    args.workload_given = args.workload is not None
    if args.workload is None:
        args.workload = "ht"
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws, rank, local = dist_env()
    if args.gpus != ws and ws > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={ws}")
    if args.calibrate:
        res = run_calibration(args) if rank == 0 else None
    elif args.impl == "reference":
        res = run_reference(args, ws, rank)
    else:
        res = run_ours(args, ws, rank, local)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
