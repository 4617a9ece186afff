"""The workloads that parity tests and the benchmark run, with their input recipe.

Shapes follow the pages' problem statements:

* ``tiny``      — N=128, H=256, E=8, top-2, 2 simulated EP ranks, no capacity.
* ``ht``        — the DeepEP-style high-throughput shape measured on the mscclpp
                  page (e256 / top-8 / hidden 7168 / 4096 tokens), 4 ranks.
* ``qwen3``     — a Qwen3-235B-A22B-like layer: N=8192, H=4096, E=128, top-8,
                  8 ranks, Zipf(1.2)-skewed expert popularity.
* ``capacity``  — N=16384, H=2048, E=64, top-2, capacity factor 1.25,
                  Zipf(1.5) skew, 2 ranks; drop and pad masks in play.
* ``ultraep``   — N=8192, H=7168, 256 logical experts, top-8, 8 ranks, the 8
                  hottest experts get one replica slot each (264 physical), Zipf(1.2)
                  skew; forward and backward.
* ``ht_align16`` — the ``ht`` shape and inputs with every expert's rows padded up to
                  a multiple of 16 (grouped-GEMM / FP8 alignment).
* ``ht_tp2``    — the ``ht`` shape and inputs folded over 2 TP peers.
* ``ht_dedup``  — the ``ht`` shape and inputs through the DeepEP-style token-dedup path.

Recipe: logits are N(0,1) float32 plus, where a workload is skewed, a per-expert
bias ``-s ln(rank+1)`` over a seeded ranking of the experts; hidden states and
output gradients are N(0,1) rounded to bf16. The seed of workload number ``i``
(1-based, in the order above) is ``0x5EED0000 + i``.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from fractions import Fraction
from typing import Optional

import numpy as np

from .generator import bf16_bits_from_f32, splitmix64, standard_normal, zipf_bias, STREAM_SHIFT

TAG_LOGITS = 1
TAG_EXPERT_RANKING = 2
TAG_HIDDEN = 3
TAG_GRAD_OUT = 4
TAG_TOKEN_MASK = 5


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    H: int
    E_log: int
    k: int
    R: int
    capacity_factor: Optional[Fraction] = None
    zipf_s: Optional[float] = None
    num_replicas: int = 0
    backward: bool = False
    row_align: int = 0
    tp_size: int = 0
    dedup: bool = False
    ep: bool = False  # the N tokens are split evenly over the R ranks, which exchange rows
    seed: int = 0x5EED0000
    note: str = field(default="", compare=False)

    @property
    def E(self) -> int:
        """Physical experts: logical experts plus replica slots."""
        return self.E_log + self.num_replicas

    @property
    def capacity(self) -> int:
        """Per-expert capacity ceil(factor * N * k / E); 0 means unlimited."""
        if self.capacity_factor is None:
            return 0
        q = Fraction(self.capacity_factor) * self.N * self.k / self.E
        return -((-q.numerator) // q.denominator)

    def scaled(self, N: int, name: Optional[str] = None) -> "Workload":
        """The same workload with a different token count (for sampled runs)."""
        return Workload(
            name=name or f"{self.name}[N={N}]",
            N=N,
            H=self.H,
            E_log=self.E_log,
            k=self.k,
            R=self.R,
            capacity_factor=self.capacity_factor,
            zipf_s=self.zipf_s,
            num_replicas=self.num_replicas,
            backward=self.backward,
            row_align=self.row_align,
            tp_size=self.tp_size,
            dedup=self.dedup,
            ep=self.ep,
            seed=self.seed,
            note=self.note,
        )

    def describe(self) -> dict:
        d = {
            "workload": self.name,
            "N": self.N,
            "H": self.H,
            "E": self.E,
            "E_logical": self.E_log,
            "top_k": self.k,
            "ranks": self.R,
            "capacity": self.capacity,
        }
        if self.zipf_s is not None:
            d["zipf_s"] = self.zipf_s
        if self.num_replicas:
            d["replicas"] = self.num_replicas
        if self.backward:
            d["backward"] = True
        if self.row_align > 1:
            d["row_align"] = self.row_align
        if self.tp_size > 1:
            d["tp_size"] = self.tp_size
        if self.dedup:
            d["dedup"] = True
        if self.ep:
            d["ep_exchange"] = f"{self.R} ranks x {self.N // self.R} tokens, simulated on one GPU"
        return d


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", N=128, H=256, E_log=8, k=2, R=2, seed=0x5EED0001),
        Workload("ht", N=4096, H=7168, E_log=256, k=8, R=4, seed=0x5EED0002),
        Workload("qwen3", N=8192, H=4096, E_log=128, k=8, R=8, zipf_s=1.2, seed=0x5EED0003),
        Workload(
            "capacity",
            N=16384,
            H=2048,
            E_log=64,
            k=2,
            R=2,
            capacity_factor=Fraction(5, 4),
            zipf_s=1.5,
            seed=0x5EED0004,
        ),
        Workload(
            "ultraep",
            N=8192,
            H=7168,
            E_log=256,
            k=8,
            R=8,
            zipf_s=1.2,
            num_replicas=8,
            backward=True,
            seed=0x5EED0005,
        ),
        # the 4096-token / e256 / top-8 shape with every expert's rows padded to a
        # multiple of 16 (grouped-GEMM / FP8 alignment); not one of the five configs
        Workload("ht_align16", N=4096, H=7168, E_log=256, k=8, R=4, row_align=16, seed=0x5EED0002),
        # the same shape folded over 2 TP peers (each peer's layout and send buffer on
        # this GPU, then one restore over both)
        Workload("ht_tp2", N=4096, H=7168, E_log=256, k=8, R=4, tp_size=2, seed=0x5EED0002),
        # the same shape through the DeepEP-style path: each token sent once per rank,
        # receiver-side partials, sender-side sum over ranks
        Workload("ht_dedup", N=4096, H=7168, E_log=256, k=8, R=4, dedup=True, seed=0x5EED0002),
        # the same 4096 tokens held by 4 ranks (1024 each) that exchange rows: every
        # rank dispatches into the owners' receive buffers and combines from them
        Workload("ht_ep4", N=4096, H=7168, E_log=256, k=8, R=4, ep=True, seed=0x5EED0002),
    ]
}


def get_workload(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None


def make_logits(w: Workload, seed_offset: int = 0) -> np.ndarray:
    """Router logits [N, E_log] float32: N(0,1), plus the Zipf bias when the workload is skewed."""
    seed = w.seed + seed_offset
    z = standard_normal(seed, TAG_LOGITS, w.N * w.E_log).reshape(w.N, w.E_log)
    if w.zipf_s is not None:
        # The expert ranking is a property of the workload, not of a rank's shard.
        z = z + zipf_bias(w.seed, TAG_EXPERT_RANKING, w.E_log, w.zipf_s)[None, :]
    return z.astype(np.float32)


def make_bf16(w: Workload, tag: int, rows: int, seed_offset: int = 0) -> np.ndarray:
    """[rows, H] N(0,1) values rounded to bf16, as uint16 bit patterns."""
    z = standard_normal(w.seed + seed_offset, tag, rows * w.H).astype(np.float32)
    return bf16_bits_from_f32(z).reshape(rows, w.H)


def make_token_mask(w: Workload, fraction: float, seed_offset: int = 0) -> np.ndarray:
    """A padding-token mask [N] uint8 with about ``fraction`` of the tokens set."""
    u = splitmix64(w.seed + seed_offset, TAG_TOKEN_MASK << STREAM_SHIFT, w.N) >> np.uint64(11)
    return (u.astype(np.float64) * (1.0 / 9007199254740992.0) < fraction).astype(np.uint8)


def make_inputs(w: Workload, *, hidden: bool = True, grad: Optional[bool] = None, seed_offset: int = 0) -> dict:
    """All inputs of a workload as numpy arrays.

    Returns ``logits`` [N,E_log] f32, ``hidden`` [N,H] bf16 bits and, for
    backward workloads, ``grad_out`` [N,H] bf16 bits. ``seed_offset`` gives
    independent batches of the same workload (one per data-parallel rank).
    """
    out = {"logits": make_logits(w, seed_offset)}
    if hidden:
        out["hidden"] = make_bf16(w, TAG_HIDDEN, w.N, seed_offset)
    if grad is None:
        grad = w.backward
    if grad:
        out["grad_out"] = make_bf16(w, TAG_GRAD_OUT, w.N, seed_offset)
    return out
