"""CPU oracle for MoE token dispatch / combine — TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. The product path never does, and this package
imports nothing from the product.
"""

from .oracle import (
    build,
    build_omp,
    omp_threads,
    omp_route_topk,
    omp_permute,
    omp_combine,
    library_path,
    rows_max,
    num_experts,
    route_topk,
    layout,
    permute,
    combine,
    restore_combined,
    ep_exchange,
    dedup_layout,
    dedup_combine_local,
    permute_backward,
    combine_backward,
    bf16_from_f32,
    COUNTER_NAMES,
)

__all__ = [
    "build",
    "build_omp",
    "omp_threads",
    "omp_route_topk",
    "omp_permute",
    "omp_combine",
    "library_path",
    "rows_max",
    "num_experts",
    "route_topk",
    "layout",
    "permute",
    "combine",
    "restore_combined",
    "ep_exchange",
    "dedup_layout",
    "dedup_combine_local",
    "permute_backward",
    "combine_backward",
    "bf16_from_f32",
    "COUNTER_NAMES",
]
