"""Helpers shared by the GPU tests: numpy <-> device copies and the tolerance
of the router probabilities. Inputs always come from ``synthetic`` or from
the oracle, never from the CUDA path."""

from __future__ import annotations

import numpy as np
import pytest
import torch


def require_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(a).cuda()
    return t if dtype is None else t.to(dtype)


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy; bf16 comes back as uint16 bit patterns."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def route_prob_tolerance(logits: np.ndarray, topk_idx: np.ndarray) -> np.ndarray:
    """Per-entry absolute bound on |p_gpu - p_exact| for the router probs.

    The GPU evaluates x = fl(l - m) (relative error u), expf(x) (at most 2 ulp
    by the CUDA documentation), a fp32 sum of E such terms (per-lane chain of at
    most E/32 terms plus a 5-level butterfly) and one rounded division. To first
    order the relative error of p is at most
        (|x_e| + 2) u  +  max_e' (|x_e'| + 2) u  +  (E/32 + 5) u  +  u,
    u = 2^-24; the exact value itself is rounded once by the oracle (u more).
    The bound below doubles that for second-order terms.
    """
    l = logits.astype(np.float64)
    m = l.max(axis=1, keepdims=True)
    x = m - l
    xmax = x.max(axis=1, keepdims=True)
    E = logits.shape[1]
    xe = np.take_along_axis(x, np.maximum(topk_idx, 0).astype(np.int64), axis=1)
    rel = (xe + 2) + (xmax + 2) + (np.ceil(E / 32) + 5) + 2
    return 2.0 * rel * 2.0 ** -24
