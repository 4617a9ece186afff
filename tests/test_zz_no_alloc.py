"""The layout entry point that allocates nothing (moe_dispatch_layout_noalloc).

It serves callers that cannot allocate device memory: the layout's scratch
lives in a fixed array inside the library instead of a workspace the caller
passes. Its results must equal those of moe_dispatch_layout, bit for bit, on
consecutive calls that share that array. This file is collected last so that
a failure here stops a -x run only after every other test has run.
"""

import ctypes

import numpy as np
import pytest
import torch

import combine_moe_route_tokens_b200 as moe
from combine_moe_route_tokens_b200 import _native

from gpu_util import dev, host, require_cuda

pytestmark = pytest.mark.gpu

KEYS = ["phys_idx", "ordinal", "dest_row", "drop_mask", "counts_logical", "placement", "counts_raw",
        "tokens_per_expert", "expert_offsets", "input_splits", "output_splits", "rank_offsets", "counters",
        "num_rows", "row_token", "row_slot", "row_local_expert", "row_prob", "pad_mask", "local_topk"]


def _inputs(N, k, E_log, seed, zipf=1.3, neg=0.05):
    rng = np.random.default_rng(seed)
    idx = (rng.zipf(zipf, size=(N, k)) % E_log).astype(np.int32)
    idx[rng.random((N, k)) < neg] = -1
    probs = rng.random((N, k)).astype(np.float32)
    return dev(idx), dev(probs)


def _noalloc_c_call(p, idx, probs, layout):
    """Call the entry point through the C ABI directly."""
    lib = _native.lib()
    P = p.c_struct()
    L = layout.c_struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.moe_dispatch_layout_noalloc(ctypes.byref(P), ctypes.c_void_p(idx.data_ptr()),
                                           ctypes.c_void_p(probs.data_ptr()), ctypes.byref(L), stream)


def _assert_same(a, b):
    for key in KEYS:
        x, y = host(a[key]), host(b[key])
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), key


CASES = [
    # N, H, k, E_log, R, capacity, replicas
    (4096, 8, 8, 256, 4, 0, 0),      # the 4096-token / e256 / top-8 shape
    (5000, 8, 2, 64, 2, 200, 0),     # capacity: drops and pad rows
    (2049, 8, 8, 512, 8, 0, 8),      # widest router the fixed scratch holds, with replicas
]


@pytest.mark.parametrize("case", CASES, ids=[f"N{c[0]}_k{c[2]}_E{c[3]}" for c in CASES])
def test_noalloc_matches_allocating_layout_on_consecutive_calls(case):
    require_cuda()
    N, H, k, E_log, R, C, reps = case
    p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps)
    for call in range(2):  # two calls in a row share the library's scratch
        idx, probs = _inputs(N, k, E_log, seed=17 * call + N)
        ref = moe.moe_dispatch_layout(p, idx, probs)
        got = moe.Layout.allocate(p)
        assert _noalloc_c_call(p, idx, probs, got) == 0
        torch.cuda.synchronize()
        _assert_same(got, ref)
        assert got.status() == 0


def test_noalloc_recovers_after_a_timed_out_call():
    """A call whose look-back ran out leaves nothing in the shared scratch that the next call must clear."""
    require_cuda()
    idx, probs = _inputs(3000, 4, 32, seed=5)
    bad = moe.Problem(N=3000, H=8, k=4, E_log=32, R=4, flags=moe.MOE_FLAG_TEST_WAIT_TIMEOUT)
    lay = moe.Layout.allocate(bad)
    assert _noalloc_c_call(bad, idx, probs, lay) == 0
    torch.cuda.synchronize()
    assert lay.status() & moe.MOE_DEV_TIMEOUT
    good = moe.Problem(N=3000, H=8, k=4, E_log=32, R=4)
    got = moe.Layout.allocate(good)
    moe.moe_dispatch_layout_noalloc(good, idx, probs, got)
    ref = moe.moe_dispatch_layout(good, idx, probs)
    torch.cuda.synchronize()
    _assert_same(got, ref)
    assert got.status() == 0


def test_noalloc_rejects_routers_wider_than_its_scratch():
    require_cuda()
    p = moe.Problem(N=16, H=8, k=2, E_log=_native.MOE_NOALLOC_MAX_E_LOG * 2, R=1)
    idx, probs = _inputs(16, 2, p.E_log, seed=1)
    lay = moe.Layout.allocate(p)
    assert _noalloc_c_call(p, idx, probs, lay) == _native.MOE_ERR_SCRATCH_LIMIT
    assert "scratch" in _native.status_string(_native.MOE_ERR_SCRATCH_LIMIT)
