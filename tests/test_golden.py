"""The hand-worked fixtures of tests/golden against the oracle (CPU) and the CUDA path (GPU).

Each fixture cites the page and the reading it follows and shows its derivation; the
expected values come from neither implementation.
"""

import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
LAYOUT_FIXTURES = ["layout_rank_major_3tok.json", "reroute_placement_2rank.json", "reroute_least_loaded_4rank.json",
                   "reroute_load_moves_3rank.json"]
COMBINE_FIXTURES = ["combine_slot_order.json", "combine_fused_multiply_add.json"]
PERMUTE_BACKWARD_FIXTURES = ["permute_backward_slot_order.json"]


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        fx = json.load(f)
    assert fx["source"] and fx["derivation"]
    return fx


@pytest.mark.parametrize("name", LAYOUT_FIXTURES)
def test_oracle_layout_matches_hand_worked(oracle_lib, name):
    fx = _load(name)
    inp = fx["inputs"]
    idx = np.asarray(inp["topk_idx"], np.int32)
    L = oracle_lib.layout(idx, None, E_log=inp["E_log"], R=inp["R"], num_replicas=inp.get("num_replicas", 0),
                          local_topk=True)
    for key, want in fx["expected"].items():
        assert np.array_equal(np.asarray(L[key]), np.asarray(want)), key


@pytest.mark.parametrize("name", COMBINE_FIXTURES)
def test_oracle_combine_matches_hand_worked(oracle_lib, name):
    fx = _load(name)
    inp = fx["inputs"]
    out = oracle_lib.combine(np.asarray(inp["expert_out"], np.uint16), np.asarray(inp["dest_row"], np.int32),
                             np.asarray(inp["topk_probs"], np.float32))
    assert np.array_equal(out, np.asarray(fx["expected"]["out"], np.uint16))


@pytest.mark.parametrize("name", PERMUTE_BACKWARD_FIXTURES)
def test_oracle_permute_backward_matches_hand_worked(oracle_lib, name):
    fx = _load(name)
    inp = fx["inputs"]
    gh = oracle_lib.permute_backward(np.asarray(inp["grad_send"], np.uint16), np.asarray(inp["dest_row"], np.int32))
    assert np.array_equal(gh, np.asarray(fx["expected"]["grad_hidden"], np.uint16))


@pytest.mark.gpu
@pytest.mark.parametrize("name", LAYOUT_FIXTURES)
def test_cuda_layout_matches_hand_worked(name):
    import torch

    import combine_moe_route_tokens_b200 as moe
    from gpu_util import dev, host, require_cuda

    require_cuda()
    fx = _load(name)
    inp = fx["inputs"]
    idx = np.asarray(inp["topk_idx"], np.int32)
    p = moe.Problem(N=idx.shape[0], H=8, k=idx.shape[1], E_log=inp["E_log"], R=inp["R"],
                    num_replicas=inp.get("num_replicas", 0))
    G = moe.moe_dispatch_layout(p, dev(idx), None)
    torch.cuda.synchronize()
    for key, want in fx["expected"].items():
        assert np.array_equal(host(G[key]).reshape(np.asarray(want).shape), np.asarray(want)), key
    assert G.status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("name", COMBINE_FIXTURES)
def test_cuda_combine_matches_hand_worked(name):
    import torch

    import combine_moe_route_tokens_b200 as moe
    from gpu_util import dev, host, require_cuda

    require_cuda()
    fx = _load(name)
    inp = fx["inputs"]
    dest = np.asarray(inp["dest_row"], np.int32)
    y = np.asarray(inp["expert_out"], np.uint16)
    N, k = dest.shape
    # a layout whose row map is the fixture's: one row per slot, in slot order
    p = moe.Problem(N=N, H=8, k=k, E_log=k, R=1)
    G = moe.moe_dispatch_layout(p, dev(np.arange(N * k, dtype=np.int32).reshape(N, k) % k), None)
    torch.cuda.synchronize()
    assert np.array_equal(host(G["dest_row"]), dest)
    y8 = np.repeat(y, 8, axis=1)  # rows of 8 bf16 (16 bytes), every column the fixture's value
    out = moe.moe_combine(p, G, dev(y8), dev(np.asarray(inp["topk_probs"], np.float32)))
    torch.cuda.synchronize()
    assert np.array_equal(host(out), np.repeat(np.asarray(fx["expected"]["out"], np.uint16), 8, axis=1))


@pytest.mark.gpu
@pytest.mark.parametrize("name", PERMUTE_BACKWARD_FIXTURES)
def test_cuda_permute_backward_matches_hand_worked(name):
    import torch

    import combine_moe_route_tokens_b200 as moe
    from gpu_util import dev, host, require_cuda

    require_cuda()
    fx = _load(name)
    inp = fx["inputs"]
    dest = np.asarray(inp["dest_row"], np.int32)
    g = np.asarray(inp["grad_send"], np.uint16)
    N, k = dest.shape
    p = moe.Problem(N=N, H=8, k=k, E_log=k, R=1)
    G = moe.moe_dispatch_layout(p, dev(np.arange(N * k, dtype=np.int32).reshape(N, k) % k), None)
    torch.cuda.synchronize()
    assert np.array_equal(host(G["dest_row"]), dest)
    gh = moe.moe_permute_backward(p, G, dev(np.repeat(g, 8, axis=1)))
    torch.cuda.synchronize()
    assert np.array_equal(host(gh), np.repeat(np.asarray(fx["expected"]["grad_hidden"], np.uint16), 8, axis=1))
