"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bar: bit-exact for every integer, mask, row-map and copied output, for the
combine / permute-backward outputs (fixed fp32 fma order, one bf16 rounding)
and for grad_expert_out (one fp32 product, one rounding). Router probs and
grad_probs are within bounds derived from their fp32 arithmetic (router:
tests/gpu_util.py; grad_probs: the fp32 summation bound gamma_H * sum|g*y|).

All five workloads run at their full sizes, with the same launch
configuration the benchmark uses. Inputs come from ``synthetic``; the oracle
route output feeds both sides so that layout/combine parity never depends on
expf rounding.
"""

import dataclasses

import numpy as np
import pytest
import torch

import combine_moe_route_tokens_b200 as moe
import oracle
from synthetic import bf16_bits_from_f32, get_workload, make_inputs
from synthetic.workloads import make_token_mask

from gpu_util import dev, host, require_cuda, route_prob_tolerance

pytestmark = pytest.mark.gpu

WORKLOAD_NAMES = ["tiny", "ht", "qwen3", "capacity", "ultraep", "ht_align16"]
LAYOUT_KEYS = [
    "phys_idx", "ordinal", "dest_row", "drop_mask", "counts_logical", "placement", "counts_raw",
    "tokens_per_expert", "expert_offsets", "input_splits", "output_splits", "rank_offsets", "counters",
    "num_rows", "row_token", "row_slot", "row_local_expert", "row_prob", "pad_mask", "local_topk",
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    require_cuda()
    moe.load_library()


_cache = {}


def workload_case(name):
    """Inputs and the oracle's route + layout for a workload (cached per module)."""
    if name not in _cache:
        w = get_workload(name)
        d = make_inputs(w, grad=True)
        idx, probs = oracle.route_topk(d["logits"], w.k)
        L = oracle.layout(idx, probs, E_log=w.E_log, R=w.R, C=w.capacity, num_replicas=w.num_replicas,
                          align=w.row_align)
        _cache.clear()
        _cache[name] = (w, d, idx, probs, L)
    return _cache[name]


def problem_of(w, N=None):
    return moe.Problem(N=w.N if N is None else N, H=w.H, k=w.k, E_log=w.E_log, R=w.R, capacity=w.capacity,
                       num_replicas=w.num_replicas, row_align=w.row_align)


def assert_layout_equal(G, L):
    for key in LAYOUT_KEYS:
        got = host(G[key]).reshape(-1)
        exp = np.asarray(L[key]).reshape(-1)
        if key == "row_prob":
            assert np.array_equal(got.view(np.uint32), exp.astype(np.float32).view(np.uint32)), key
        else:
            assert np.array_equal(got.astype(np.int64), exp.astype(np.int64)), key


def check_dispatch(p, idx, probs, hidden, L):
    """The fused dispatch (layout + permute in one call): its layout and its send buffer,
    written over a canary, equal the oracle's, bit for bit."""
    canary = torch.tensor(0x7F7F, dtype=torch.int16).view(torch.bfloat16).item()
    send = torch.full((L["rows_max"], p.H), canary, dtype=torch.bfloat16, device="cuda")
    G, send = moe.moe_dispatch(p, dev(idx), None if probs is None else dev(probs), dev(hidden), send=send)
    torch.cuda.synchronize()
    assert_layout_equal(G, L)
    assert np.array_equal(host(send), oracle.permute(hidden, L["dest_row"], L["rows_max"]))
    assert G.status() == 0
    return G, send


@pytest.mark.parametrize("name", WORKLOAD_NAMES)
def test_dispatch_fused(name):
    w, d, idx, probs, L = workload_case(name)
    check_dispatch(problem_of(w), idx, probs, d["hidden"], L)
    # the same call with the rows staged through shared memory by bulk copies
    check_dispatch(dataclasses.replace(problem_of(w), flags=moe.MOE_FLAG_DISPATCH_BULK_COPY), idx, probs,
                   d["hidden"], L)


@pytest.mark.parametrize("name", WORKLOAD_NAMES)
def test_route(name):
    w, d, idx, probs, _ = workload_case(name)
    gi, gp = moe.moe_route_topk(dev(d["logits"]), w.k)
    torch.cuda.synchronize()
    assert np.array_equal(host(gi), idx)
    tol = route_prob_tolerance(d["logits"], idx) * probs.astype(np.float64)
    assert np.all(np.abs(host(gp).astype(np.float64) - probs.astype(np.float64)) <= tol)


@pytest.mark.parametrize("name", WORKLOAD_NAMES)
def test_layout(name):
    w, d, idx, probs, L = workload_case(name)
    G = moe.moe_dispatch_layout(problem_of(w), dev(idx), dev(probs))
    torch.cuda.synchronize()
    assert_layout_equal(G, L)
    assert G.status() == 0


@pytest.mark.parametrize("name", WORKLOAD_NAMES)
def test_permute_combine(name):
    w, d, idx, probs, L = workload_case(name)
    p = problem_of(w)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    send = moe.moe_permute(p, G, dev(d["hidden"]))
    send_h = host(send)
    exp_send = oracle.permute(d["hidden"], L["dest_row"], L["rows_max"])
    assert np.array_equal(send_h, exp_send)
    # identity experts: y = send
    out = moe.moe_combine(p, G, send, dev(probs))
    assert np.array_equal(host(out), oracle.combine(exp_send, L["dest_row"], probs))
    out1 = moe.moe_combine(p, G, send, None)
    assert np.array_equal(host(out1), oracle.combine(exp_send, L["dest_row"], None))
    assert G.status() == 0


def test_combine_special_values():
    """NaN, +-inf and signed zeros in the expert outputs: every non-NaN output is bit-exact; a NaN
    output is NaN on both sides at the same places (the GPU's is the canonical bf16 NaN, the CPU
    definition keeps sign and payload: the one documented exception to bit-exactness)."""
    N, H, k, E_log, R = 300, 64, 4, 16, 2
    idx, probs, hidden = _small_case(N, H, k, E_log, R, seed=21)
    L = oracle.layout(idx, probs, E_log=E_log, R=R)
    y = oracle.permute(hidden, L["dest_row"], L["rows_max"])
    rng = np.random.default_rng(21)
    specials = np.array([0x7FC0, 0xFFC1, 0x7F81, 0x7F80, 0xFF80, 0x8000, 0x0000], np.uint16)  # NaNs, +-inf, -0, +0
    mask = rng.random(y.shape) < 0.02
    y[mask] = specials[rng.integers(0, len(specials), mask.sum())]
    p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    for pr in (probs, None):
        got = host(moe.moe_combine(p, G, dev(y), None if pr is None else dev(pr)))
        want = oracle.combine(y, L["dest_row"], pr)
        nan_g = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
        nan_w = ((want & 0x7F80) == 0x7F80) & ((want & 0x7F) != 0)
        assert nan_g.any() and np.array_equal(nan_g, nan_w)
        assert np.array_equal(got[~nan_g], want[~nan_w])
        assert ((want & 0x7F80) == 0x7F80)[~nan_w].any()  # infinities reached the output too


@pytest.mark.parametrize("name", WORKLOAD_NAMES)
def test_backward(name):
    w, d, idx, probs, L = workload_case(name)
    p = problem_of(w)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    y = oracle.permute(d["hidden"], L["dest_row"], L["rows_max"])  # identity-expert outputs
    gy, gp = moe.moe_combine_backward(p, G, dev(d["grad_out"]), dev(y), dev(probs))
    exp_gy, exp_gp = oracle.combine_backward(d["grad_out"], y, L["dest_row"], L["row_token"], L["row_prob"])
    assert np.array_equal(host(gy), exp_gy)
    # grad_probs: fp32 accumulation in some fixed order vs the oracle's double sum
    gf = d["grad_out"].astype(np.uint32) << 16
    g = gf.view(np.float32).astype(np.float64)
    yf = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    dest = L["dest_row"]
    S = np.zeros_like(exp_gp, dtype=np.float64)
    for j in range(w.k):
        rows = np.maximum(dest[:, j], 0)
        S[:, j] = np.einsum("nh,nh->n", np.abs(g), np.abs(yf[rows]))
    u = 2.0 ** -24
    gamma = w.H * u / (1 - w.H * u)
    got = host(gp).astype(np.float64)
    assert np.all(np.abs(got - exp_gp.astype(np.float64)) <= gamma * S + 2 * u * np.abs(exp_gp) + 1e-30)
    assert np.all(got[dest < 0] == 0)
    # permute backward = unit-weight combine of grad_send (here: the grads just produced)
    gh = moe.moe_permute_backward(p, G, gy)
    assert np.array_equal(host(gh), oracle.permute_backward(exp_gy, L["dest_row"]))
    assert G.status() == 0


def test_layout_is_deterministic_and_reusable():
    w, d, idx, probs, L = workload_case("qwen3")
    p = problem_of(w)
    G = moe.Layout.allocate(p)
    for _ in range(3):  # the workspace's barrier state is left ready for the next call
        moe.moe_dispatch_layout(p, dev(idx), dev(probs), layout=G)
        torch.cuda.synchronize()
        assert_layout_equal(G, L)


# ---------------------------------------------------------------- edge cases


def _small_case(N, H, k, E_log, R, C=0, reps=0, neg=0.0, seed=0, zipf=None, bad=0):
    rng = np.random.default_rng(seed)
    if zipf:
        idx = (rng.zipf(zipf, size=(N, k)) % E_log).astype(np.int32)
    else:
        idx = rng.integers(0, E_log, size=(N, k)).astype(np.int32)
    if neg:
        idx[rng.random((N, k)) < neg] = -1
    if bad:
        flat = idx.reshape(-1)
        pos = rng.choice(flat.size, size=min(bad, flat.size), replace=False)
        flat[pos] = np.where(rng.random(len(pos)) < 0.5, E_log + 3, -7)
    probs = rng.random((N, k)).astype(np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    return idx, probs, hidden


EDGE_CASES = [
    # N, H, k, E_log, R, C, reps, neg, zipf
    (1, 8, 1, 1, 1, 0, 0, 0.0, None),
    (3, 24, 3, 5, 1, 0, 0, 0.0, None),  # generic-k kernels, ragged row (3 x 16 B)
    (37, 264, 6, 12, 3, 0, 0, 0.2, None),
    (1000, 1032, 12, 40, 4, 0, 0, 0.1, 1.3),  # k beyond the specialised set
    (5000, 520, 2, 64, 4, 90, 0, 0.05, 1.5),  # capacity with drops and pads
    (4099, 136, 8, 128, 8, 0, 8, 0.0, 1.2),  # reroute, ragged block tail
    (2048, 64, 4, 32, 2, 40, 4, 0.1, 1.4),  # reroute + capacity
    (777, 16, 8, 2048, 1, 0, 0, 0.0, None),  # widest router supported
    (300, 20000, 2, 8, 2, 0, 0, 0.0, None),  # row of 40000 B: three 16 KB pieces, the last ragged
    (70000, 8, 1, 4, 2, 0, 0, 0.0, None),  # many blocks, tiny rows
    (36000, 8, 8, 256, 8, 0, 8, 0.0, 1.2),  # 288k assignments: 8 per lane in registers, reroute
    (75000, 8, 8, 64, 4, 0, 0, 0.05, 1.2),  # 600k assignments: slices too long for registers
]
ALIGN_CASES = [
    # N, H, k, E_log, R, C, reps, neg, zipf, align
    (1000, 72, 4, 24, 4, 0, 0, 0.05, 1.4, 16),
    (3000, 40, 2, 16, 2, 256, 0, 0.1, 1.5, 128),  # capacity and alignment
    (2049, 24, 8, 64, 8, 0, 8, 0.0, 1.2, 8),  # reroute and alignment
    (5, 8, 2, 4, 2, 0, 0, 0.0, None, 1000),  # alignment far above the counts
]


@pytest.mark.parametrize("case", EDGE_CASES + ALIGN_CASES,
                         ids=[f"N{c[0]}_H{c[1]}_k{c[2]}_E{c[3]}" + (f"_A{c[9]}" if len(c) > 9 else "")
                              for c in EDGE_CASES + ALIGN_CASES])
def test_edge_cases_full_path(case):
    N, H, k, E_log, R, C, reps, neg, zipf = case[:9]
    A = case[9] if len(case) > 9 else 0
    idx, probs, hidden = _small_case(N, H, k, E_log, R, C, reps, neg, seed=N, zipf=zipf)
    L = oracle.layout(idx, probs, E_log=E_log, R=R, C=C, num_replicas=reps, align=A)
    p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps, row_align=A)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    torch.cuda.synchronize()
    assert_layout_equal(G, L)
    send = moe.moe_permute(p, G, dev(hidden))
    exp_send = oracle.permute(hidden, L["dest_row"], L["rows_max"])
    assert np.array_equal(host(send), exp_send)
    assert np.array_equal(host(moe.moe_combine(p, G, send, dev(probs))),
                          oracle.combine(exp_send, L["dest_row"], probs))
    rng = np.random.default_rng(1)
    g = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    gy, gp = moe.moe_combine_backward(p, G, dev(g), send, dev(probs))
    exp_gy, exp_gp = oracle.combine_backward(g, exp_send, L["dest_row"], L["row_token"], L["row_prob"])
    assert np.array_equal(host(gy), exp_gy)
    assert np.allclose(host(gp), exp_gp, rtol=1e-4, atol=1e-4 * np.sqrt(H))
    assert np.array_equal(host(moe.moe_permute_backward(p, G, gy)), oracle.permute_backward(exp_gy, L["dest_row"]))
    assert G.status() == 0
    check_dispatch(p, idx, probs, hidden, L)
    check_dispatch(dataclasses.replace(p, flags=moe.MOE_FLAG_DISPATCH_BULK_COPY), idx, probs, hidden, L)


@pytest.mark.parametrize("C", [0, 5])
def test_empty_batch(C):
    p = moe.Problem(N=0, H=16, k=2, E_log=4, R=2, capacity=C)
    idx = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    G = moe.moe_dispatch_layout(p, idx, None)
    send = moe.moe_permute(p, G, torch.zeros((0, 16), dtype=torch.bfloat16, device="cuda"))
    out = moe.moe_combine(p, G, send, None)
    torch.cuda.synchronize()
    L = oracle.layout(np.zeros((0, 2), np.int32), None, E_log=4, R=2, C=C)
    assert_layout_equal(G, L)
    assert out.shape == (0, 16) and send.shape == (L["rows_max"], 16)
    assert torch.all(send == 0)
    check_dispatch(p, np.zeros((0, 2), np.int32), None, np.zeros((0, 16), np.uint16), L)


def test_padding_tokens_via_route_mask():
    w = dataclasses.replace(get_workload("tiny"), N=300)
    d = make_inputs(w)
    mask = make_token_mask(w, 0.3)
    gi, gp = moe.moe_route_topk(dev(d["logits"]), w.k, token_mask=dev(mask))
    idx, probs = oracle.route_topk(d["logits"], w.k, token_mask=mask)
    torch.cuda.synchronize()
    assert np.array_equal(host(gi), idx)
    assert np.all(host(gp)[mask == 1] == 0)
    p = problem_of(w)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    L = oracle.layout(idx, probs, E_log=w.E_log, R=w.R)
    torch.cuda.synchronize()
    assert_layout_equal(G, L)
    assert int(host(G["num_rows"])[0]) < w.N * w.k  # a tail of pad rows
    send = moe.moe_permute(p, G, dev(d["hidden"]))
    assert np.array_equal(host(send), oracle.permute(d["hidden"], L["dest_row"], L["rows_max"]))


def test_out_of_range_ids_flagged_and_skipped():
    idx, probs, hidden = _small_case(500, 64, 4, 16, 4, bad=37, seed=3)
    p = moe.Problem(N=500, H=64, k=4, E_log=16, R=4)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    L = oracle.layout(idx, probs, E_log=16, R=4)
    torch.cuda.synchronize()
    assert L["counters"][7] == 1
    assert G.status() == moe.MOE_DEV_EXPERT_RANGE
    got = host(G["counters"])
    assert got[7] == moe.MOE_DEV_EXPERT_RANGE
    L["counters"][7] = moe.MOE_DEV_EXPERT_RANGE  # the device reports the bit, the oracle a flag
    assert_layout_equal(G, L)


def test_outputs_stay_inside_their_buffers():
    """Canary rows after every row-indexed output must be untouched."""
    idx, probs, hidden = _small_case(600, 72, 4, 16, 4, C=100, neg=0.1, zipf=1.4, seed=9)
    p = moe.Problem(N=600, H=72, k=4, E_log=16, R=4, capacity=100)
    RM = p.rows_max
    guard = 17
    G = moe.Layout.allocate(p)
    for key in ("row_token", "row_slot", "row_local_expert", "row_prob", "pad_mask"):
        big = torch.full((RM + guard,), 0x5A, dtype=G[key].dtype, device="cuda")
        G.tensors[key] = big[:RM]
        G.tensors[key + "_guard"] = big
    moe.moe_dispatch_layout(p, dev(idx), dev(probs), layout=G)
    send_big = torch.full((RM + guard, 72), 1.5, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(p, G, dev(hidden), send=send_big[:RM])
    out_big = torch.full((600 + guard, 72), -2.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(p, G, send_big[:RM], dev(probs), out=out_big[:600])
    gy_big = torch.full((RM + guard, 72), 3.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine_backward(p, G, out_big[:600].clone(), send_big[:RM], dev(probs), grad_expert_out=gy_big[:RM])
    torch.cuda.synchronize()
    for key in ("row_token", "row_slot", "row_local_expert", "row_prob", "pad_mask"):
        tail = G.tensors[key + "_guard"][RM:]
        assert torch.all(tail == torch.full_like(tail, 0x5A)), key
    assert torch.all(send_big[RM:] == 1.5) and torch.all(out_big[600:] == -2.0) and torch.all(gy_big[RM:] == 3.0)


def test_lookback_timeout_reports_and_recovers():
    """The layout's look-back gives up on a word that never comes after its limit and says so;
    the context stays usable and the same workspace serves the next call unchanged."""
    idx, probs, hidden = _small_case(4000, 16, 2, 8, 2, seed=4)
    p_bad = moe.Problem(N=4000, H=16, k=2, E_log=8, R=2, flags=moe.MOE_FLAG_TEST_WAIT_TIMEOUT)
    G = moe.moe_dispatch_layout(p_bad, dev(idx), dev(probs))
    torch.cuda.synchronize()
    assert G.status() & moe.MOE_DEV_TIMEOUT
    # the timed-out call's outputs are invalid but stay inside their buffers
    d = host(G["dest_row"])
    assert d.min() >= -1 and d.max() < G.problem.rows_max
    # the next call on the very same workspace (not zeroed again) is exact
    p = dataclasses.replace(p_bad, flags=0)
    G2 = moe.Layout.allocate(p)
    G2.workspace = G.workspace
    moe.moe_dispatch_layout(p, dev(idx), dev(probs), layout=G2)
    torch.cuda.synchronize()
    assert G2.status() == 0
    assert_layout_equal(G2, oracle.layout(idx, probs, E_log=8, R=2))


def test_misaligned_tensor_rejected_by_library():
    p = moe.Problem(N=4, H=8, k=2, E_log=4, R=2)
    idx = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    G = moe.moe_dispatch_layout(p, idx, None)
    base = torch.zeros(4 * 8 + 1, dtype=torch.bfloat16, device="cuda")
    hidden = base[1:].view(4, 8)  # 2-byte offset
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute(p, G, hidden)
    assert ei.value.code == -1


def test_streams_are_respected():
    w, d, idx, probs, L = workload_case("tiny")
    p = problem_of(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ii, pp = dev(idx), dev(probs)
        hid = dev(d["hidden"])
        G = moe.moe_dispatch_layout(p, ii, pp)
        send = moe.moe_permute(p, G, hid)
        out = moe.moe_combine(p, G, send, pp)
    s.synchronize()
    exp_send = oracle.permute(d["hidden"], L["dest_row"], L["rows_max"])
    assert np.array_equal(host(out), oracle.combine(exp_send, L["dest_row"], probs))


ROUTE_CASES = [(5, 5), (8, 1), (33, 7), (100, 8), (256, 8), (256, 32), (600, 12), (1000, 2), (1024, 32)]


@pytest.mark.parametrize("E,k", ROUTE_CASES, ids=[f"E{e}_k{k}" for e, k in ROUTE_CASES])
@pytest.mark.parametrize("kind", ["normal", "ties", "signed_zero"])
def test_route_edge_cases(E, k, kind):
    rng = np.random.default_rng(E * 100 + k)
    N = 257
    if kind == "normal":
        logits = (rng.standard_normal((N, E)) * 4).astype(np.float32)
    elif kind == "ties":
        logits = rng.integers(-2, 3, size=(N, E)).astype(np.float32)
    else:
        logits = np.where(rng.random((N, E)) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
        logits[:, ::7] = 0.5
    gi, gp = moe.moe_route_topk(dev(logits), k)
    idx, probs = oracle.route_topk(logits, k)
    torch.cuda.synchronize()
    assert np.array_equal(host(gi), idx)
    tol = route_prob_tolerance(logits, idx) * probs.astype(np.float64)
    assert np.all(np.abs(host(gp).astype(np.float64) - probs.astype(np.float64)) <= tol)


# ------------------------------------------------------------- TP folding


TP_CASES = [
    # N, H, k, E_log, R, C, reps, align, T
    (1000, 64, 4, 32, 4, 0, 0, 0, 2),
    (3000, 40, 2, 16, 2, 256, 0, 0, 4),  # capacity: drops are global, slots ceil(C/T)
    (2049, 72, 8, 64, 8, 0, 8, 16, 3),  # reroute and alignment
    (4096, 7168, 8, 256, 4, 0, 0, 0, 2),  # the 4096-token / e256 / top-8 shape
]


@pytest.mark.parametrize("case", TP_CASES, ids=[f"N{c[0]}_E{c[3]}_T{c[8]}" for c in TP_CASES])
def test_tp_fold_layout_permute_restore(case):
    N, H, k, E_log, R, C, reps, A, T = case
    idx, probs, hidden = _small_case(N, H, k, E_log, R, C, reps, 0.05, seed=N + T, zipf=1.3)
    full = oracle.layout(idx, probs, E_log=E_log, R=R, C=C, num_replicas=reps, align=A)
    exp_send_full = oracle.permute(hidden, full["dest_row"], full["rows_max"])
    expect = oracle.combine(exp_send_full, full["dest_row"], probs)
    layouts, sends, oracle_sends, oracle_dests = [], [], [], []
    for r in range(T):
        L = oracle.layout(idx, probs, E_log=E_log, R=R, C=C, num_replicas=reps, align=A, tp_size=T, tp_rank=r)
        p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps, row_align=A,
                        tp_size=T, tp_rank=r)
        G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
        torch.cuda.synchronize()
        assert_layout_equal(G, L)
        send = moe.moe_permute(p, G, dev(hidden))
        exp_send = oracle.permute(hidden, L["dest_row"], L["rows_max"])
        assert np.array_equal(host(send), exp_send)
        layouts.append(G)
        sends.append(send)
        oracle_sends.append(exp_send)
        oracle_dests.append(L["dest_row"])
    p0 = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps, row_align=A, tp_size=T)
    out = moe.moe_restore_combined(p0, layouts, sends, dev(probs))
    got = host(out)
    assert np.array_equal(got, oracle.restore_combined(oracle_sends, oracle_dests, probs))
    assert np.array_equal(got, expect)  # restore over all peers = the unfolded combine
    assert all(G.status() == 0 for G in layouts)


# ------------------------------------------- short rows with one or two slots

ROW_CASES = [
    # N, H, k, E_log, R, C, neg: k <= 2 with H / 8 in {128, 256, 512, 1024} takes the
    # combine kernel that holds several tokens per CTA and four chunks per thread
    (1, 1024, 1, 4, 2, 0, 0.0),  # a single token: one partly filled CTA
    (1001, 1024, 2, 16, 2, 0, 0.1),  # eight tokens per CTA, ragged last CTA, -1 ids
    (4099, 2048, 2, 64, 2, 60, 0.05),  # capacity: most tokens keep nothing, rows of zeros
    (333, 4096, 1, 8, 4, 0, 0.2),  # two tokens per CTA
    (77, 8192, 2, 32, 4, 3, 0.0),  # one token per CTA, heavy drops
]


@pytest.mark.parametrize("case", ROW_CASES, ids=[f"N{c[0]}_H{c[1]}_k{c[2]}_C{c[5]}" for c in ROW_CASES])
def test_combine_short_rows(case):
    N, H, k, E_log, R, C, neg = case
    idx, probs, hidden = _small_case(N, H, k, E_log, R, C, 0, neg, seed=N + H, zipf=1.5)
    L = oracle.layout(idx, probs, E_log=E_log, R=R, C=C)
    p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    send = moe.moe_permute(p, G, dev(hidden))
    exp_send = oracle.permute(hidden, L["dest_row"], L["rows_max"])
    assert np.array_equal(host(send), exp_send)
    for w in (probs, None):
        out = moe.moe_combine(p, G, send, None if w is None else dev(w))
        assert np.array_equal(host(out), oracle.combine(exp_send, L["dest_row"], w))
    rng = np.random.default_rng(N)
    g = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    gy, _ = moe.moe_combine_backward(p, G, dev(g), send, dev(probs))
    exp_gy, _ = oracle.combine_backward(g, exp_send, L["dest_row"], L["row_token"], L["row_prob"])
    assert np.array_equal(host(gy), exp_gy)
    assert np.array_equal(host(moe.moe_permute_backward(p, G, gy)), oracle.permute_backward(exp_gy, L["dest_row"]))
    assert G.status() == 0


# ------------------------------------------------------- DeepEP-style dedup


DEDUP_CASES = [
    # N, H, k, E_log, R, C, reps, align, T
    (4096, 7168, 8, 256, 4, 0, 0, 0, 0),  # the 4096-token / e256 / top-8 shape
    (1000, 72, 4, 32, 8, 0, 0, 0, 0),
    (3000, 40, 2, 16, 2, 256, 0, 16, 0),  # capacity + alignment
    (2049, 24, 8, 64, 8, 0, 8, 0, 2),  # reroute + TP folding (peer 0)
    (300, 16, 12, 48, 16, 0, 0, 0, 0),  # k > 8, E_loc not a multiple of 16
    (70000, 8, 1, 4, 2, 0, 0, 0, 0),  # many tokens, several per lane
    (2500, 2048, 2, 16, 2, 0, 0, 0, 0),  # sender-side sum over two ranks on 4 KB rows
]


@pytest.mark.parametrize("case", DEDUP_CASES, ids=[f"N{c[0]}_k{c[2]}_E{c[3]}_R{c[4]}" for c in DEDUP_CASES])
def test_dedup_path(case):
    N, H, k, E_log, R, C, reps, A, T = case
    idx, probs, hidden = _small_case(N, H, k, E_log, R, C, reps, 0.05, seed=N + R, zipf=1.3)
    L = oracle.layout(idx, probs, E_log=E_log, R=R, C=C, num_replicas=reps, align=A, tp_size=T)
    D = oracle.dedup_layout(L, probs, E_log=E_log, R=R, num_replicas=reps)
    p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps, row_align=A, tp_size=T)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    V = moe.moe_dedup_layout(p, G, dev(probs))
    torch.cuda.synchronize()
    for key in ("num_tokens_per_rank", "recv_rank_offsets", "num_recv", "is_token_in_rank", "token_rank_row",
                "recv_src_token", "recv_topk_idx", "recv_topk_weights", "recv_routing_map", "recv_probs",
                "recv_pad_mask"):
        got = host(V[key]).reshape(-1)
        exp = np.asarray(D[key]).reshape(-1)
        assert np.array_equal(got.view(np.uint8), exp.astype(got.dtype).view(np.uint8)), key
    recv_x = moe.moe_dedup_dispatch(p, V, dev(hidden))
    assert np.array_equal(host(recv_x), oracle.permute(hidden, D["token_rank_row"], D["recv_max"]))
    send = moe.moe_permute(p, G, dev(hidden))
    exp_send = oracle.permute(hidden, L["dest_row"], L["rows_max"])
    partial = moe.moe_dedup_combine_local(p, G, V, send, dev(probs))
    exp_partial = oracle.dedup_combine_local(exp_send, L, D, probs, R)
    assert np.array_equal(host(partial), exp_partial)
    out = moe.moe_dedup_combine(p, V, partial)
    assert np.array_equal(host(out), oracle.combine(exp_partial, D["token_rank_row"], None))
    assert G.status() == 0 and V.status() == 0


# ------------------------------------------------- expert-parallel exchange

EP_CASES = [
    # R, N, H, k, E_log, C, replicas, row_align
    (2, 300, 64, 2, 8, 0, 0, 0),
    (4, 1000, 136, 4, 16, 0, 0, 0),
    (4, 2000, 264, 4, 16, 80, 0, 0),  # capacity: drops and padding rows
    (4, 1500, 72, 4, 16, 0, 4, 0),  # reroute: one replica slot per rank
    (4, 1200, 40, 3, 16, 0, 0, 8),  # alignment padding, k = 3
    (8, 2048, 1024, 8, 64, 0, 0, 0),  # 8 ranks, top-8
]


@pytest.mark.parametrize("case", EP_CASES, ids=[f"R{c[0]}_N{c[1]}_H{c[2]}_k{c[3]}_C{c[5]}_rep{c[6]}_A{c[7]}"
                                                for c in EP_CASES])
def test_ep_exchange(case):
    """R ranks' dispatch into each other's receive buffers and the combine back, against the oracle."""
    R, N, H, k, E_log, C, reps, A = case
    p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps, row_align=A)
    srcs = [_small_case(N, H, k, E_log, R, C, reps, 0.05, seed=1000 * R + s, zipf=1.3) for s in range(R)]
    layouts = [moe.moe_dispatch_layout(p, dev(idx), dev(probs)) for idx, probs, _ in srcs]
    offsets_all = torch.stack([G["expert_offsets"] for G in layouts])
    plans = [moe.moe_ep_plan(p, offsets_all, s) for s in range(R)]
    RR = moe.moe_ep_recv_rows_max(p)
    canary = torch.tensor(0x7F7F, dtype=torch.int16).view(torch.bfloat16).item()
    recv = [torch.full((RR, H), canary, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    table = moe.peer_table(recv)
    for s, (_, _, hidden) in enumerate(srcs):
        moe.moe_ep_dispatch(p, layouts[s], plans[s], dev(hidden), table)
    outs = [moe.moe_ep_combine(p, layouts[s], plans[s], table, dev(srcs[s][1])) for s in range(R)]  # identity experts
    torch.cuda.synchronize()
    L_or = [oracle.layout(idx, probs, E_log=E_log, R=R, C=C, num_replicas=reps, align=A) for idx, probs, _ in srcs]
    sends = [oracle.permute(h, L["dest_row"], L["rows_max"]) for (_, _, h), L in zip(srcs, L_or)]
    rv, roff, base = oracle.ep_exchange(L_or, sends, R)
    for r in range(R):
        n = len(rv[r])
        got = host(recv[r])
        assert int(host(plans[r].num_recv)[0]) == n
        assert np.array_equal(host(plans[r].recv_expert_offsets), roff[r])
        assert np.array_equal(got[:n], rv[r])
        assert np.all(got[n:] == 0x7F7F)  # rows past num_recv are left alone
    for s in range(R):
        assert np.array_equal(host(plans[s].base), base[s])
        assert np.array_equal(host(outs[s]), oracle.combine(sends[s], L_or[s]["dest_row"], srcs[s][1]))
        assert layouts[s].status() == 0 and int(host(plans[s].status)[0]) == 0

    # backward through the exchange: combine backward into the owners' gradient buffers,
    # then the dispatch backward (the EP combine with unit weights over them)
    rng = np.random.default_rng(R * 7 + N)
    grads = [bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32)) for _ in range(R)]
    gbufs = [torch.full((RR, H), canary, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    gtable = moe.peer_table(gbufs)
    gps = [moe.moe_ep_combine_backward(p, layouts[s], plans[s], dev(grads[s]), table, dev(srcs[s][1]), gtable)
           for s in range(R)]
    torch.cuda.synchronize()
    ghs = [moe.moe_ep_combine(p, layouts[s], plans[s], gtable, None) for s in range(R)]
    torch.cuda.synchronize()
    exp_gy = []
    for s in range(R):
        gy, gp = oracle.combine_backward(grads[s], sends[s], L_or[s]["dest_row"], L_or[s]["row_token"],
                                         L_or[s]["row_prob"])
        exp_gy.append(gy)
        # same arithmetic as the one-buffer backward: grad_probs bit for bit
        _, gp_local = moe.moe_combine_backward(p, layouts[s], dev(grads[s]), dev(sends[s]), dev(srcs[s][1]))
        torch.cuda.synchronize()
        assert np.array_equal(host(gps[s]).view(np.uint32), host(gp_local).view(np.uint32))
        assert np.allclose(host(gps[s]), gp, rtol=1e-4, atol=1e-4 * np.sqrt(H))
        assert np.array_equal(host(ghs[s]), oracle.permute_backward(gy, L_or[s]["dest_row"]))
    g_rv, _, _ = oracle.ep_exchange(L_or, exp_gy, R)
    for r in range(R):
        n = len(g_rv[r])
        got = host(gbufs[r])
        assert np.array_equal(got[:n], g_rv[r])
        assert np.all(got[n:] == 0x7F7F)
    assert all(G.status() == 0 for G in layouts)


# ------------------------------------------------- randomized sweep


def _sweep_cases(n=40, seed=20261202):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        R = int(rng.choice([1, 2, 3, 4, 8]))
        E_log = R * int(rng.integers(1, 9))
        k = int(rng.integers(1, min(E_log, 10) + 1))
        reps = R * int(rng.integers(0, 2)) if E_log > R else 0
        reps = min(reps, E_log)
        N = int(rng.choice([1, 2, 31, 33, 257, 1000, 3001]))
        H = 8 * int(rng.choice([1, 3, 16, 33, 130]))
        C = int(rng.choice([0, 0, 1, 7, 40]))
        A = int(rng.choice([0, 0, 2, 8])) if C == 0 else 0
        if C and A:
            continue
        neg = float(rng.choice([0.0, 0.1]))
        cases.append((N, H, k, E_log, R, C, reps, A, neg, int(rng.integers(1 << 30))))
    return cases


@pytest.mark.parametrize("case", _sweep_cases(), ids=lambda c: "N{}_H{}_k{}_E{}_R{}_C{}_rep{}_A{}".format(*c[:8]))
def test_random_sweep_full_path(case):
    """Random small problems (every option mixed) through layout, permute, combine and both backwards."""
    N, H, k, E_log, R, C, reps, A, neg, seed = case
    idx, probs, hidden = _small_case(N, H, k, E_log, R, C, reps, neg, seed=seed, zipf=1.3)
    L = oracle.layout(idx, probs, E_log=E_log, R=R, C=C, num_replicas=reps, align=A)
    p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps, row_align=A)
    G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
    send = moe.moe_permute(p, G, dev(hidden))
    out = moe.moe_combine(p, G, send, dev(probs))
    rng = np.random.default_rng(seed + 1)
    g = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    gy, gp = moe.moe_combine_backward(p, G, dev(g), send, dev(probs))
    gh = moe.moe_permute_backward(p, G, gy)
    torch.cuda.synchronize()
    assert_layout_equal(G, L)
    exp_send = oracle.permute(hidden, L["dest_row"], L["rows_max"])
    assert np.array_equal(host(send), exp_send)
    assert np.array_equal(host(out), oracle.combine(exp_send, L["dest_row"], probs))
    exp_gy, exp_gp = oracle.combine_backward(g, exp_send, L["dest_row"], L["row_token"], L["row_prob"])
    assert np.array_equal(host(gy), exp_gy)
    assert np.allclose(host(gp), exp_gp, rtol=1e-4, atol=1e-4 * np.sqrt(H))
    assert np.array_equal(host(gh), oracle.permute_backward(exp_gy, L["dest_row"]))
    assert G.status() == 0
    check_dispatch(p, idx, probs, hidden, L)
    check_dispatch(dataclasses.replace(p, flags=moe.MOE_FLAG_DISPATCH_BULK_COPY), idx, probs, hidden, L)


def _sweep_next_cases(n=36, seed=20261203):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        mode = ("tp", "dedup", "ep")[len(cases) % 3]
        R = int(rng.choice([1, 2, 3, 4, 8])) if mode != "ep" else int(rng.choice([2, 3, 4, 8]))
        E_log = R * int(rng.integers(1, 9))
        k = int(rng.integers(1, min(E_log, 10) + 1))
        reps = R if (E_log > R and rng.random() < 0.4) else 0
        N = int(rng.choice([1, 33, 257, 1000, 3001]))
        H = 8 * int(rng.choice([1, 3, 16, 33]))
        C = int(rng.choice([0, 0, 8, 40]))
        A = int(rng.choice([0, 0, 2, 8]))
        if C and A and C % A:
            continue
        T = int(rng.choice([2, 3, 4])) if mode == "tp" else 0
        if mode == "tp" and C and A and (-(-C // T)) % A:
            continue
        cases.append((mode, N, H, k, E_log, R, C, reps, A, T))
    return cases


@pytest.mark.parametrize("case", _sweep_next_cases(),
                         ids=lambda c: "{}_N{}_H{}_k{}_E{}_R{}_C{}_rep{}_A{}_T{}".format(*c))
def test_random_sweep_next_rows(case):
    """Random small problems through the TP-fold restore, the dedup view or the EP exchange."""
    mode, N, H, k, E_log, R, C, reps, A, T = case
    if mode == "tp":
        test_tp_fold_layout_permute_restore((N, H, k, E_log, R, C, reps, A, T))
    elif mode == "dedup":
        test_dedup_path((N, H, k, E_log, R, C, reps, A, T))
    else:
        test_ep_exchange((R, N, H, k, E_log, C, reps, A))


def test_lookback_epochs_across_many_launches():
    """Every launch of the layout advances the workspace's epoch by one and leaves its ticket
    count at zero; 4200 launches in a row on one workspace, alternating two grid sizes, stay
    exact (each launch's look-back ignores the words of the launches before it)."""
    cases = []
    for N, seed in ((4096, 99), (1000, 98)):  # 16 and 4 count blocks
        idx, probs, _ = _small_case(N, 8, 2, 16, 4, seed=seed)
        p = moe.Problem(N=N, H=8, k=2, E_log=16, R=4)
        cases.append((p, idx, probs, dev(idx), dev(probs)))
    ws = moe.Layout.allocate(cases[0][0]).workspace
    lays = []
    for p, *_ in cases:
        G = moe.Layout.allocate(p)
        G.workspace = ws
        lays.append(G)
    for i in range(4200):
        p, _, _, d_idx, d_probs = cases[i % 2]
        moe.moe_dispatch_layout(p, d_idx, d_probs, layout=lays[i % 2])
    torch.cuda.synchronize()
    for (p, idx, probs, _, _), G in zip(cases, lays):
        assert G.status() == 0
        assert_layout_equal(G, oracle.layout(idx, probs, E_log=16, R=4))
    ticket = int(ws[:8].view(torch.int64).item())
    assert ticket == 4200 << 32  # epoch 4200, no ticket outstanding


def test_nvtx_ranges_on():
    """With MOE_RT_NVTX=1 every entry point opens and closes an NVTX range; the path is unchanged."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, MOE_RT_NVTX="1")
    r = subprocess.run([sys.executable, "-c", "import __graft_entry__ as g; g.smoke()"], cwd=root, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "smoke: ok" in r.stdout


@pytest.mark.parametrize("kind", ["ties_spread", "ties_dense", "one_lane_heavy"])
def test_route_candidate_paths(kind):
    """The router's candidate fast path (at most two keys per lane at or above the k-th
    lane maximum) and its fallback must pick the same ids, ties at the threshold included."""
    rng = np.random.default_rng(11)
    N, E, k = 300, 256, 8
    logits = (rng.standard_normal((N, E)) - 3.0).astype(np.float32)
    if kind == "ties_spread":  # ten equal maxima on ten different lanes: fast path, ties at t0
        hot = [1, 34, 67, 100, 133, 166, 199, 232, 9, 42]
        logits[:, hot] = 5.0
    elif kind == "ties_dense":  # equal maxima three per lane: the fallback
        hot = [3, 35, 67, 99, 4, 36, 68, 100, 5]
        logits[:, hot] = 5.0
    else:  # one lane holds all the large keys
        hot = [7, 39, 71, 103, 135, 167, 199, 231]
        logits[:, hot] = 4.0 + rng.random((N, len(hot))).astype(np.float32)
    gi, gp = moe.moe_route_topk(dev(logits), k)
    idx, probs = oracle.route_topk(logits, k)
    torch.cuda.synchronize()
    assert np.array_equal(host(gi), idx)
    tol = route_prob_tolerance(logits, idx) * probs.astype(np.float64)
    assert np.all(np.abs(host(gp).astype(np.float64) - probs.astype(np.float64)) <= tol)


def test_counts_prefetch_to_host():
    """Layout.prefetch_counts: pinned host copies of the counts, readable after the layout without a sync point."""
    w, d, idx, probs, L = workload_case("capacity")
    G = moe.moe_dispatch_layout(problem_of(w), dev(idx), dev(probs))
    pf = G.prefetch_counts()
    got = pf.get()
    for key in ("tokens_per_expert", "expert_offsets", "input_splits", "output_splits", "num_rows", "counters"):
        assert got[key].is_pinned()
        assert np.array_equal(got[key].numpy().reshape(-1), np.asarray(L[key]).reshape(-1)), key
    assert pf.ready()
