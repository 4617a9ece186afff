"""Pipeline (two batches in flight) against the same batches run one at a time.

Each batch's output under the pipelined schedule (route and layout on a side stream
beside the previous batch's combine, permutes and combines in batch order on the main
stream, two lanes of buffers) must equal, bit for bit, the output of the same batch
through moe_route_topk -> moe_dispatch -> moe_combine on one stream, which the parity
tests compare with the oracle at every workload's full size. Six batches, so that both
lanes come round several times, enqueued eagerly and replayed from a CUDA graph; small
problems with each layout option, and the headline's batch.
"""

import pytest
import torch

CASES = [
    # N, H, k, E, R, capacity, replicas, row alignment
    (512, 1024, 8, 64, 4, 0, 0, 0),
    (300, 256, 2, 16, 2, 40, 0, 0),  # capacity: drops and pad rows
    (513, 512, 8, 32, 4, 0, 4, 0),  # hot-expert replicas (reroute)
    (257, 768, 4, 16, 2, 0, 0, 8),  # rows aligned to 8 per expert
    (4096, 7168, 8, 256, 4, 0, 0, 0),  # the headline's batch (4096 x 7168, e256, top-8, 4 ranks)
]


def _bits(t):
    return t.view(torch.int16)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[f"N{c[0]}_H{c[1]}_k{c[2]}_E{c[3]}_C{c[5]}_rep{c[6]}_A{c[7]}" for c in CASES])
def test_pipeline_matches_one_batch_at_a_time(case):
    from gpu_util import require_cuda

    require_cuda()
    import numpy as np

    import combine_moe_route_tokens_b200 as moe
    import oracle

    N, H, k, E, R, C, reps, A = case
    p = moe.Problem(N=N, H=H, k=k, E_log=E, R=R, capacity=C, num_replicas=reps, row_align=A)
    g = torch.Generator(device="cuda").manual_seed(1234 + N)
    B = 6
    logits = [torch.randn(N, E, device="cuda", generator=g) for _ in range(B)]
    hidden = [torch.randn(N, H, device="cuda", generator=g).to(torch.bfloat16) for _ in range(B)]

    ref = []
    for b in range(B):
        idx, probs = moe.moe_route_topk(logits[b], k)
        L, send = moe.moe_dispatch(p, idx, probs, hidden[b])
        ref.append(moe.moe_combine(p, L, send, probs))
        assert L.status() == 0
        # and the oracle's combine of the same routing (ids and probs from the router above)
        ids_h, probs_h = idx.cpu().numpy(), probs.cpu().numpy()
        h = hidden[b].cpu().view(torch.int16).numpy().view(np.uint16)
        OL = oracle.layout(ids_h, probs_h, E_log=E, R=R, C=C, num_replicas=reps, align=A)
        exp = oracle.combine(oracle.permute(h, OL["dest_row"], OL["rows_max"]), OL["dest_row"], probs_h)
        assert np.array_equal(ref[b].cpu().view(torch.int16).numpy().view(np.uint16), exp), f"oracle batch {b}"
    torch.cuda.synchronize()

    # eager
    pipe = moe.Pipeline(p)
    ready = torch.cuda.Event()
    ready.record()
    outs = []
    for b in range(B):
        outs.append(pipe.submit(logits[b], hidden[b], ready=ready).clone())  # before the lane comes round
    pipe.join()
    torch.cuda.synchronize()
    assert pipe.status() == 0
    for b in range(B):
        assert torch.equal(_bits(outs[b]), _bits(ref[b])), f"batch {b}"

    # captured once, replayed
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    gp = moe.Pipeline(p, stream=s)
    got = [torch.zeros_like(ref[0]) for _ in range(B)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        ready = torch.cuda.Event()
        ready.record(s)
        for b in range(B):
            got[b].copy_(gp.submit(logits[b], hidden[b], ready=ready))
        gp.join()
    for _ in range(2):
        for t in got:
            t.zero_()
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert gp.status() == 0
        for b in range(B):
            assert torch.equal(_bits(got[b]), _bits(ref[b])), f"graph batch {b}"


WORKLOADS = ["tiny", "ht", "qwen3", "capacity", "ultraep"]


@pytest.mark.gpu
@pytest.mark.parametrize("name", WORKLOADS)
def test_pipeline_at_full_size(name):
    """The forward path of each surveyed configuration at its full size with the benchmark's
    input recipe (four batches: seed offsets 0-3), two batches in flight against each batch
    alone; the batches alone are the calls the parity tests compare with the oracle."""
    from gpu_util import require_cuda

    require_cuda()
    import numpy as np

    import combine_moe_route_tokens_b200 as moe
    from synthetic import get_workload, make_inputs

    w = get_workload(name)
    p = moe.Problem(N=w.N, H=w.H, k=w.k, E_log=w.E_log, R=w.R, capacity=w.capacity,
                    num_replicas=w.num_replicas, row_align=w.row_align)
    B = 4
    logits, hidden = [], []
    for b in range(B):
        d = make_inputs(w, grad=False, seed_offset=b)
        logits.append(torch.from_numpy(d["logits"]).cuda())
        hidden.append(torch.from_numpy(d["hidden"].view(np.int16)).cuda().view(torch.bfloat16))
    ref = []
    for b in range(B):
        idx, probs = moe.moe_route_topk(logits[b], w.k)
        L, send = moe.moe_dispatch(p, idx, probs, hidden[b])
        ref.append(moe.moe_combine(p, L, send, probs))
        assert L.status() == 0
    pipe = moe.Pipeline(p)
    ready = torch.cuda.Event()
    ready.record()
    outs = [pipe.submit(logits[b], hidden[b], ready=ready).clone() for b in range(B)]
    pipe.join()
    torch.cuda.synchronize()
    assert pipe.status() == 0
    for b in range(B):
        assert torch.equal(_bits(outs[b]), _bits(ref[b])), f"{name} batch {b}"


@pytest.mark.gpu
def test_pipeline_token_mask_and_empty_batches():
    """Padding tokens masked out of routing (Megatron MORI page: router.py) go through the
    pipeline like one batch at a time; an empty batch enqueues nothing and breaks nothing."""
    from gpu_util import require_cuda

    require_cuda()
    import combine_moe_route_tokens_b200 as moe

    N, H, k, E, R = 300, 512, 4, 32, 4
    p = moe.Problem(N=N, H=H, k=k, E_log=E, R=R)
    g = torch.Generator(device="cuda").manual_seed(99)
    B = 4
    logits = [torch.randn(N, E, device="cuda", generator=g) for _ in range(B)]
    hidden = [torch.randn(N, H, device="cuda", generator=g).to(torch.bfloat16) for _ in range(B)]
    masks = [(torch.rand(N, device="cuda", generator=g) < 0.3).to(torch.uint8) for _ in range(B)]
    ref = []
    for b in range(B):
        idx, probs = moe.moe_route_topk(logits[b], k, token_mask=masks[b])
        L, send = moe.moe_dispatch(p, idx, probs, hidden[b])
        ref.append(moe.moe_combine(p, L, send, probs))
    pipe = moe.Pipeline(p)
    ready = torch.cuda.Event()
    ready.record()
    outs = [pipe.submit(logits[b], hidden[b], token_mask=masks[b], ready=ready).clone() for b in range(B)]
    pipe.join()
    torch.cuda.synchronize()
    assert pipe.status() == 0
    for b in range(B):
        assert torch.equal(_bits(outs[b]), _bits(ref[b])), f"masked batch {b}"
        assert torch.all(_bits(outs[b])[masks[b].bool()] == 0)  # a masked token keeps no slot: zero row

    p0 = moe.Problem(N=0, H=H, k=k, E_log=E, R=R)
    pipe0 = moe.Pipeline(p0)
    for _ in range(3):
        out = pipe0.submit(torch.empty((0, E), device="cuda"), torch.empty((0, H), dtype=torch.bfloat16, device="cuda"))
        assert out.shape == (0, H)
    pipe0.join()
    torch.cuda.synchronize()
    assert pipe0.status() == 0
