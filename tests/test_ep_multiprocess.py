"""The expert-parallel exchange between processes (combine_moe_route_tokens_b200.EpGroup).

CPU (gloo, world size 2 and 3): the host logic — every rank gets every other rank's
exported handles in rank order, the peer tables hold the rank's own buffers at its own
index and the opened peers' buffers elsewhere, and the host all-gather of expert
offsets returns every rank's layout offsets in rank order.

GPU (-m gpu): R processes, one rank each, all on one GPU; each maps the others' receive,
gradient and offset-table buffers through CUDA IPC, publishes its offsets over peer
memory, plans, dispatches into the owners' receive buffers, combines back and runs the
backward through the gradient buffers, ordered by interprocess events and host barriers.
Every rank's received rows, plan, combine output and both backward outputs are
compared with the oracle's exchange bit for bit (grad_probs within the fp32 bound).
"""

import os
import socket
import tempfile
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from synthetic import bf16_bits_from_f32


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(R, rank, N, H, k, E_log, C, reps, neg=0.05):
    """Rank `rank`'s tokens: ids (Zipf-skewed, some -1), probs, hidden rows, output gradients."""
    rng = np.random.default_rng(1000 * R + rank)
    idx = (rng.zipf(1.3, size=(N, k)) % E_log).astype(np.int32)
    idx[rng.random((N, k)) < neg] = -1
    probs = rng.random((N, k)).astype(np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    grad = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    return idx, probs, hidden, grad


# ---------------------------------------------------------------- host logic


def _host_worker(rank, world, port, outdir):
    from combine_moe_route_tokens_b200 import ep_group

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        blobs = ep_group.exchange(None, {"rank": rank, "payload": bytes([rank]) * (rank + 1)})
        own = {"recv": 1000 + rank, "grad": 2000 + rank, "offsets_all": 3000 + rank}
        opened = []

        def fake_open(blob):  # stands in for moe_ipc_open: records what it was asked to map
            opened.append(blob)
            return 10000 + len(opened), 20000 + len(opened)

        theirs = [{name: f"{name}:{r}".encode() for name in own} for r in range(world)]
        tables, mappings = ep_group.peer_pointers(rank, own, theirs, fake_open)
        N, k, E_log = 50 + 7 * rank, 3, 12
        idx, probs, _, _ = _inputs(world, rank, N, 8, k, E_log, 0, 0)
        L = oracle.layout(idx, probs, E_log=E_log, R=world)
        table = ep_group.gather_offsets_host(None, np.asarray(L["expert_offsets"], np.int32))
        np.savez(os.path.join(outdir, f"r{rank}.npz"), blobs=np.array(blobs, dtype=object),
                 tables=np.array([tables], dtype=object), mappings=np.array(mappings),
                 opened=np.array(opened, dtype=object), table=table)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_host_logic_of_the_exchange(world):
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(_host_worker, args=(world, _free_port(), outdir), nprocs=world, join=True,
                           start_method="spawn")
        res = [np.load(os.path.join(outdir, f"r{r}.npz"), allow_pickle=True) for r in range(world)]
    offsets = []
    for r in range(world):
        N = 50 + 7 * r
        idx, probs, _, _ = _inputs(world, r, N, 8, 3, 12, 0, 0)
        offsets.append(np.asarray(oracle.layout(idx, probs, E_log=12, R=world)["expert_offsets"], np.int32))
    for r, d in enumerate(res):
        blobs = list(d["blobs"])
        assert [b["rank"] for b in blobs] == list(range(world))  # rank order
        assert all(b["payload"] == bytes([q]) * (q + 1) for q, b in enumerate(blobs))
        tables = d["tables"][0]
        for name, base in (("recv", 1000), ("grad", 2000), ("offsets_all", 3000)):
            assert tables[name][r] == base + r  # own buffer at own index
            peers = [tables[name][q] for q in range(world) if q != r]
            assert all(p > 10000 for p in peers)  # every other index was opened
        opened = [bytes(b) for b in d["opened"]]
        want = [f"{name}:{q}".encode() for q in range(world) if q != r for name in ("recv", "grad", "offsets_all")]
        assert opened == want
        assert len(d["mappings"]) == 3 * (world - 1)
        assert np.array_equal(d["table"], np.stack(offsets))  # every rank's offsets, rank order


# ---------------------------------------------------------------- GPU, R processes


def _gpu_worker(rank, R, port, case, outdir):
    import combine_moe_route_tokens_b200 as moe

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=R,
                            timeout=timedelta(seconds=120))
    try:
        N, H, k, E_log, C, reps, A = case
        idx, probs, hidden, grad = _inputs(R, rank, N, H, k, E_log, C, reps)
        dev = lambda a: torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()  # noqa: E731
        bf = lambda a: dev(a).view(torch.bfloat16)  # noqa: E731
        p = moe.Problem(N=N, H=H, k=k, E_log=E_log, R=R, capacity=C, num_replicas=reps, row_align=A)
        G = moe.moe_dispatch_layout(p, dev(idx), dev(probs))
        grp = moe.EpGroup(p, rank)
        canary = torch.tensor(0x7F7F, dtype=torch.int16).view(torch.bfloat16).item()
        grp.recv.fill_(canary)
        grp.grad.fill_(canary)
        grp.fence()  # every rank's canaries are in place before anyone writes into them
        grp.publish_offsets(G)
        grp.fence()
        grp.plan_exchange()
        grp.dispatch(G, bf(hidden))
        grp.fence()  # all rows have arrived; identity experts: the receive buffer is the expert output
        out = grp.combine(G, dev(probs))
        gp = grp.combine_backward(G, bf(grad), dev(probs))
        grp.fence()  # all gradient rows have arrived
        gh = grp.dispatch_backward(G)
        torch.cuda.synchronize()
        host = lambda t: t.cpu().view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 \
            else t.cpu().numpy()  # noqa: E731
        np.savez(os.path.join(outdir, f"r{rank}.npz"), recv=host(grp.recv), grad=host(grp.grad), out=host(out),
                 gp=host(gp), gh=host(gh), base=host(grp.plan.base), num_recv=host(grp.plan.num_recv),
                 recv_off=host(grp.plan.recv_expert_offsets), offsets_all=host(grp.offsets_all),
                 status=np.array([G.status(), int(grp.plan.status.item())]))
        grp.close()
    finally:
        dist.destroy_process_group()


EP_CASES = [
    # R, N, H, k, E_log, C, reps, A
    (2, 700, 72, 4, 16, 0, 0, 0),
    (4, 513, 40, 8, 32, 0, 4, 0),  # hot-expert replicas
    (4, 900, 24, 2, 16, 60, 0, 0),  # capacity: drops and padding rows
    (2, 300, 16, 3, 8, 0, 0, 8),  # row alignment
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", EP_CASES, ids=[f"R{c[0]}_N{c[1]}_k{c[3]}_C{c[5]}_rep{c[6]}_A{c[7]}" for c in EP_CASES])
def test_exchange_between_processes(case):
    from gpu_util import require_cuda

    require_cuda()
    R, N, H, k, E_log, C, reps, A = case
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(_gpu_worker, args=(R, _free_port(), (N, H, k, E_log, C, reps, A), outdir), nprocs=R,
                           join=True, start_method="spawn")
        res = [dict(np.load(os.path.join(outdir, f"r{r}.npz"))) for r in range(R)]
    srcs = [_inputs(R, r, N, H, k, E_log, C, reps) for r in range(R)]
    L = [oracle.layout(i, p, E_log=E_log, R=R, C=C, num_replicas=reps, align=A) for i, p, _, _ in srcs]
    sends = [oracle.permute(h, l["dest_row"], l["rows_max"]) for (_, _, h, _), l in zip(srcs, L)]
    rv, roff, base = oracle.ep_exchange(L, sends, R)
    exp_gy = []
    for s in range(R):
        gy, gp = oracle.combine_backward(srcs[s][3], sends[s], L[s]["dest_row"], L[s]["row_token"], L[s]["row_prob"])
        exp_gy.append(gy)
        d = res[s]
        assert list(d["status"]) == [0, 0]
        assert np.array_equal(d["offsets_all"], np.stack([l["expert_offsets"] for l in L]))  # the all-gather
        assert np.array_equal(d["base"], base[s])
        assert np.array_equal(d["out"], oracle.combine(sends[s], L[s]["dest_row"], srcs[s][1]))
        assert np.allclose(d["gp"], gp, rtol=1e-4, atol=1e-4 * np.sqrt(H))
        assert np.array_equal(d["gh"], oracle.permute_backward(gy, L[s]["dest_row"]))
    g_rv, _, _ = oracle.ep_exchange(L, exp_gy, R)
    for r in range(R):
        n = len(rv[r])
        d = res[r]
        assert int(d["num_recv"][0]) == n
        assert np.array_equal(d["recv_off"], roff[r])
        assert np.array_equal(d["recv"][:n], rv[r]) and np.all(d["recv"][n:] == 0x7F7F)
        assert np.array_equal(d["grad"][:n], g_rv[r]) and np.all(d["grad"][n:] == 0x7F7F)
