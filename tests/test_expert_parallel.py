"""Expert parallelism: the exchange of grouped rows between ranks, and the layer built on it.

CPU (gloo, two and four ranks): every rank routes its own tokens with the oracle, then the
module's exchange functions move the grouped rows to the ranks that own their experts and back;
each rank computes its received rows with the oracle's expert FFN and combines.  The result must
equal, bit for bit, the oracle's single-process layer on the same tokens: a row sent to the wrong
rank or expert, lost, duplicated or returned out of order changes it.

GPU (one rank over NCCL): the whole expert-parallel forward runs through the library's kernels
(route without allocation, routed expert compute on the owned experts, combine) and is compared
with the oracle; with one rank the exchanges are local copies, so this checks the compute path
and the bookkeeping around it, not NVLink transfers (every GPU call of this build has one GPU).
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    sys.path.insert(0, ROOT)
    import inputgen

    wl = inputgen.custom("ep", T=40, d=64, E=8, k=2, f=128)
    return inputgen.make_problem(wl, seed=12)


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    from sparse_expert_ffn_router_b200 import expert_parallel as ep

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        p = _problem()
        wl = p.wl
        per = wl.T // world
        toks = list(range(rank * per, (rank + 1) * per))
        x = p.x[toks].contiguous()
        # Gate + Scatter of this rank's tokens (oracle)
        logits = oracle.router_logits(x, p.router_w, p.router_b)
        idx, w, _ = oracle.topk(logits, wl.k)
        counts, offsets, src, dst = oracle.group(idx, wl.E)
        Xp = x[src.long()].contiguous()
        plan = ep.exchange_counts(counts, world)
        recv = ep.dispatch_rows(Xp, plan)
        local = ep.received_experts(plan)
        owned = ep.owned_experts(wl.E, world, rank)
        assert recv.shape[0] == sum(plan.recv_rows) and local.shape == (recv.shape[0], 1)
        # expert compute of the received rows on their owned experts (oracle)
        y_recv = torch.stack([oracle.expert_row(recv, r, p.expert_w, p.expert_stride, wl.f, None,
                                                owned[int(local[r, 0])]) for r in range(recv.shape[0])]) \
            if recv.shape[0] else torch.empty(0, wl.d)
        back = ep.return_rows(y_recv, plan)
        # Gather in slot order, float64 accumulation rounded once (the oracle's combine)
        y = torch.zeros(per, wl.d, dtype=torch.float64)
        for t in range(per):
            for j in range(wl.k):
                y[t] += float(w[t, j]) * back[int(dst[t, j])].double()
        ref = oracle.problem_forward(p, toks)["y"]
        q.put((rank, bool(torch.equal(y.float(), ref)), plan.send_rows, plan.recv_rows))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_reproduces_the_single_process_layer(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, equal, send, recv in got:
        assert equal, f"rank {rank}: layer output differs from the single-process oracle"
    # every row sent is received exactly once: the send matrix is the transpose of the receive one
    send = [g[2] for g in got]
    recv = [g[3] for g in got]
    for a in range(world):
        for b in range(world):
            assert send[a][b] == recv[b][a]


def test_owned_experts_partition_and_reject_uneven_split():
    sys.path.insert(0, ROOT)
    from sparse_expert_ffn_router_b200 import expert_parallel as ep

    parts = [list(ep.owned_experts(16, 4, r)) for r in range(4)]
    assert sum(parts, []) == list(range(16))
    with pytest.raises(ValueError):
        ep.owned_experts(10, 4, 0)


def test_received_experts_follow_source_then_expert_order():
    sys.path.insert(0, ROOT)
    from sparse_expert_ffn_router_b200 import expert_parallel as ep

    plan = ep.ExchangePlan([0, 0], [3, 2], torch.tensor([[2, 1], [0, 2]], dtype=torch.int32))
    assert ep.received_experts(plan).reshape(-1).tolist() == [0, 0, 1, 1, 1]


@pytest.mark.gpu
def test_expert_parallel_forward_on_one_rank_matches_oracle():
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    import sparse_expert_ffn_router_b200 as colibri
    from sparse_expert_ffn_router_b200 import expert_parallel as ep
    from tests import gpu_harness as H

    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        p = _problem()
        wl = p.wl
        layer = ep.ExpertParallelMoE(wl.d, wl.f, wl.E, wl.k, colibri.COLIBRI_BF16, colibri.COLIBRI_BF16,
                                     max_tokens=wl.T)
        assert layer.expert_stride == p.expert_stride
        t = H.to_device(p)
        y = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
        for _ in range(2):  # a second call over the same buffers
            layer.forward(t["x"], t["router_w"], t["router_b"], t["expert_w"], y)
            torch.cuda.synchronize()
        colibri.colibri_route_noalloc_check()
        ref = oracle.problem_forward(p)
        H.check_y(p, y.float().cpu(), ref["y"])
        layer.close()
    finally:
        dist.destroy_process_group()
