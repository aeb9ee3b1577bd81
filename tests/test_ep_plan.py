"""Expert parallelism, the host side (no GPU): the grouping plan of the rows a
rank receives (lmoe_ep_local_plan) against its definition, and the
exchange of counts and rows between gloo ranks (mixture_experts_layer_64_b200.ep)
against a single-process routing of all ranks' tokens, bit for bit.

The paper's deployment (LatentMoE, Section 2.2 and the paragraph after
Eq. (1)) splits the N experts over the ranks and moves each token's rows to
the owners of its experts and back; the plan decides where every row goes
and in which order the owner sees it."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402
from mixture_experts_layer_64_b200 import ep, lmoe, workloads  # noqa: E402


def _plan_by_definition(rc: np.ndarray):
    """Received rows are source-major (then expert); the grouped order is
    expert-major, then source, each block's rows as sent."""
    world, n = rc.shape
    recv_start = np.zeros((world, n), dtype=np.int64)
    run = 0
    for s in range(world):
        for e in range(n):
            recv_start[s, e] = run
            run += rc[s, e]
    perm, offsets = [], [0]
    for e in range(n):
        for s in range(world):
            perm += list(range(recv_start[s, e], recv_start[s, e] + rc[s, e]))
        offsets.append(len(perm))
    return np.array(offsets, dtype=np.int32), np.array(perm, dtype=np.int32)


@pytest.mark.parametrize("world,n,seed", [(1, 4, 0), (2, 3, 1), (4, 8, 2), (8, 1, 3), (3, 5, 4)])
def test_local_plan_matches_its_definition(world, n, seed):
    rng = np.random.default_rng(seed)
    rc = rng.integers(0, 7, size=(world, n)).astype(np.int32)
    rc[rng.random((world, n)) < 0.3] = 0  # empty blocks, sources and experts
    got = lmoe.ep_local_plan(rc)
    off, perm = _plan_by_definition(rc)
    np.testing.assert_array_equal(got["offsets"], off)
    np.testing.assert_array_equal(got["perm"], perm)
    assert sorted(got["perm"].tolist()) == list(range(int(rc.sum())))  # a permutation


def test_local_plan_rejects_bad_counts():
    with pytest.raises(lmoe.LmoeError):
        lmoe.ep_local_plan(np.array([[1, -1]], dtype=np.int32))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


T_RANK, N, K = 37, 16, 4


def _routing(rank: int):
    """Rank r's routing of its own T_RANK tokens (seeded logits, oracle)."""
    lg = workloads.make_logits(T_RANK, N, seed=100 + rank, ties=True).numpy()
    return oracle.route(lg, K)


def _rank_main(rank, world, port, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        n = N // world
        idx, _, offsets, perm = _routing(rank)
        counts = torch.from_numpy(np.diff(offsets).astype(np.int32))
        recv_counts, send_splits, recv_splits = ep.exchange_counts(counts, world)
        # the payload of sorted row r: (source rank, token, slot) packed in an int64
        ids = torch.from_numpy((rank << 32) + perm.astype(np.int64))
        recv = ep.exchange_rows(ids, send_splits, recv_splits)
        plan = lmoe.ep_local_plan(recv_counts.numpy())
        grouped = recv.numpy()[plan["perm"]]
        # the return trip: a function of each received row, back in send order
        back = ep.exchange_rows(recv * 3 + 1, recv_splits, send_splits)
        q.put((rank, recv_counts.numpy().tolist(), plan["offsets"].tolist(), grouped.tolist(),
               bool(torch.equal(back, ids * 3 + 1))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_groups_rows_like_a_single_routing(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # reference: every rank's routing in one process; the owner of expert e
    # must see its rows grouped by expert, then by source rank, then token
    routes = [_routing(r) for r in range(world)]
    n = N // world
    for rank, recv_counts, offsets, grouped, back_ok in res:
        assert back_ok  # every source got its own rows back, in send order
        want, want_off = [], [0]
        for e_local in range(n):
            e = rank * n + e_local
            for s in range(world):
                idx = routes[s][0]
                for t in range(T_RANK):
                    for j in range(K):
                        if idx[t, j] == e:
                            want.append((s << 32) + t * K + j)
            want_off.append(len(want))
        assert grouped == want
        assert offsets == want_off
        for s in range(world):  # counts: what source s routed to my experts
            off = routes[s][2]
            assert recv_counts[s] == [int(off[rank * n + e + 1] - off[rank * n + e])
                                      for e in range(n)]
