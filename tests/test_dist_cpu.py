"""Multi-rank host logic on CPU: gloo, world size 2, two real processes."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from uncertainty_routed_heterogeneous_b200 import dist as D
from uncertainty_routed_heterogeneous_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    info = D.rank_info()
    D.init("gloo", info, timeout_s=30)
    D.barrier(info)
    # each rank reports its own elapsed time; every rank must see the max
    m = D.max_over_ranks(1.5 + rank, info)
    w = D.rank_workload(W.WAN21, info.rank)
    q.put((rank, m, w.qkv_seed, w.u_seeds, w.x_seed, D.head_range(12, world, rank)))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_agree_on_max_and_get_independent_samples():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    (r0, m0, s0, u0, x0, h0), (r1, m1, s1, u1, x1, h1) = res
    assert m0 == m1 == 2.5
    assert s0 != s1 and u0 != u1 and x0 != x1
    assert h0 == (0, 6) and h1 == (6, 12)


@pytest.mark.parametrize("H,world", [(12, 1), (12, 5), (24, 8), (3, 4)])
def test_head_ranges_partition(H, world):
    seen = []
    for r in range(world):
        lo, hi = D.head_range(H, world, r)
        seen += list(range(lo, hi))
    assert seen == list(range(H))


def _worker_one_dies(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    info = D.rank_info()
    D.init("gloo", info, timeout_s=5)
    if rank == 1:
        # a rank that fails between steps: it leaves without its next collective
        os._exit(3)
    import time
    t0 = time.monotonic()
    try:
        D.barrier(info)
        D.max_over_ranks(1.0, info)
        q.put(("no error", time.monotonic() - t0))
    except Exception as e:  # the surviving rank learns of it as an error, not a hang
        q.put((type(e).__name__, time.monotonic() - t0))


def test_a_rank_that_dies_ends_the_others_collective_with_an_error():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_one_dies, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    what, secs = q.get(timeout=120)
    for p in procs:
        p.join(60)
    assert what != "no error"
    assert secs < 60
    assert procs[1].exitcode == 3


def _worker_heads(rank, world, port, q):
    """One sample split by heads: each rank computes its head block of the
    attention and its token rows of the uncertainty head with the oracle, then
    the blocks are gathered the way the head-sharded bench step gathers them."""
    import numpy as np
    import torch

    import oracle
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    info = D.rank_info()
    D.init("gloo", info, timeout_s=30)
    w = W.scaled(W.WAN21, H=4, d=64, grid=(3, 8, 10), win=(3, 5, 5), u_kind="uniform",
                 u_seeds=(41,), C=64)
    q_, k_, v_ = (W.bf16_to_f32(a) for a in W.make_qkv(w))
    u = W.make_u(w)
    X, wv = W.make_head(w)
    X = W.bf16_to_f32(X)
    kk = oracle.dense_count(w.N, w.rho)
    dense, _, _ = oracle.route(u, kk)  # every rank routes the same u itself
    h0, h1 = D.head_range(w.H, world, rank)
    out = oracle.attention(q_[:, h0:h1], k_[:, h0:h1], v_[:, h0:h1], w.grid, w.win, dense)
    r0, r1 = D.row_range(w.B * w.N, world, rank)
    u_next = oracle.uncertainty(X.reshape(1, -1, w.C)[:, r0:r1], wv)
    out_all = D.all_gather_equal(torch.from_numpy(np.ascontiguousarray(out)), info)
    u_all = D.all_gather_equal(torch.from_numpy(np.ascontiguousarray(u_next)), info)
    q.put((rank, out_all.numpy(), u_all.numpy()))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_head_sharded_step_gathers_to_the_single_rank_result():
    import numpy as np

    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_heads, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    w = W.scaled(W.WAN21, H=4, d=64, grid=(3, 8, 10), win=(3, 5, 5), u_kind="uniform",
                 u_seeds=(41,), C=64)
    q_, k_, v_ = (W.bf16_to_f32(a) for a in W.make_qkv(w))
    u = W.make_u(w)
    X, wv = W.make_head(w)
    kk = oracle.dense_count(w.N, w.rho)
    dense, _, _ = oracle.route(u, kk)
    want_out = oracle.attention(q_, k_, v_, w.grid, w.win, dense)
    want_u = oracle.uncertainty(W.bf16_to_f32(X), wv)
    for _, out_all, u_all in res:
        assert np.array_equal(out_all.reshape(want_out.shape), want_out)
        assert np.array_equal(u_all.reshape(want_u.shape), want_u)
