"""The step -- route, routed attention, uncertainty head -- captured in a CUDA
graph and replayed gives the eager results.

A diffusion sampler runs the same step shapes every denoising step, so it can
capture the three library calls once and replay them; every call is a
stream-ordered memset or kernel launch on the caller's stream (a first eager
call loads the kernels, so the capture sees no module load).  New inputs are
copied into the captured buffers before each replay.
"""
import numpy as np
import pytest

from helpers import to_dev, to_dev_bf16
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_step_replays_in_a_cuda_graph(gpu_lib):
    import torch
    heta = gpu_lib
    w = W.scaled(W.WAN21, H=2, d=128, grid=(6, 12, 20), win=(3, 5, 7), u_kind="uniform",
                 u_seeds=(17,), C=256)
    q, k, v = W.make_qkv(w)
    X, wv = W.make_head(w)
    Q, K, V, Xd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), to_dev_bf16(X)
    wd = to_dev(wv)
    u = to_dev(W.make_u(w))
    kk = heta.dense_count(w.N, 0.2)
    dense = torch.empty((1, kk), dtype=torch.int32, device="cuda")
    local = torch.empty((1, w.N - kk), dtype=torch.int32, device="cuda")
    out = torch.empty_like(Q)
    ws = torch.empty(max(256, heta.attention_workspace_size(1, w.H, w.d, w.grid, w.win, kk)),
                     dtype=torch.uint8, device="cuda")
    u_next = torch.empty((1, w.N), dtype=torch.float32, device="cuda")

    def step():
        heta.route(u, kk, out=(dense, local, None, None))
        heta.attention(Q, K, V, w.grid, w.win, dense, out=out, workspace=ws)
        heta.uncertainty(Xd, wd, 0.0, out=u_next)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # eager: loads every kernel before the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    want = (dense.clone(), local.clone(), out.clone(), u_next.clone())

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for rep in range(3):
        out.fill_(float("nan"))
        u_next.fill_(float("nan"))
        dense.fill_(-1)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(dense, want[0]) and torch.equal(local, want[1]), rep
        assert torch.equal(out.view(torch.int16), want[2].view(torch.int16)), rep
        assert torch.equal(u_next, want[3]), rep

    # new inputs copied into the captured buffers: the replay routes them
    u2 = W.make_u(W.scaled(w, u_seeds=(18,)))
    u.copy_(to_dev(u2))
    g.replay()
    torch.cuda.synchronize()
    d2, l2, _, _ = heta.route(to_dev(u2), kk)
    assert torch.equal(dense, d2) and torch.equal(local, l2)
    del g
