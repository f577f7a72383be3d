"""heta_attention on the GPU against the fp64 oracle.

"Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion": Eq. (2) dense rows, Eq. (3) windowed local rows, Eq. (13) merge.
Tolerance: max abs <= 2e-2 and mean abs <= 2e-3 against fp64 on the same
bf16-rounded inputs (bf16 inputs, fp32 accumulation, bf16 output).
Every output is pre-filled with NaN, so a row the kernels never write fails.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from helpers import assert_close, from_dev_bf16, sample_rows, to_dev, to_dev_bf16
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def run(heta, w, rho=None, n_sample=None, u=None, seed=0):
    import torch
    rho = w.rho if rho is None else rho
    q, k, v = W.make_qkv(w)
    if u is None:
        u = W.make_u(w)
    kk = heta.dense_count(w.N, rho)
    Qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    dense, _, _, _ = heta.route(to_dev(u), kk)
    out = torch.full_like(Qd, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    heta.attention(Qd, Kd, Vd, w.grid, w.win, dense, out=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    od, _, _ = oracle.route(u, kk)
    assert np.array_equal(dense.cpu().numpy(), od)
    got = from_dev_bf16(out).reshape(-1, w.d)
    assert not np.isnan(got).any(), "rows left unwritten"
    qf, kf, vf = W.bf16_to_f32(q), W.bf16_to_f32(k), W.bf16_to_f32(v)
    if n_sample is None:
        rows = np.arange(w.B * w.H * w.N, dtype=np.int64)
    else:
        rows = sample_rows(np.random.default_rng(seed), w.B, w.H, w.N, w.grid, w.win, od,
                           n_sample)
    want = oracle.attention_rows(qf, kf, vf, w.grid, w.win, od, rows)
    return assert_close(got[rows], want, w.name)


def test_tiny_all_rows(gpu_lib):
    run(gpu_lib, W.TINY)


MULTI_TILE = [
    # several 128-row tiles with ragged tails on every axis
    W.scaled(W.WAN21, H=2, grid=(5, 12, 20), u_kind="smooth"),
    dataclasses.replace(W.scaled(W.WAN21, H=3, d=64, grid=(3, 17, 19), win=(3, 5, 7),
                                 u_kind="uniform", u_seeds=(9,)), name="ragged-d64"),
    dataclasses.replace(W.scaled(W.WAN21, B=2, H=2, grid=(6, 10, 14), win=(1, 3, 5),
                                 u_kind="clustered", u_seeds=(3, 4)), name="b2-clustered"),
    dataclasses.replace(W.scaled(W.WAN21, H=1, grid=(3, 9, 9), win=(3, 9, 9),
                                 u_kind="uniform", u_seeds=(5,)), name="window-is-grid"),
]


@pytest.mark.parametrize("w", MULTI_TILE, ids=lambda w: w.name)
@pytest.mark.parametrize("rho", [0.0, 0.2, 0.35, 1.0])
def test_multi_tile_all_rows(gpu_lib, w, rho):
    run(gpu_lib, w, rho=rho)


@pytest.mark.parametrize("name", ["wan2.1-1.3b-21x30x52", "wan2.2-5b-31x22x40",
                                  "wan2.1-1.3b-batched-b2"])
def test_full_size_sampled_rows(gpu_lib, name):
    """4096 random rows per head on average, plus every border-clamped window
    class and the first and last dense rows of the first and last head."""
    w = W.ALL[name]
    run(gpu_lib, w, n_sample=4096 * w.B * w.H)


@pytest.mark.parametrize("rho", [0.05, 0.5])
def test_sweep_clustered_sampled_rows(gpu_lib, rho):
    w = W.sweep(rho, "clustered")
    run(gpu_lib, w, n_sample=800)


def test_rho1_equals_dense_and_rho0_equals_local(gpu_lib):
    """Two calls on one input: every row matches the oracle's dense (rho=1) or
    purely local (rho=0) result, and the two differ."""
    w = MULTI_TILE[0]
    a = run(gpu_lib, w, rho=1.0)
    b = run(gpu_lib, w, rho=0.0)
    assert a and b


# The paper's window ablation (Table 7): 9^3, 11^3 (its default) and 13^3
# neighbourhoods.  All rows on a grid just large enough for 13 along every
# axis (ragged tiles everywhere), then sampled rows at the Wan2.1 shape.
@pytest.mark.parametrize("n", W.WINDOW_CUBES)
@pytest.mark.parametrize("rho", [0.0, 0.2])
def test_window_cube_all_rows(gpu_lib, n, rho):
    w = dataclasses.replace(W.scaled(W.WAN21, H=2, grid=(13, 17, 27), win=(n, n, n),
                                     u_kind="uniform", u_seeds=(12,)),
                            name="window%d-13x17x27" % n)
    run(gpu_lib, w, rho=rho)


@pytest.mark.parametrize("n", W.WINDOW_CUBES)
def test_window_cube_full_size_sampled_rows(gpu_lib, n):
    run(gpu_lib, W.window_cube(n), n_sample=1000)


# Degenerate cases of the method: a single dense row, all but one row dense,
# a one-frame grid, a 1x1x1 window (each local row attends to itself only, so
# its output is its own v), one head and three samples.
@pytest.mark.parametrize("case", ["k1", "k_n_minus_1", "one_frame", "win111", "b3_h1"])
def test_degenerate_cases(gpu_lib, case):
    import torch
    heta = gpu_lib
    base = W.scaled(W.WAN21, H=2, grid=(3, 10, 14), win=(3, 5, 5), u_kind="uniform",
                    u_seeds=(21,))
    if case == "k1":
        w, kk = base, 1
    elif case == "k_n_minus_1":
        w, kk = base, base.N - 1
    elif case == "one_frame":
        w = dataclasses.replace(base, grid=(1, 12, 20), win=(1, 7, 9))
        kk = heta.dense_count(w.N, 0.2)
    elif case == "win111":
        w = dataclasses.replace(base, win=(1, 1, 1))
        kk = heta.dense_count(w.N, 0.2)
    else:
        w = dataclasses.replace(base, B=3, H=1, u_seeds=(21, 22, 23))
        kk = heta.dense_count(w.N, 0.3)
    w = dataclasses.replace(w, name="degenerate-" + case)
    rho = kk / w.N
    mx, mean = run(heta, w, rho=rho)
    if case == "win111":
        # local rows reproduce their own value vector (bf16 in, bf16 out)
        q, k, v = W.make_qkv(w)
        Qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
        dense, local, _, _ = heta.route(to_dev(W.make_u(w)), kk)
        out = heta.attention(Qd, Kd, Vd, w.grid, w.win, dense)
        torch.cuda.synchronize()
        loc = local.cpu().numpy()[0]
        got = from_dev_bf16(out)[0][:, loc]
        want = W.bf16_to_f32(v)[0][:, loc]
        assert np.array_equal(got, want)
