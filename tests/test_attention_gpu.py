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
                                  "wan2.1-1.3b-batched-b2", "wan2.1-1.3b-720p-21x45x80"])
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


# ---------------------------------------------------------------------------
# A routing list that breaks the contract (Eq. (12)-(13): the dense set is a
# subset of the sample's N tokens, listed in increasing order).  Q, K, V and
# out live inside larger buffers with guard rows before and after, so an
# access the kernel should not make lands in memory the test owns and checks.
# ---------------------------------------------------------------------------

_GUARD = 64  # rows of d values before and after each tensor
_SENTINEL = 0x7FC1  # a bf16 NaN pattern the kernel never writes


def _guarded(bits, B, H, N, d):
    """bf16 bits [B,H,N,d] placed inside a [B*H*N + 2*_GUARD, d] device buffer."""
    import torch
    total = B * H * N + 2 * _GUARD
    host = np.full((total, d), _SENTINEL, np.uint16)
    if bits is not None:
        host[_GUARD:_GUARD + B * H * N] = bits.reshape(-1, d)
    buf = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16).cuda()
    view = buf[_GUARD:_GUARD + B * H * N].view(B, H, N, d)
    return buf, view


def _noalloc_call(heta, Q, K, V, grid, win, dense, out, st):
    import ctypes
    import math
    import torch
    fn = heta.load().heta_attention_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp] + [i] * 9 + [ctypes.c_float, vp, i, vp, vp, vp]
    fn.restype = i
    B, H, N, d = Q.shape
    rc = fn(vp(Q.data_ptr()), vp(K.data_ptr()), vp(V.data_ptr()), B, H, d, *grid, *win,
            ctypes.c_float(1.0 / math.sqrt(d)), vp(dense.data_ptr()), dense.shape[1],
            vp(out.data_ptr()), vp(st.data_ptr()),
            vp(torch.cuda.current_stream().cuda_stream))
    assert rc == heta.HETA_OK, heta.status_string(rc)


@pytest.mark.parametrize("entry", ["attention", "attention_counts", "attention_noalloc"])
def test_bad_dense_idx_is_reported_and_stays_in_bounds(gpu_lib, entry):
    """Sample 0's list starts with -1 and sample 2's ends with N + 5 (both
    still increasing); sample 1's holds N in the middle and one swapped pair.
    The status must read HETA_ERR_INVALID_ARG, no guard row of out may
    change, samples 0 and 2 must equal the oracle with the bad entries left
    out (their tokens get the local result), and the key range of the dense
    rows is split in two (N = 2560), so both halves check their rows."""
    import torch
    heta = gpu_lib
    w = dataclasses.replace(W.scaled(W.WAN21, B=3, H=2, d=128, grid=(4, 16, 40),
                                     win=(3, 5, 7), u_kind="uniform", u_seeds=(31, 32, 33)),
                            name="bad-dense-idx")
    B, H, N, d = w.B, w.H, w.N, w.d
    q, k, v = W.make_qkv(w)
    u = W.make_u(w)
    kk = heta.dense_count(N, 0.2)
    od, _, _ = oracle.route(u, kk)
    bad = od.copy()
    bad[0, 0] = -1
    bad[2, kk - 1] = N + 5
    bad[1, 100] = N
    bad[1, 200], bad[1, 201] = od[1, 201], od[1, 200]
    qb, Qd = _guarded(q, B, H, N, d)
    kb, Kd = _guarded(k, B, H, N, d)
    vb, Vd = _guarded(v, B, H, N, d)
    ob, out = _guarded(None, B, H, N, d)
    out.fill_(float("nan"))
    dense = to_dev(bad)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if entry == "attention":
        heta.attention(Qd, Kd, Vd, w.grid, w.win, dense, out=out, status=st)
    elif entry == "attention_counts":
        counts = torch.full((B,), kk, dtype=torch.int32, device="cuda")
        heta.attention_counts(Qd, Kd, Vd, w.grid, w.win, dense, counts, out=out, status=st)
    else:
        _noalloc_call(heta, Qd, Kd, Vd, w.grid, w.win, dense, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == heta.HETA_ERR_INVALID_ARG
    raw = ob.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(raw[:_GUARD] == _SENTINEL), "a row before out was written"
    assert np.all(raw[_GUARD + B * H * N:] == _SENTINEL), "a row after out was written"
    got = from_dev_bf16(out)
    qf, kf, vf = W.bf16_to_f32(q), W.bf16_to_f32(k), W.bf16_to_f32(v)
    for b, keep in ((0, od[0, 1:]), (2, od[2, :kk - 1])):
        want = oracle.attention(qf[b:b + 1], kf[b:b + 1], vf[b:b + 1], w.grid, w.win,
                                keep[None, :])
        assert_close(got[b:b + 1].reshape(-1, d), want.reshape(-1, d), "sample %d" % b)


def test_out_16_byte_aligned_gives_the_same_rows(gpu_lib):
    """An out that is 16- but not 32-byte aligned takes the epilogue's
    16-byte stores instead of its 32-byte ones; every row must equal, bit for
    bit, the rows written into a 32-byte aligned out (DENSE and LOCAL rows
    alike), and none may be left unwritten."""
    import torch
    heta = gpu_lib
    w = MULTI_TILE[0]
    q, k, v = W.make_qkv(w)
    kk = heta.dense_count(w.N, 0.2)
    Qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    dense, _, _, _ = heta.route(to_dev(W.make_u(w)), kk)
    a = torch.full_like(Qd, float("nan"))
    buf = torch.full((Qd.numel() + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    b = buf[8:].view(Qd.shape)
    assert a.data_ptr() % 32 == 0 and b.data_ptr() % 32 == 16
    for out in (a, b):
        heta.attention(Qd, Kd, Vd, w.grid, w.win, dense, out=out)
    torch.cuda.synchronize()
    ga, gb = from_dev_bf16(a), from_dev_bf16(b)
    assert not np.isnan(ga).any(), "rows left unwritten"
    assert np.array_equal(a.view(torch.int16).cpu().numpy(), b.view(torch.int16).cpu().numpy())
