"""heta_attention_noalloc: the allocation-free entry point.

Some callers cannot allocate device memory (no cudaMalloc allowed where they
run), so they cannot hand heta_attention a workspace.  heta_attention_noalloc
takes the same arguments minus the workspace and keeps its scratch in a fixed
16 MiB array inside the library.  This file checks, through the C ABI, on
two calls in a row (the second call reuses the array the first one left
behind):

* where both entry points plan the same work (the split scratch fits the
  array), that its output equals heta_attention's bit for bit;
* where the split scratch would not fit, that it runs every dense pair
  unsplit and still matches heta_attention within the output tolerance;
* in both cases, that sampled rows (and every border class) match the fp64
  oracle within the output tolerance.

The file name sorts last so that a run stopping at the first failure has run
every other test first.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
from helpers import MAX_ABS, MEAN_ABS, assert_close, from_dev_bf16, sample_rows, to_dev, to_dev_bf16
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc(lib):
    fn = lib.heta_attention_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp] + [i] * 9 + [ctypes.c_float, vp, i, vp, vp, vp]
    fn.restype = i
    return fn


def _against_oracle(w, q, k, v, dense_np, got, n_sample, seed):
    """Sampled output rows (plus border classes and first/last dense rows)
    against the fp64 oracle."""
    rows = sample_rows(np.random.default_rng(seed), w.B, w.H, w.N, w.grid, w.win, dense_np,
                       n_sample)
    want = oracle.attention_rows(W.bf16_to_f32(q), W.bf16_to_f32(k), W.bf16_to_f32(v),
                                 w.grid, w.win, dense_np, rows)
    assert_close(got.reshape(-1, w.d)[rows], want, w.name)


@pytest.mark.parametrize("grid,win,rho,H,d", [
    ((8, 16, 24), (3, 9, 9), 0.2, 2, 128),   # dense key range split in two
    ((5, 12, 20), (3, 5, 7), 0.35, 3, 64),   # no split
])
def test_noalloc_matches_workspace_entry_point(gpu_lib, grid, win, rho, H, d):
    import torch
    heta = gpu_lib
    lib = heta.load()
    fn = _noalloc(lib)
    w = W.scaled(W.WAN21, H=H, d=d, grid=grid, win=win, u_kind="uniform", u_seeds=(11,))
    q, k, v = W.make_qkv(w)
    Q, K, V = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    kk = heta.dense_count(w.N, rho)
    dense, _, _, _ = heta.route(to_dev(W.make_u(w)), kk)
    ref = heta.attention(Q, K, V, w.grid, w.win, dense)
    torch.cuda.synchronize()
    want = from_dev_bf16(ref)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(Q, float("nan"))
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = fn(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                ctypes.c_void_p(V.data_ptr()), w.B, w.H, w.d, grid[0], grid[1], grid[2],
                win[0], win[1], win[2], ctypes.c_float(1.0 / math.sqrt(d)),
                ctypes.c_void_p(dense.data_ptr()), kk, ctypes.c_void_p(out.data_ptr()),
                ctypes.c_void_p(st.data_ptr()), stream)
        assert rc == heta.HETA_OK, heta.status_string(rc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        got = from_dev_bf16(out)
        assert np.all(np.isfinite(got)), "call %d left rows unwritten" % call
        # the same plan and the same kernel as heta_attention: the same bits
        assert np.array_equal(got, want), "call %d differs from heta_attention" % call
        _against_oracle(w, q, k, v, dense.cpu().numpy(), got, 2048, call)


def test_noalloc_runs_unsplit_when_its_array_is_too_small(gpu_lib):
    """A size whose split partials would not fit the 16 MiB array runs with
    every dense pair over its whole key range and still matches
    heta_attention (which splits)."""
    import torch
    heta = gpu_lib
    fn = _noalloc(heta.load())
    # two heads of the Wan2.1 grid with 28416 dense rows: 222 pairs = one
    # wave of 148 + 74 pairs cut in halves, ~19.5 MB of partials
    grid, win, kk = (21, 30, 52), (3, 9, 9), 28416
    assert heta.attention_workspace_size(1, 2, 128, grid, win, kk) > 16 << 20
    w = W.scaled(W.WAN21, H=2, d=128, grid=grid, win=win, u_kind="uniform", u_seeds=(5,))
    q, k, v = W.make_qkv(w)
    Q, K, V = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    dense, _, _, _ = heta.route(to_dev(W.make_u(w)), kk)
    want = from_dev_bf16(heta.attention(Q, K, V, grid, win, dense))
    out = torch.full_like(Q, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = fn(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
            ctypes.c_void_p(V.data_ptr()), 1, 2, 128, grid[0], grid[1], grid[2],
            win[0], win[1], win[2], ctypes.c_float(1.0 / math.sqrt(128)),
            ctypes.c_void_p(dense.data_ptr()), kk, ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(st.data_ptr()), stream)
    assert rc == heta.HETA_OK, heta.status_string(rc)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = from_dev_bf16(out)
    assert np.all(np.isfinite(got))
    err = np.abs(got - want)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    _against_oracle(w, q, k, v, dense.cpu().numpy(), got, 4096, 7)


def test_binding_wrapper_matches_workspace_entry_point(gpu_lib):
    """The Python binding's attention_noalloc passes its arguments to the same
    entry point: bit for bit heta_attention's output where both plan the same
    work."""
    import torch
    heta = gpu_lib
    w = W.scaled(W.WAN21, H=2, d=128, grid=(8, 16, 24), win=(3, 9, 9), u_kind="uniform",
                 u_seeds=(11,))
    q, k, v = W.make_qkv(w)
    Q, K, V = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    kk = heta.dense_count(w.N, 0.2)
    dense, _, _, _ = heta.route(to_dev(W.make_u(w)), kk)
    want = from_dev_bf16(heta.attention(Q, K, V, w.grid, w.win, dense))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = from_dev_bf16(heta.attention_noalloc(Q, K, V, w.grid, w.win, dense, status=st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(got, want)
