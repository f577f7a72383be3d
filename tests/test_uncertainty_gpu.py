"""heta_uncertainty (Eq. (7) head) against the oracle, and the full step.

Head tolerance: |u_gpu - u_oracle| <= 1e-5 * (1 + |u|) (fp32 accumulation of
C products against fp64).  The full step (head -> route -> attention) checks
routing bit-exact on the u the GPU produced, as the path consumes it.
"""
import numpy as np
import pytest

import oracle
from helpers import assert_close, from_dev_bf16, sample_rows, to_dev, to_dev_bf16
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def check_head(heta, X_bits, w, bias):
    import torch
    u = heta.uncertainty(to_dev_bf16(X_bits), to_dev(w), bias)
    torch.cuda.synchronize()
    got = u.cpu().numpy()
    want = oracle.uncertainty(W.bf16_to_f32(X_bits), w, bias)
    assert np.all(got >= 0)
    assert np.max(np.abs(got - want) / (1 + np.abs(want))) <= 1e-5
    return got


@pytest.mark.parametrize("B,N,C", [(1, 1, 8), (3, 1000, 96), (2, 777, 1536), (1, 64, 16384),
                                   (2, 300, 3072),
                                   # C = 256 U: each lane's weights in registers
                                   (1, 1, 256), (3, 5, 512), (2, 1001, 768), (1, 4000, 1024),
                                   (2, 333, 1280), (1, 2500, 1536), (1, 97, 1792),
                                   (2, 150, 2048), (1, 1201, 2304), (1, 60, 2560),
                                   (3, 211, 2816), (1, 3000, 3072), (1, 40, 3328),
                                   (2, 1234, 1544)])
def test_head_shapes(gpu_lib, B, N, C):
    rng = np.random.default_rng(B * N + C)
    X = W.bf16_bits(rng.standard_normal((B, N, C), dtype=np.float32))
    w = (rng.standard_normal(C) / np.sqrt(C)).astype(np.float32)
    check_head(gpu_lib, X, w, 0.1)


def test_head_full_batched_shape(gpu_lib):
    X, w = W.make_head(W.BATCHED)
    check_head(gpu_lib, X, w, 0.0)


def test_full_step_batched(gpu_lib):
    """X -> u (head) -> route on the GPU u -> attention, at the B=2 Wan2.1 shape."""
    import torch
    wl = W.BATCHED
    X, w = W.make_head(wl)
    u_dev = gpu_lib.uncertainty(to_dev_bf16(X), to_dev(w), 0.0)
    k = gpu_lib.dense_count(wl.N, wl.rho)
    dense, local, _, _ = gpu_lib.route(u_dev, k)
    q, kk, v = W.make_qkv(wl)
    Qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(kk), to_dev_bf16(v)
    out = torch.full_like(Qd, float("nan"))
    gpu_lib.attention(Qd, Kd, Vd, wl.grid, wl.win, dense, out=out)
    torch.cuda.synchronize()
    u_gpu = u_dev.cpu().numpy()
    od, ol, _ = oracle.route(u_gpu, k)
    assert np.array_equal(dense.cpu().numpy(), od)
    assert np.array_equal(local.cpu().numpy(), ol)
    # diagnostic: routing on the oracle's fp64 u may flip a few boundary tokens
    u_ref = oracle.uncertainty(W.bf16_to_f32(X), w, 0.0).astype(np.float32)
    od_ref, _, _ = oracle.route(u_ref, k)
    flips = sum(len(set(od[b].tolist()) ^ set(od_ref[b].tolist())) for b in range(wl.B))
    assert flips <= 0.01 * wl.B * k
    got = from_dev_bf16(out).reshape(-1, wl.d)
    assert not np.isnan(got).any()
    rows = sample_rows(np.random.default_rng(1), wl.B, wl.H, wl.N, wl.grid, wl.win, od, 800)
    want = oracle.attention_rows(W.bf16_to_f32(q), W.bf16_to_f32(kk), W.bf16_to_f32(v),
                                 wl.grid, wl.win, od, rows)
    assert_close(got[rows], want, "full step")
