"""heta_route on the GPU against the oracle: index lists must be bit-exact.

"Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion", §3.2.2 Eq. (11)-(12), in top-k form (k = ceil(rho*N) per sample,
Eq. (14)); ties go to the smaller token index.
"""
import numpy as np
import pytest

import oracle
from helpers import to_dev
from test_oracle_pins import read_route_ties
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def check_route(heta, u, k):
    import torch
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    d, l, th, m = heta.route(to_dev(u), k, want_thresh=True, want_mask=True, status=st)
    # the same call without the optional outputs takes the kernel's other
    # compaction path (no mask stores)
    d2, l2, _, _ = heta.route(to_dev(u), k, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    od, ol, om = oracle.route(u, k)
    assert np.array_equal(d.cpu().numpy(), od)
    assert np.array_equal(l.cpu().numpy(), ol)
    assert np.array_equal(m.cpu().numpy(), om)
    assert np.array_equal(d2.cpu().numpy(), od)
    assert np.array_equal(l2.cpu().numpy(), ol)
    th = th.cpu().numpy()
    for b in range(u.shape[0]):
        if k == 0:
            assert th[b] == np.inf
        else:
            assert th[b] == u[b, od[b]].min()


@pytest.mark.parametrize("name", ["tiny-4x8x8", "wan2.1-1.3b-21x30x52", "wan2.2-5b-31x22x40",
                                  "wan2.1-1.3b-batched-b2", "wan2.1-1.3b-720p-21x45x80"])
def test_route_workloads(gpu_lib, name):
    w = W.ALL[name]
    u = W.make_u(w)
    check_route(gpu_lib, u, gpu_lib.dense_count(w.N, w.rho))


@pytest.mark.parametrize("kind", ["uniform", "clustered"])
@pytest.mark.parametrize("rho", W.SWEEP_RHOS)
def test_route_sweep(gpu_lib, kind, rho):
    w = W.sweep(rho, kind)
    check_route(gpu_lib, W.make_u(w), gpu_lib.dense_count(w.N, rho))


@pytest.mark.parametrize("case", read_route_ties())
def test_route_golden_ties(gpu_lib, case):
    k, u, _, _ = case
    check_route(gpu_lib, u[None, :].copy(), k)


@pytest.mark.parametrize("k", [0, 1, 2, 6551, 32759, 32760])
def test_route_extreme_k(gpu_lib, k):
    u = W.make_u(W.WAN21)
    check_route(gpu_lib, u, k)


@pytest.mark.parametrize("N,B,kind", [(1, 1, "u"), (33, 2, "u"), (1001, 3, "u"),
                                      (53248, 1, "ties"), (32760, 2, "equal"),
                                      (4097, 2, "signed_zero"), (5000, 1, "denormal"),
                                      (1024, 4, "inf"), (3001, 3, "offset"),
                                      (2050, 2, "wide"), (53248, 2, "normal"),
                                      (777, 5, "few_values")])
def test_route_edge_inputs(gpu_lib, N, B, kind):
    rng = np.random.default_rng(N * 7 + B)
    if kind == "u":
        u = rng.random((B, N), dtype=np.float32)
    elif kind == "ties":
        u = rng.integers(0, 7, (B, N)).astype(np.float32)
    elif kind == "equal":
        u = np.full((B, N), 0.5, np.float32)
    elif kind == "signed_zero":
        u = rng.choice(np.array([-0.0, 0.0, 1.0, -1.0], np.float32), (B, N))
    elif kind == "denormal":
        u = (rng.integers(-20, 20, (B, N)) * np.float32(1e-45)).astype(np.float32)
    elif kind == "inf":
        u = rng.choice(np.array([np.inf, -np.inf, 0.0, 3.0], np.float32), (B, N))
    elif kind == "offset":
        # far from 0 relative to the spread: the two-rounding bucket form
        u = (np.float32(1e6) + rng.random((B, N), dtype=np.float32)).astype(np.float32)
    elif kind == "wide":
        # magnitudes from 1e-30 to 1e30 of both signs
        u = (rng.choice([-1.0, 1.0], (B, N)) * 10.0 ** rng.uniform(-30, 30, (B, N)))
        u = u.astype(np.float32)
    elif kind == "normal":
        u = rng.standard_normal((B, N)).astype(np.float32)
    else:
        # a handful of distinct values: buckets with hundreds of equal tokens
        u = rng.choice(np.array([0.1, 0.25, 0.5, 0.75], np.float32), (B, N))
    for rho in (0.0, 0.2, 0.5, 1.0):
        check_route(gpu_lib, u, gpu_lib.dense_count(N, rho))


def test_route_nan_sets_status(gpu_lib):
    import torch
    u = np.random.default_rng(0).random((2, 1000), dtype=np.float32)
    u[1, 17] = np.nan
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu_lib.route(to_dev(u), 100, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == gpu_lib.HETA_ERR_NONFINITE


def test_route_many_samples(gpu_lib):
    """More samples than SMs: each CTA walks several samples (prefetching the
    next one into L2), some rows 16-byte aligned and some not (N odd)."""
    rng = np.random.default_rng(99)
    for N in (1000, 1001):
        u = rng.standard_normal((300, N)).astype(np.float32)
        check_route(gpu_lib, u, gpu_lib.dense_count(N, 0.3))


@pytest.mark.parametrize("N", [33, 4097, 32760, 53248])
def test_route_cluster_and_single_cta_agree(gpu_lib, N):
    """Up to eight samples a call split each sample over a cluster of CTAs;
    more samples take one CTA each.  The same rows routed in a call of 8
    samples and in a call of 9 give the same lists, and the oracle's."""
    rng = np.random.default_rng(N)
    u = rng.standard_normal((9, N)).astype(np.float32)
    u[3] = rng.integers(0, 5, N).astype(np.float32)  # heavy ties: the key select
    k = gpu_lib.dense_count(N, 0.2)
    d9, l9, _, _ = gpu_lib.route(to_dev(u), k)
    d8, l8, _, _ = gpu_lib.route(to_dev(u[:8].copy()), k)
    od, ol, _ = oracle.route(u, k)
    assert np.array_equal(d9.cpu().numpy(), od) and np.array_equal(l9.cpu().numpy(), ol)
    assert np.array_equal(d8.cpu().numpy(), od[:8]) and np.array_equal(l8.cpu().numpy(), ol[:8])


@pytest.mark.parametrize("N,B", [(53249, 1), (75600, 1), (75600, 9), (75601, 3),
                                 (8 * 49152, 1)])
def test_route_above_one_cta(gpu_lib, N, B):
    """Samples too large for one SM's shared memory (53248 tokens) take the
    cluster kernel whatever the batch size: the 720p Wan latent (75600), a
    ragged size, more samples than one cluster a call, and the largest N."""
    rng = np.random.default_rng(N + B)
    u = rng.standard_normal((B, N)).astype(np.float32)
    if B > 1:
        u[1] = rng.integers(0, 9, N).astype(np.float32)  # heavy ties: the key select
    for rho in (0.0, 0.2, 1.0):
        check_route(gpu_lib, u, gpu_lib.dense_count(N, rho))


def test_route_above_the_limit_is_unsupported(gpu_lib):
    import torch
    u = torch.zeros((1, 8 * 49152 + 1), dtype=torch.float32, device="cuda")
    with pytest.raises(gpu_lib.HetaError) as e:
        gpu_lib.route(u, 10)
    assert e.value.code == gpu_lib.HETA_ERR_UNSUPPORTED
