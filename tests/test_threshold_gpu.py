"""Routing by the paper's own rule T = mu + c*sigma, and attention on its
per-sample counts, on the GPU against the fp64 oracle.

"Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion", §3.2.2 Eq. (11)-(12): u_i >= T goes dense.  Both sides compute
mu, sigma and T in fp64 but sum in different orders, so T agrees to ~1e-15
relative and a u inside that band may land on either side.  The checks: T
within 1e-12 (relative) of the oracle's; the GPU's dense set is exactly
{u >= T_gpu} (its own threshold, compared in fp64); outside the band it is
the oracle's set; counts, complements and masks are consistent.  Attention
on those sets: max abs <= 2e-2 and mean abs <= 2e-3 against fp64.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from helpers import assert_close, from_dev_bf16, sample_rows, to_dev, to_dev_bf16
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu

BAND = 1e-9


def check_threshold(heta, u, c):
    import torch
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    counts, dense, local, thresh, mask = heta.route_threshold(
        to_dev(u), c, want_thresh=True, want_mask=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    counts, dense, local = counts.cpu().numpy(), dense.cpu().numpy(), local.cpu().numpy()
    thresh, mask = thresh.cpu().numpy(), mask.cpu().numpy()
    oc, od, ol, ot, om = oracle.route_threshold(u, c)
    B, N = u.shape
    assert np.allclose(thresh, ot, rtol=1e-12, atol=1e-300)
    u64 = u.astype(np.float64)
    for b in range(B):
        got = dense[b, :counts[b]]
        assert np.array_equal(got, np.nonzero(u64[b] >= thresh[b])[0])
        band = np.nonzero(np.abs(u64[b] - ot[b]) <= BAND * max(1.0, abs(ot[b])))[0]
        assert np.array_equal(np.setdiff1d(got, band), np.setdiff1d(od[b, :oc[b]], band))
        assert np.array_equal(local[b, :N - counts[b]], np.setdiff1d(np.arange(N), got))
        assert np.array_equal(mask[b] == 0, np.isin(np.arange(N), got))
    return counts, dense


@pytest.mark.parametrize("c", [-0.5, 0.0, 0.9, 2.0])
@pytest.mark.parametrize("kind", ["gauss", "uniform", "smooth", "clustered"])
def test_threshold_route_matches_oracle(gpu_lib, kind, c):
    rng = np.random.default_rng(21)
    if kind == "gauss":
        u = rng.standard_normal((3, 32760)).astype(np.float32)
    elif kind == "uniform":
        u = rng.random((2, 27280), dtype=np.float32)
    else:
        u = W.make_u(dataclasses.replace(W.WAN21, B=2, u_kind=kind, u_seeds=(2, 6)))
    check_threshold(gpu_lib, u, c)


def test_threshold_route_ragged_rows(gpu_lib):
    """N = 1001: rows start off the 16-byte grid (B > 1) and end in a partial
    warp segment."""
    u = np.random.default_rng(3).standard_normal((5, 1001)).astype(np.float32)
    for c in (0.0, 0.9):
        check_threshold(gpu_lib, u, c)


def test_threshold_route_special_cases(gpu_lib):
    import torch
    heta = gpu_lib
    # sigma = 0: T equals every u, all dense; max size
    counts, _ = check_threshold(heta, np.full((1, 53248), 0.75, np.float32), 1.0)
    assert counts.tolist() == [53248]
    # one token
    counts, _ = check_threshold(heta, np.array([[0.5]], np.float32), 0.0)
    assert counts.tolist() == [1]
    # a huge c sends nothing dense, a very negative one everything
    u = np.random.default_rng(4).random((2, 4096), dtype=np.float32)
    assert check_threshold(heta, u, 50.0)[0].tolist() == [0, 0]
    assert check_threshold(heta, u, -50.0)[0].tolist() == [4096, 4096]
    # NaN is reported
    bad = u.copy()
    bad[1, 77] = np.nan
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    heta.route_threshold(to_dev(bad), 0.9, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == heta.HETA_ERR_NONFINITE


def test_threshold_route_is_repeatable(gpu_lib):
    import torch
    u = to_dev(W.make_u(W.WAN21))
    a = [t.clone() for t in gpu_lib.route_threshold(u, 0.9, want_thresh=True)[:4]]
    b = gpu_lib.route_threshold(u, 0.9, want_thresh=True)[:4]
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def run_counts(heta, w, c, n_sample=None, seed=0):
    """Attention on the threshold routing of w's u, per-sample counts on the
    device, against the oracle run sample by sample on the same sets."""
    import torch
    q, k, v = W.make_qkv(w)
    u = W.make_u(w)
    Qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    counts, dense, _, _, _ = heta.route_threshold(to_dev(u), c)
    out = torch.full_like(Qd, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    heta.attention_counts(Qd, Kd, Vd, w.grid, w.win, dense, counts, out=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = from_dev_bf16(out)
    assert not np.isnan(got).any(), "rows left unwritten"
    cnt, idx = counts.cpu().numpy(), dense.cpu().numpy()
    qf, kf, vf = W.bf16_to_f32(q), W.bf16_to_f32(k), W.bf16_to_f32(v)
    errs = []
    for b in range(w.B):
        d_b = idx[b:b + 1, :cnt[b]]
        if n_sample is None:
            rows = np.arange(w.H * w.N, dtype=np.int64)
        else:
            rows = sample_rows(np.random.default_rng(seed + b), 1, w.H, w.N, w.grid, w.win,
                               d_b, n_sample)
        want = oracle.attention_rows(qf[b:b + 1], kf[b:b + 1], vf[b:b + 1], w.grid, w.win,
                                     d_b, rows)
        errs.append(assert_close(got[b].reshape(-1, w.d)[rows], want, "%s b=%d" % (w.name, b)))
    return cnt, errs


@pytest.mark.parametrize("c", [-0.3, 0.9, 1.8, 50.0])
def test_attention_counts_all_rows(gpu_lib, c):
    """Two samples with different counts; c = 50 leaves both with none."""
    w = dataclasses.replace(W.scaled(W.WAN21, B=2, H=2, grid=(5, 12, 20), u_kind="clustered",
                                     u_seeds=(3, 8)), name="counts-b2")
    cnt, _ = run_counts(gpu_lib, w, c)
    if c == 50.0:
        assert cnt.tolist() == [0, 0]
    else:
        assert cnt[0] != cnt[1]


def test_attention_counts_d64_ragged(gpu_lib):
    w = dataclasses.replace(W.scaled(W.WAN21, B=3, H=3, d=64, grid=(3, 17, 19), win=(3, 5, 7),
                                     u_kind="uniform", u_seeds=(9, 10, 11)), name="counts-d64")
    run_counts(gpu_lib, w, 0.4)


def test_attention_counts_full_size_sampled(gpu_lib):
    """The Wan2.1 shape at the paper's c = 0.9 (about 18% dense)."""
    cnt, _ = run_counts(gpu_lib, W.WAN21, 0.9, n_sample=1200)
    assert 0.1 < cnt[0] / W.WAN21.N < 0.3


@pytest.mark.parametrize("N", [7, 1001, 32760, 53248])
def test_threshold_cluster_and_single_cta_agree(gpu_lib, N):
    """Up to eight samples a call split each sample over a cluster of CTAs,
    more take one CTA each; both sum the same eight slices in the same order,
    so the same rows give bit-identical T, counts and lists in a call of 8
    samples and in a call of 12 (and the oracle's, outside the rounding band)."""
    import torch
    heta = gpu_lib
    u = np.random.default_rng(N).standard_normal((12, N)).astype(np.float32)
    c12, d12, l12, t12, _ = heta.route_threshold(to_dev(u), 0.9, want_thresh=True)
    c8, d8, l8, t8, _ = heta.route_threshold(to_dev(u[:8].copy()), 0.9, want_thresh=True)
    torch.cuda.synchronize()
    assert np.array_equal(t8.cpu().numpy(), t12.cpu().numpy()[:8])
    assert np.array_equal(c8.cpu().numpy(), c12.cpu().numpy()[:8])
    c = c8.cpu().numpy()
    for b in range(8):
        assert np.array_equal(d8[b, :c[b]].cpu().numpy(), d12[b, :c[b]].cpu().numpy())
        assert np.array_equal(l8[b, :N - c[b]].cpu().numpy(), l12[b, :N - c[b]].cpu().numpy())
    check_threshold(heta, u, 0.9)
    check_threshold(heta, u[:8].copy(), 0.9)


@pytest.mark.parametrize("N,B", [(75600, 1), (75600, 9), (8 * 49152, 2)])
def test_threshold_above_one_cta(gpu_lib, N, B):
    """Samples above one SM's shared memory (53248 tokens; the 720p Wan latent
    has 75600) take the cluster kernel for any batch size."""
    rng = np.random.default_rng(N - B)
    u = rng.standard_normal((B, N)).astype(np.float32)
    for c in (0.0, 0.9):
        check_threshold(gpu_lib, u, c)
