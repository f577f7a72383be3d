"""The per-block random swap (heta_route_swap) on the GPU against the oracle.

"Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion", §3.2.2 after Eq. (12) and App. B Table 8.  Both sides draw from
Philox4x32-10 with the same counters and key, so the new index lists must
match bit for bit.
"""
import numpy as np
import pytest

import oracle
from helpers import to_dev
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def check(heta, u, k, s, seed, block, in_place=False):
    import torch
    B, N = u.shape
    dense, _, _, _ = heta.route(to_dev(u), k)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    want_d, want_l = oracle.route_swap(dense.cpu().numpy(), N, s, seed, block)
    if in_place:
        local = torch.empty((B, N - k), dtype=torch.int32, device="cuda")
        mask = torch.empty((B, N), dtype=torch.uint8, device="cuda")
        got_d, got_l, mask = heta.route_swap(dense, N, s, seed, block, out=(dense, local, mask),
                                             status=st)
    else:
        got_d, got_l, mask = heta.route_swap(dense, N, s, seed, block, want_mask=True,
                                             status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(got_d.cpu().numpy(), want_d)
    assert np.array_equal(got_l.cpu().numpy(), want_l)
    m = mask.cpu().numpy()
    for b in range(B):
        assert np.array_equal(np.nonzero(m[b] == 0)[0], want_d[b])


@pytest.mark.parametrize("block", [0, 1, 29])
def test_swap_wan21_table8_setting(gpu_lib, block):
    """r = 7% of N per block at the Wan2.1 shape, rho = 0.2, two samples."""
    heta = gpu_lib
    N = W.WAN21.N
    k = heta.dense_count(N, 0.2)
    s = heta.swap_count(N, k, 0.07)
    assert s == 2294
    u = np.stack([W.make_u(W.WAN21)[0], np.random.default_rng(5).random(N, dtype=np.float32)])
    check(heta, u, k, s, seed=0x5EED5EED12345678, block=block)


@pytest.mark.parametrize("N,k,s", [(1001, 300, 77), (4099, 2049, 2050), (53248, 10650, 3728),
                                   (64, 32, 32), (300, 150, 0), (257, 1, 1),
                                   # above one SM's shared memory: draws computed per pass
                                   (53249, 10650, 3728), (75600, 15120, 5292)])
def test_swap_sizes(gpu_lib, N, k, s):
    rng = np.random.default_rng(N)
    u = rng.standard_normal((3, N)).astype(np.float32)
    s = min(s, k, N - k)
    check(gpu_lib, u, k, s, seed=N * 7919, block=3)


def test_swap_in_place(gpu_lib):
    u = np.random.default_rng(8).random((2, 5000), dtype=np.float32)
    check(gpu_lib, u, 1000, 350, seed=1, block=2, in_place=True)


def test_swap_bad_index_is_reported(gpu_lib):
    import torch
    heta = gpu_lib
    d = torch.tensor([[0, 5, 9, 70000]], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    heta.route_swap(d, 100, 2, seed=3, block=0, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == heta.HETA_ERR_INVALID_ARG


@pytest.mark.parametrize("N,k,s,B", [(32760, 6552, 2294, 2), (1001, 300, 77, 3),
                                     (75600, 15120, 5292, 1)])
def test_swap_blocks_matches_one_block_calls(gpu_lib, N, k, s, B):
    """All 30 blocks of a step in one launch (heta_route_swap_blocks) give,
    block for block, the lists of 30 single-block calls; blocks 0 and 29 are
    also checked against the oracle."""
    import torch
    heta = gpu_lib
    rng = np.random.default_rng(N + B)
    u = rng.standard_normal((B, N)).astype(np.float32)
    dense, _, _, _ = heta.route(to_dev(u), k)
    seed, block0, nb = 0xABCDEF0123456789, 5, 30
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    all_d, all_l, all_m = heta.route_swap_blocks(dense, N, s, seed, block0, nb, want_mask=True,
                                                 status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for j in range(nb):
        d1, l1, m1 = heta.route_swap(dense, N, s, seed, block0 + j, want_mask=True)
        assert torch.equal(all_d[j], d1) and torch.equal(all_l[j], l1)
        assert torch.equal(all_m[j], m1)
    dn = dense.cpu().numpy()
    for j in (0, nb - 1):
        want_d, want_l = oracle.route_swap(dn, N, s, seed, block0 + j)
        assert np.array_equal(all_d[j].cpu().numpy(), want_d)
        assert np.array_equal(all_l[j].cpu().numpy(), want_l)
