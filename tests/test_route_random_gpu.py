"""Randomised parity sweep of heta_route against the oracle (bit-exact lists).

"Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion", §3.2.2 Eq. (11)-(12), in top-k form.  Eighty seeded calls draw
B from 1 to 12 (up to 8 samples take the cluster kernel, more the one-CTA
kernel), N from 1 to 6000 (ragged rows, so samples start off 16-byte
boundaries), k anywhere in [0, N], and u from distributions that steer the
kernels down each path: continuous values (the bucket select), narrow
ranges far from zero (its two-rounding bucket form), a few repeated values
(heavy ties: the key select), signed zeros, infinities, and values spanning
many binades.  Lists, masks and thresholds must equal the oracle's.
"""
import numpy as np
import pytest

import oracle
from helpers import to_dev

pytestmark = pytest.mark.gpu


def _u(rng, B, N):
    kind = int(rng.integers(0, 7))
    if kind == 0:
        return rng.standard_normal((B, N)).astype(np.float32)
    if kind == 1:
        return rng.random((B, N), dtype=np.float32)
    if kind == 2:
        return (np.float32(5e5) + rng.random((B, N), dtype=np.float32)).astype(np.float32)
    if kind == 3:
        return rng.integers(-3, 4, (B, N)).astype(np.float32)
    if kind == 4:
        return rng.choice(np.array([-0.0, 0.0, 0.5, -0.5], np.float32), (B, N))
    if kind == 5:
        u = rng.standard_normal((B, N)).astype(np.float32)
        u[rng.random((B, N)) < 0.05] = np.inf
        u[rng.random((B, N)) < 0.05] = -np.inf
        return u
    s = rng.choice([-1.0, 1.0], (B, N)) * 10.0 ** rng.uniform(-20, 20, (B, N))
    return s.astype(np.float32)


@pytest.mark.parametrize("case", range(80))
def test_route_random(gpu_lib, case):
    import torch
    heta = gpu_lib
    rng = np.random.default_rng(5000 + case)
    B = int(rng.integers(1, 13))
    N = int(rng.integers(1, 6001))
    k = int(rng.choice([0, N, int(rng.integers(0, N + 1))]))
    u = _u(rng, B, N)
    d, l, th, m = heta.route(to_dev(u), k, want_thresh=True, want_mask=True)
    d2, l2, _, _ = heta.route(to_dev(u), k)
    torch.cuda.synchronize()
    od, ol, om = oracle.route(u, k)
    assert np.array_equal(d.cpu().numpy(), od)
    assert np.array_equal(l.cpu().numpy(), ol)
    assert np.array_equal(m.cpu().numpy(), om)
    assert np.array_equal(d2.cpu().numpy(), od)
    assert np.array_equal(l2.cpu().numpy(), ol)
    th = th.cpu().numpy()
    for b in range(B):
        if k == 0:
            assert th[b] == np.inf
        else:
            assert th[b] == u[b, od[b]].min()
