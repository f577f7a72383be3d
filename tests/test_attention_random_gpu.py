"""Randomised parity sweep of heta_attention / heta_attention_counts.

"Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion", §3.1.1 Eq. (2)-(3) and §3.2.2 Eq. (13): every output row is
dense attention over all N keys (rows of the dense set) or attention over
the row's clamped 3D window (the others).  Sixty seeded configurations draw
the grid (1-10 x 1-24 x 1-40 tokens, so down to single-token axes and grids
smaller than one key sub-tile), an odd window per axis up to the grid, the
head dimension (64 or 128), B and H (1-3), and either a top-k routing with a
random rho (including 0 and 1) or per-sample dense counts with a random
capacity.  Q/K/V are iid N(0,1) rounded to bf16, the inputs the tolerance is
stated for; every row of every sample is compared with the fp64 oracle.
"""
import numpy as np
import pytest

import oracle
from helpers import MAX_ABS, MEAN_ABS, from_dev_bf16, to_dev, to_dev_bf16
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _config(rng):
    while True:
        grid = (int(rng.integers(1, 11)), int(rng.integers(1, 25)), int(rng.integers(1, 41)))
        N = grid[0] * grid[1] * grid[2]
        if N <= 6000:
            break
    win = tuple(int(rng.choice(np.arange(1, g + 1, 2))) for g in grid)
    return dict(grid=grid, N=N, win=win, d=int(rng.choice([64, 128])),
                B=int(rng.integers(1, 4)), H=int(rng.integers(1, 4)),
                counts=bool(rng.random() < 0.35))


@pytest.mark.parametrize("case", range(60))
def test_attention_random_configs(gpu_lib, case):
    import torch
    heta = gpu_lib
    rng = np.random.default_rng(1000 + case)
    c = _config(rng)
    B, H, N, d, grid, win = c["B"], c["H"], c["N"], c["d"], c["grid"], c["win"]
    bits = [W.bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32)) for _ in range(3)]
    Qf, Kf, Vf = (W.bf16_to_f32(a) for a in bits)
    Q, K, V = (to_dev_bf16(a) for a in bits)
    if not c["counts"]:
        rho = float(rng.choice([0.0, 1.0, rng.random()]))
        k = heta.dense_count(N, rho)
        dense, _, _, _ = heta.route(to_dev(rng.standard_normal((B, N)).astype(np.float32)), k)
        out = heta.attention(Q, K, V, grid, win, dense)
        dn = dense.cpu().numpy()
        lists = [dn[b] for b in range(B)]
    else:
        cap = int(rng.integers(1, N + 1)) if rng.random() < 0.5 else N
        counts = rng.integers(0, cap + 1, B).astype(np.int32)
        dl = np.zeros((B, cap), np.int32)
        lists = []
        for b in range(B):
            sel = np.sort(rng.choice(N, size=int(counts[b]), replace=False)).astype(np.int32)
            dl[b, :counts[b]] = sel
            lists.append(sel)
        out = heta.attention_counts(Q, K, V, grid, win, to_dev(dl), to_dev(counts))
    torch.cuda.synchronize()
    got = from_dev_bf16(out)
    assert np.all(np.isfinite(got)), "rows left unwritten"
    for b in range(B):
        want = oracle.attention(Qf[b:b + 1], Kf[b:b + 1], Vf[b:b + 1], grid, win,
                                lists[b].reshape(1, -1))
        err = np.abs(got[b:b + 1].astype(np.float64) - want)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (c, b, err.max(), err.mean())
