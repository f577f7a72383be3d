"""Shared test helpers: host<->device conversion and parity metrics.

Holds none of the method's arithmetic; the oracle computes every expected
value and the CUDA library every observed one.
"""
import numpy as np

from uncertainty_routed_heterogeneous_b200 import workloads as W

# Output tolerance for bf16 inputs, fp32 accumulation and a bf16 output,
# against the fp64 oracle on the same bf16-rounded inputs.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t):
    import torch
    return W.bf16_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def sample_rows(rng, B, H, N, grid, win, dense, n_random):
    """Flat row ids: random rows plus every border class and the first/last dense rows."""
    T, Hg, Wg = grid
    rows = set(int(r) for r in rng.choice(B * H * N, size=min(n_random, B * H * N),
                                          replace=False))
    edges = []
    for t in sorted({0, 1, T // 2, T - 2, T - 1}):
        for h in sorted({0, win[1] // 2, Hg // 2, Hg - 1 - win[1] // 2, Hg - 1}):
            for w in sorted({0, win[2] // 2, Wg // 2, Wg - 1 - win[2] // 2, Wg - 1}):
                if 0 <= t < T and 0 <= h < Hg and 0 <= w < Wg:
                    edges.append((t * Hg + h) * Wg + w)
    for b in range(B):
        for h in (0, H - 1):
            base = (b * H + h) * N
            rows.update(base + i for i in edges)
            d = dense[b]
            if d.size:
                rows.update(base + int(i) for i in d[:3])
                rows.update(base + int(i) for i in d[-3:])
    return np.array(sorted(rows), np.int64)


def assert_close(got, want, what=""):
    err = np.abs(got.astype(np.float64) - want)
    assert np.all(np.isfinite(got)), "%s: non-finite output rows" % what
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, "%s: max %.3g mean %.3g" % (what, mx, mean)
    return mx, mean
