"""Pins for the fp64 oracle: each checks it against something other than itself.

Sources ("Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion"): Eq. (2) dense attention, Eq. (3) local attention, Eq. (7)
uncertainty u_i >= 0, Eq. (11)-(12) routing, Eq. (13) the mix, Eq. (14) rho.

What pins what:
  * dense count  -- exact decimal arithmetic (fractions.Fraction) and the
                    hand-worked table in golden/dense_count.txt
  * window       -- hand-worked starts (golden/window_starts.txt), and an
                    independent definition: the in-grid run of width w that
                    holds p and whose centre is nearest p (brute force)
  * route        -- hand-worked tie cases (golden/route_ties.txt), Python's own
                    sort on (-u, i), and the complete characterisation of a
                    top-k set with index tie-break
  * threshold    -- hand-worked mu + c*sigma cases (golden/route_threshold.txt),
                    numpy's mean/std (ddof=0) in fp64, the Gaussian tail
                    fraction 1 - Phi(c), shift/scale invariance, u == T dense
  * swap         -- Philox4x32-10 known-answer vectors (golden/philox_kat.txt),
                    a brute-force restatement on small inputs (sorting the
                    draws), set sizes and identities, and the coverage
                    1 - (1 - s/(N-k))^30 over 30 blocks
  * attention    -- torch's scaled_dot_product_attention in fp64 (a library
                    routine) with no mask (rho = 1) and with a boolean window
                    mask built from the independent window definition (rho=0);
                    the mix row by row (Eq. (13)); constant-V and zero-K closed
                    forms
  * head         -- numpy's logaddexp(0, z) on a library matmul in fp64;
                    softplus(0) = ln 2; a one-hot weight selects a column
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from uncertainty_routed_heterogeneous_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# helpers that are independent of the oracle
# --------------------------------------------------------------------------


def nearest_centred_start(p, extent, w):
    """Among in-grid runs of width w that contain p, the one centred nearest p."""
    cands = [s for s in range(0, extent - w + 1) if s <= p < s + w]
    return min(cands, key=lambda s: abs(s + (w - 1) / 2.0 - p))


def window_mask(grid, win):
    """[N,N] boolean: key j in the window of query i (independent definition)."""
    T, H, Wd = grid
    N = T * H * Wd
    coords = [(i // (H * Wd), (i // Wd) % H, i % Wd) for i in range(N)]
    starts = [(nearest_centred_start(t, T, win[0]),
               nearest_centred_start(h, H, win[1]),
               nearest_centred_start(w, Wd, win[2])) for (t, h, w) in coords]
    m = np.zeros((N, N), bool)
    for i in range(N):
        st, sh, sw = starts[i]
        for j in range(N):
            t, h, w = coords[j]
            m[i, j] = (st <= t < st + win[0] and sh <= h < sh + win[1]
                       and sw <= w < sw + win[2])
    return m


def sdpa64(Q, K, V, mask=None, scale=None):
    q = torch.from_numpy(np.asarray(Q, np.float64))
    k = torch.from_numpy(np.asarray(K, np.float64))
    v = torch.from_numpy(np.asarray(V, np.float64))
    am = None if mask is None else torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=am, scale=scale).numpy()


def random_qkv(rng, B, H, N, d):
    f = lambda: W.bf16_to_f32(W.bf16_bits(rng.standard_normal((B, H, N, d),
                                                              dtype=np.float32)))
    return f(), f(), f()


# --------------------------------------------------------------------------
# dense count (Eq. (14) rho)
# --------------------------------------------------------------------------


def read_dense_count():
    rows = []
    with open(os.path.join(GOLDEN, "dense_count.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                n, r, k = line.split()
                rows.append((int(n), r, int(k)))
    return rows


@pytest.mark.parametrize("N,rho,k", read_dense_count())
def test_dense_count_golden(N, rho, k):
    assert oracle.dense_count(N, float(rho)) == k


def test_dense_count_matches_exact_decimal():
    for N in list(range(0, 301)) + [1000, 27280, 32760, 65520, 123457]:
        for hundredths in range(0, 101):
            exact = Fraction(hundredths, 100) * N
            want = math.ceil(exact)
            assert oracle.dense_count(N, hundredths / 100.0) == want, (N, hundredths)


def test_dense_count_rejects_bad_rho():
    for bad in (-0.01, 1.01, float("nan")):
        with pytest.raises(oracle.OracleError):
            oracle.dense_count(10, bad)


# --------------------------------------------------------------------------
# window (Eq. (3), reading R3)
# --------------------------------------------------------------------------


def read_window_starts():
    rows = []
    with open(os.path.join(GOLDEN, "window_starts.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.mark.parametrize("row", read_window_starts())
def test_window_golden(row):
    Tg, Hg, Wg, wt, wh, ww, t, h, w, st, sh, sw = row
    i = (t * Hg + h) * Wg + w
    keys = oracle.window((Tg, Hg, Wg), (wt, wh, ww), i)
    want = sorted(((a * Hg + c) * Wg + e) for a in range(st, st + wt)
                  for c in range(sh, sh + wh) for e in range(sw, sw + ww))
    assert list(keys) == want


@pytest.mark.parametrize("extent,w", [(4, 3), (8, 3), (21, 3), (30, 9), (52, 9),
                                      (9, 9), (13, 11), (1, 1), (22, 9)])
def test_window_start_is_nearest_centred_run(extent, w):
    for p in range(extent):
        assert oracle.window_start(p, extent, w) == nearest_centred_start(p, extent, w)


def test_window_properties_wan_grid():
    grid, win = (21, 30, 52), (3, 9, 9)
    rng = np.random.default_rng(11)
    N = 21 * 30 * 52
    for i in list(rng.integers(0, N, 300)) + [0, N - 1]:
        keys = oracle.window(grid, win, int(i))
        assert len(keys) == 243 and len(set(keys.tolist())) == 243
        assert int(i) in set(keys.tolist())
        t, h, w = i // (30 * 52), (i // 52) % 30, i % 52
        if 1 <= t <= 19 and 4 <= h <= 25 and 4 <= w <= 47:  # interior: centred
            assert keys[0] == ((t - 1) * 30 + (h - 4)) * 52 + (w - 4)
            assert keys[-1] == ((t + 1) * 30 + (h + 4)) * 52 + (w + 4)


# --------------------------------------------------------------------------
# route (Eq. (11)-(12), readings R1/R2)
# --------------------------------------------------------------------------


def read_route_ties():
    cases = []
    with open(os.path.join(GOLDEN, "route_ties.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, u, dense, local = [p.strip() for p in line.split("|")]
            u = np.array([int(x, 16) for x in u.split()], np.uint32).view(np.float32)
            cases.append((int(k), u, [int(x) for x in dense.split()],
                          [int(x) for x in local.split()]))
    return cases


@pytest.mark.parametrize("case", read_route_ties())
def test_route_golden(case):
    k, u, dense, local = case
    d, l, m = oracle.route(u[None, :], k)
    assert d[0].tolist() == dense
    assert l[0].tolist() == local
    assert m[0].tolist() == [0 if i in dense else 1 for i in range(u.size)]


def assert_is_topk_with_index_ties(u, k, dense, local):
    """Complete characterisation of the top-k set with index tie-break."""
    N = u.size
    assert dense.size == k and local.size == N - k
    assert np.all(np.diff(dense) > 0) and np.all(np.diff(local) > 0)
    assert sorted(dense.tolist() + local.tolist()) == list(range(N))
    if k == 0 or k == N:
        return
    ud = u[dense].astype(np.float64)
    ul = u[local].astype(np.float64)
    # every dense token beats every local one: larger u, or equal u and smaller index
    lo = ud.min()
    hi = ul.max()
    assert lo >= hi
    if lo == hi:
        tie_d = dense[ud == lo]
        tie_l = local[ul == hi]
        assert tie_d.max() < tie_l.min()


@pytest.mark.parametrize("N,k,kind", [(1, 0, "u"), (1, 1, "u"), (257, 64, "u"),
                                      (1000, 1, "ties"), (4096, 4095, "ties"),
                                      (5000, 1234, "neg"), (32760, 6552, "smooth")])
def test_route_vs_python_sort(N, k, kind):
    rng = np.random.default_rng(N + k)
    if kind == "u":
        u = rng.random(N, dtype=np.float32)
    elif kind == "ties":
        u = rng.integers(0, 7, N).astype(np.float32)
    elif kind == "neg":
        u = rng.standard_normal(N).astype(np.float32)
        u[::17] = -0.0
        u[::19] = 0.0
    else:
        u = W.make_u(W.WAN21)[0]
    d, l, _ = oracle.route(u[None, :], k)
    order = sorted(range(N), key=lambda i: (-float(u[i]), i))
    assert d[0].tolist() == sorted(order[:k])
    assert l[0].tolist() == sorted(order[k:])
    assert_is_topk_with_index_ties(u, k, d[0], l[0])


def test_route_samples_are_independent():
    u = W.make_u(W.BATCHED)
    k = oracle.dense_count(u.shape[1], 0.2)
    d, l, _ = oracle.route(u, k)
    for b in range(2):
        d1, l1, _ = oracle.route(u[b:b + 1], k)
        assert np.array_equal(d[b], d1[0]) and np.array_equal(l[b], l1[0])
    assert not np.array_equal(d[0], d[1])


def test_route_nan_is_an_error():
    u = np.array([[0.1, float("nan"), 0.3]], np.float32)
    with pytest.raises(oracle.OracleError) as e:
        oracle.route(u, 1)
    assert e.value.code == oracle.NONFINITE


# --------------------------------------------------------------------------
# threshold routing, the paper's own rule (Eq. (11)-(12), reading R10)
# --------------------------------------------------------------------------

def read_threshold_golden():
    """golden/route_threshold.txt: u values | c | T | dense ids (worked by hand)."""
    cases = []
    for line in open(os.path.join(GOLDEN, "route_threshold.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        u, c, T, dense = (f.strip() for f in line.split("|"))
        cases.append((np.array([[float(x) for x in u.split()]], np.float32), float(c),
                      float(T), [int(x) for x in dense.split()] if dense else []))
    return cases


@pytest.mark.parametrize("case", read_threshold_golden())
def test_threshold_golden(case):
    u, c, T, dense = case
    counts, d, l, thresh, mask = oracle.route_threshold(u, c)
    assert abs(thresh[0] - T) <= 1e-6 * max(1.0, abs(T))
    assert counts[0] == len(dense)
    assert d[0, :counts[0]].tolist() == dense
    N = u.shape[1]
    assert sorted(d[0, :counts[0]].tolist() + l[0, :N - counts[0]].tolist()) == list(range(N))
    assert all(mask[0, i] == (0 if i in dense else 1) for i in range(N))


def _numpy_threshold_sets(u, c):
    """Independent restatement with numpy's own mean and std in fp64."""
    T = np.mean(u.astype(np.float64), axis=1) + c * np.std(u.astype(np.float64), axis=1, ddof=0)
    return T, u.astype(np.float64) >= T[:, None]


@pytest.mark.parametrize("c", [-0.5, 0.0, 0.9, 2.0])
@pytest.mark.parametrize("kind", ["gauss", "uniform", "smooth"])
def test_threshold_vs_numpy(c, kind):
    rng = np.random.default_rng(7)
    B, N = 3, 4099
    if kind == "gauss":
        u = rng.standard_normal((B, N)).astype(np.float32)
    elif kind == "uniform":
        u = rng.random((B, N), dtype=np.float32)
    else:
        u = np.stack([W.make_u(W.scaled(W.WAN21, grid=(3, 29, 47), u_seeds=(s,)))[0]
                      for s in (1, 2, 3)])
        B, N = u.shape
    counts, d, l, thresh, mask = oracle.route_threshold(u, c)
    T, dense = _numpy_threshold_sets(u, c)
    assert np.allclose(thresh, T, rtol=1e-12, atol=1e-12)
    for b in range(B):
        want = np.nonzero(dense[b])[0]
        # decisions are only uncertain inside the rounding band of T
        band = np.abs(u[b].astype(np.float64) - T[b]) <= 1e-9 * max(1.0, abs(T[b]))
        got = d[b, :counts[b]]
        assert np.array_equal(np.setdiff1d(got, np.nonzero(band)[0]),
                              np.setdiff1d(want, np.nonzero(band)[0]))
        assert np.array_equal(l[b, :N - counts[b]], np.setdiff1d(np.arange(N), got))
        assert np.array_equal(mask[b] == 0, np.isin(np.arange(N), got))


def test_threshold_gaussian_tail_fraction():
    """c = 0.9 on Gaussian u keeps 1 - Phi(0.9) = 0.184 of the tokens dense
    (the paper's rho ~ 0.2 setting), c = 0 half of them."""
    rng = np.random.default_rng(11)
    u = rng.standard_normal((4, 32760)).astype(np.float32)
    for c in (0.0, 0.9, 1.5):
        counts = oracle.route_threshold(u, c)[0]
        tail = 0.5 * math.erfc(c / math.sqrt(2.0))
        # binomial std at N = 32760 is < 0.003; the estimated mu/sigma add less
        assert np.all(np.abs(counts / 32760.0 - tail) < 0.012), (c, counts)


def test_threshold_shift_and_scale_invariant():
    """T moves with an affine map a*u + b (a > 0) and the sets do not change.
    Values on a 1/8 grid keep every step exact in fp32 and fp64."""
    rng = np.random.default_rng(5)
    u = (rng.integers(-64, 64, size=(2, 3001)) / 8.0).astype(np.float32)
    base = oracle.route_threshold(u, 0.7)
    for a, b in ((4.0, 0.0), (1.0, 96.0), (0.5, -3.0)):
        v = (u * np.float32(a) + np.float32(b)).astype(np.float32)
        got = oracle.route_threshold(v, 0.7)
        assert np.array_equal(got[0], base[0])
        assert np.array_equal(got[1], base[1])
        assert np.allclose(got[3], a * base[3] + b, rtol=1e-12)


def test_threshold_constant_u_is_all_dense():
    """sigma = 0 puts T on every u; u == T goes dense (Eq. (12)'s strict <)."""
    u = np.full((2, 777), 0.3125, np.float32)
    counts, d, l, thresh, mask = oracle.route_threshold(u, 1.0)
    assert counts.tolist() == [777, 777]
    assert np.all(thresh == 0.3125)
    assert not mask.any()


def test_threshold_edge_cases():
    empty = np.zeros((2, 0), np.float32)
    counts = oracle.route_threshold(empty, 0.9)[0]
    assert counts.tolist() == [0, 0]
    with pytest.raises(oracle.OracleError) as e:
        oracle.route_threshold(np.array([[0.1, float("nan")]], np.float32), 0.0)
    assert e.value.code == oracle.NONFINITE
    # samples are routed independently
    u = np.stack([np.arange(10, dtype=np.float32), -np.arange(10, dtype=np.float32)])
    counts, d, _, thresh, _ = oracle.route_threshold(u, 0.0)
    assert counts.tolist() == [5, 5]
    assert d[0, :5].tolist() == [5, 6, 7, 8, 9] and d[1, :5].tolist() == [0, 1, 2, 3, 4]
    assert thresh.tolist() == [4.5, -4.5]


# --------------------------------------------------------------------------
# per-block random swap (§3.2.2, App. B Table 8; reading R11)
# --------------------------------------------------------------------------

def read_philox_kat():
    cases = []
    for line in open(os.path.join(GOLDEN, "philox_kat.txt")):
        line = line.split("#")[0].strip()
        if line:
            ctr, key, out = ([int(x, 16) for x in f.split()] for f in line.split("|"))
            cases.append((ctr, key, out))
    return cases


@pytest.mark.parametrize("case", read_philox_kat())
def test_philox_known_answers(case):
    ctr, key, out = case
    assert oracle.philox4x32_10(ctr, key).tolist() == out


def _draws_bruteforce(N, b, block, seed):
    """rho_i for every token, from the oracle's Philox (pinned above)."""
    return [int(oracle.philox4x32_10([i, b, block, 0],
                                     [seed & 0xffffffff, seed >> 32])[0]) for i in range(N)]


@pytest.mark.parametrize("N,k,s", [(40, 12, 5), (33, 16, 16), (64, 1, 1), (50, 30, 0)])
def test_swap_vs_bruteforce(N, k, s):
    rng = np.random.default_rng(N + k)
    u = rng.random((2, N), dtype=np.float32)
    dense, _, _ = oracle.route(u, k)
    seed, block = 0x123456789ABCDEF, 7
    got_d, got_l = oracle.route_swap(dense, N, s, seed, block)
    for b in range(2):
        draw = _draws_bruteforce(N, b, block, seed)
        D = [int(i) for i in dense[b]]
        L = [i for i in range(N) if i not in set(D)]
        out_d = sorted(D, key=lambda i: (draw[i], i))[:s]
        in_l = sorted(L, key=lambda i: (draw[i], i))[:s]
        want = sorted((set(D) - set(out_d)) | set(in_l))
        assert got_d[b].tolist() == want
        assert got_l[b].tolist() == sorted(set(range(N)) - set(want))


def test_swap_identities():
    rng = np.random.default_rng(1)
    u = rng.random((3, 500), dtype=np.float32)
    dense, local, _ = oracle.route(u, 250)
    d0, l0 = oracle.route_swap(dense, 500, 0, 9, 0)
    assert np.array_equal(d0, dense) and np.array_equal(l0, local)
    # s = k = N - k swaps every token
    d1, l1 = oracle.route_swap(dense, 500, 250, 9, 0)
    assert np.array_equal(d1, local) and np.array_equal(l1, dense)
    # s of each: sizes, overlaps, and a different draw per block and per sample
    d2, _ = oracle.route_swap(dense, 500, 35, 9, 0)
    d3, _ = oracle.route_swap(dense, 500, 35, 9, 1)
    for b in range(3):
        assert len(set(d2[b]) & set(dense[b])) == 250 - 35
        assert len(set(d2[b]) - set(dense[b])) == 35
    assert not np.array_equal(d2, d3)
    assert not np.array_equal(np.setdiff1d(d2[0], dense[0]), np.setdiff1d(d2[1], dense[1]))
    with pytest.raises(oracle.OracleError):
        oracle.route_swap(dense, 500, 251, 9, 0)


def test_swap_coverage_over_30_blocks():
    """Table 8's setting: r = 7% of N swapped per block, 30 blocks.  A token
    outside D is drawn with probability p = s/(N-k) per block, so the share
    of them dense at least once is 1 - (1-p)^30 (the paper's 1 - (1-r)^30 =
    0.89 takes p = r); the dense tokens keep their place with probability
    1 - s/k per block."""
    N = 32760
    k = oracle.dense_count(N, 0.2)
    s = min(oracle.dense_count(N, 0.07), k, N - k)
    u = W.make_u(W.WAN21)
    dense, local, _ = oracle.route(u, k)
    seen = np.zeros(N, bool)
    kept = []
    for block in range(30):
        d, _ = oracle.route_swap(dense, N, s, 2024, block)
        seen[d[0]] = True
        kept.append(len(np.intersect1d(d[0], dense[0])) / k)
    p = s / (N - k)
    assert abs(seen[local[0]].mean() - (1 - (1 - p) ** 30)) < 0.01
    assert abs(np.mean(kept) - (1 - s / k)) < 1e-12


# --------------------------------------------------------------------------
# attention (Eq. (2), (3), (13))
# --------------------------------------------------------------------------

TINY_GRID, TINY_WIN = (4, 8, 8), (3, 3, 3)


@pytest.fixture(scope="module")
def tiny_mask():
    return window_mask(TINY_GRID, TINY_WIN)


def test_rho1_is_dense_attention():
    rng = np.random.default_rng(1)
    Q, K, V = random_qkv(rng, 1, 2, 256, 64)
    dense = np.arange(256, dtype=np.int32)[None]
    got = oracle.attention(Q, K, V, TINY_GRID, TINY_WIN, dense)
    want = sdpa64(Q, K, V)
    assert np.max(np.abs(got - want)) < 1e-12


def test_rho0_is_window_attention(tiny_mask):
    rng = np.random.default_rng(2)
    Q, K, V = random_qkv(rng, 1, 2, 256, 64)
    dense = np.zeros((1, 0), np.int32)
    got = oracle.attention(Q, K, V, TINY_GRID, TINY_WIN, dense)
    want = sdpa64(Q, K, V, mask=tiny_mask)
    assert np.max(np.abs(got - want)) < 1e-12


def test_mix_picks_one_computation_per_row(tiny_mask):
    """Eq. (13): each row equals exactly the dense or the local result."""
    wl = W.TINY
    q, k, v = (W.bf16_to_f32(x) for x in W.make_qkv(wl))
    u = W.make_u(wl)
    kk = oracle.dense_count(wl.N, wl.rho)
    dense, local, mask = oracle.route(u, kk)
    got = oracle.attention(q, k, v, wl.grid, wl.win, dense)
    full = sdpa64(q, k, v)
    loc = sdpa64(q, k, v, mask=tiny_mask)
    is_dense = np.zeros(wl.N, bool)
    is_dense[dense[0]] = True
    for h in range(wl.H):
        assert np.max(np.abs(got[0, h, is_dense] - full[0, h, is_dense])) < 1e-12
        assert np.max(np.abs(got[0, h, ~is_dense] - loc[0, h, ~is_dense])) < 1e-12
    # the two computations really differ, so a swapped choice would fail
    assert np.min(np.abs(full - loc).max(axis=-1)) > 1e-3
    assert np.array_equal(mask[0] == 0, is_dense)


def test_rows_api_matches_full(tiny_mask):
    rng = np.random.default_rng(3)
    Q, K, V = random_qkv(rng, 2, 3, 256, 64)
    dense = np.stack([rng.choice(256, 40, replace=False) for _ in range(2)]).astype(np.int32)
    full = oracle.attention(Q, K, V, TINY_GRID, TINY_WIN, dense)
    rows = rng.choice(2 * 3 * 256, 77, replace=False)
    part = oracle.attention_rows(Q, K, V, TINY_GRID, TINY_WIN, dense, rows)
    assert np.array_equal(part, full.reshape(-1, 64)[rows])


def test_closed_forms():
    rng = np.random.default_rng(4)
    Q, K, V = random_qkv(rng, 1, 1, 256, 64)
    dense = np.sort(rng.choice(256, 64, replace=False)).astype(np.int32)[None]
    # V constant per channel -> output equals that constant
    Vc = np.broadcast_to(V[:, :, :1, :], V.shape).copy()
    out = oracle.attention(Q, K, Vc, TINY_GRID, TINY_WIN, dense)
    assert np.max(np.abs(out - Vc[:, :, :1, :])) < 1e-12
    # K = 0 -> uniform weights: mean of V over all keys (dense) / the window (local)
    out = oracle.attention(Q, np.zeros_like(K), V, TINY_GRID, TINY_WIN, dense)
    is_dense = np.zeros(256, bool)
    is_dense[dense[0]] = True
    mean_all = V[0, 0].astype(np.float64).mean(axis=0)
    for i in range(256):
        if is_dense[i]:
            want = mean_all
        else:
            keys = oracle.window(TINY_GRID, TINY_WIN, i)
            want = V[0, 0, keys].astype(np.float64).mean(axis=0)
        assert np.max(np.abs(out[0, 0, i] - want)) < 1e-12


def test_scale_argument():
    rng = np.random.default_rng(5)
    Q, K, V = random_qkv(rng, 1, 1, 64, 64)
    dense = np.arange(64, dtype=np.int32)[None]
    got = oracle.attention(Q, K, V, (1, 8, 8), (1, 3, 3), dense, scale=0.3)
    assert np.max(np.abs(got - sdpa64(Q, K, V, scale=0.3))) < 1e-12


# --------------------------------------------------------------------------
# uncertainty head (Eq. (7), reading R7)
# --------------------------------------------------------------------------


def test_head_vs_library():
    rng = np.random.default_rng(6)
    X = W.bf16_to_f32(W.bf16_bits(rng.standard_normal((2, 300, 96), dtype=np.float32)))
    w = (rng.standard_normal(96) / math.sqrt(96)).astype(np.float32)
    got = oracle.uncertainty(X, w, bias=0.25)
    z = np.einsum("bnc,c->bn", X.astype(np.float64), w.astype(np.float64)) + 0.25
    want = np.logaddexp(0.0, z)
    assert np.max(np.abs(got - want) / (1 + np.abs(want))) < 1e-13
    assert np.all(got >= 0)


def test_head_special_cases():
    rng = np.random.default_rng(7)
    X = rng.standard_normal((1, 50, 32)).astype(np.float32)
    assert np.allclose(oracle.uncertainty(X, np.zeros(32, np.float32)), math.log(2.0),
                       rtol=0, atol=1e-15)
    e = np.zeros(32, np.float32)
    e[5] = 1.0
    got = oracle.uncertainty(X, e, bias=0.0)
    assert np.max(np.abs(got[0] - np.logaddexp(0.0, X[0, :, 5].astype(np.float64)))) < 1e-14
    big = np.full((1, 1, 1), 60.0, np.float32)
    assert abs(oracle.uncertainty(big, np.ones(1, np.float32))[0, 0] - 60.0) < 1e-12
    small = np.full((1, 1, 1), -60.0, np.float32)
    assert abs(oracle.uncertainty(small, np.ones(1, np.float32))[0, 0] - math.exp(-60)) < 1e-36


def test_window_111_local_rows_return_their_own_value():
    """A 1x1x1 neighbourhood holds only the token itself (R3): its softmax has
    one term, so a local row's output is its own v exactly."""
    rng = np.random.default_rng(2)
    grid, win = (2, 4, 5), (1, 1, 1)
    N = 40
    q, k, v = (rng.standard_normal((1, 2, N, 8)).astype(np.float32) for _ in range(3))
    dense = np.array([[3, 17, 30]], np.int32)
    out = oracle.attention(q, k, v, grid, win, dense)
    loc = np.setdiff1d(np.arange(N), dense[0])
    assert np.array_equal(out[0][:, loc], v[0][:, loc].astype(np.float64))
