"""The C-ABI library builds, loads and exports what include/heta.h declares.

CPU only: no call here reaches the GPU.  The validation cases return from the
host-side checks before any CUDA call is made.
"""
import ctypes
import os
import re

import pytest

import oracle
import uncertainty_routed_heterogeneous_b200 as heta
from uncertainty_routed_heterogeneous_b200 import build as heta_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    heta_build.build()
    return heta.load()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"HETA_API\s+[\w\s\*]*?\b(heta_\w+)\s*\(", text))
    return names


def test_header_declares_the_three_path_calls():
    names = declared_symbols()
    assert {"heta_route", "heta_attention", "heta_uncertainty", "heta_dense_count",
            "heta_status_string", "heta_version", "heta_attention_workspace_size",
            "heta_route_threshold", "heta_attention_counts", "heta_route_swap",
            "heta_route_swap_blocks", "heta_attention_counts_workspace_size"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(6):
        s = heta.status_string(code)
        assert s and s != "unknown status"
    assert heta.status_string(99) == "unknown status"
    assert lib.heta_version() >> 16 == 1


def test_dense_count_matches_oracle(lib):
    for N in (0, 1, 7, 10, 30, 100, 256, 27280, 32760):
        for rho in (0.0, 0.01, 0.05, 0.07, 0.1, 0.2, 0.25, 0.3, 0.35, 0.5, 0.99, 1.0):
            assert heta.dense_count(N, rho) == oracle.dense_count(N, rho), (N, rho)
    with pytest.raises(heta.HetaError):
        heta.dense_count(10, 1.5)
    with pytest.raises(heta.HetaError):
        heta.dense_count(-1, 0.5)


def test_host_validation_returns_before_any_launch(lib):
    N = None
    # B = 0 / k > N / null pointers are rejected on the host
    assert lib.heta_route(N, 0, 10, 1, N, N, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    assert lib.heta_route(N, 1, 10, 11, N, N, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    assert lib.heta_route(N, 1, 10, 2, N, N, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)
    assert lib.heta_route(fake, 1, 8 * 49152 + 1, 2, fake, fake, N, N, N, N) == \
        heta.HETA_ERR_UNSUPPORTED
    # misaligned pointer
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert lib.heta_route(odd, 1, 10, 2, fake, fake, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    args = [fake, fake, fake, 1, 2, 128, 4, 8, 8, 3, 3, 3, ctypes.c_float(0.1), fake, 3, fake,
            fake, 1 << 30, N, N]
    bad_d = list(args)
    bad_d[5] = 96
    assert lib.heta_attention(*bad_d) == heta.HETA_ERR_UNSUPPORTED
    even_win = list(args)
    even_win[10] = 4
    assert lib.heta_attention(*even_win) == heta.HETA_ERR_UNSUPPORTED
    big_win = list(args)
    big_win[9] = 5
    assert lib.heta_attention(*big_win) == heta.HETA_ERR_INVALID_ARG
    bad_k = list(args)
    bad_k[14] = 257
    assert lib.heta_attention(*bad_k) == heta.HETA_ERR_INVALID_ARG
    bad_scale = list(args)
    bad_scale[12] = ctypes.c_float(float("nan"))
    assert lib.heta_attention(*bad_scale) == heta.HETA_ERR_INVALID_ARG
    small_ws = list(args)
    small_ws[17] = 16
    assert lib.heta_attention(*small_ws) == heta.HETA_ERR_INVALID_ARG
    no_ws = list(args)
    no_ws[16] = N
    assert lib.heta_attention(*no_ws) == heta.HETA_ERR_INVALID_ARG
    assert lib.heta_uncertainty(fake, fake, ctypes.c_float(0.0), 1, 10, 12, fake, N, N) == \
        heta.HETA_ERR_INVALID_ARG
    assert lib.heta_uncertainty(fake, fake, ctypes.c_float(0.0), 1, 10, 32768, fake, N, N) == \
        heta.HETA_ERR_UNSUPPORTED


def test_threshold_entry_points_validate_on_the_host(lib):
    N = None
    fake = ctypes.c_void_p(1 << 20)
    d = ctypes.c_double
    rt = lib.heta_route_threshold
    rt.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, d] + [ctypes.c_void_p] * 7
    assert rt(fake, 0, 10, d(0.9), fake, fake, fake, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    assert rt(fake, 1, 0, d(0.9), fake, fake, fake, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    assert rt(fake, 1, 8 * 49152 + 1, d(0.9), fake, fake, fake, N, N, N, N) == \
        heta.HETA_ERR_UNSUPPORTED
    assert rt(fake, 1, 10, d(float("nan")), fake, fake, fake, N, N, N, N) == \
        heta.HETA_ERR_INVALID_ARG
    assert rt(fake, 1, 10, d(float("inf")), fake, fake, fake, N, N, N, N) == \
        heta.HETA_ERR_INVALID_ARG
    assert rt(fake, 1, 10, d(0.9), N, fake, fake, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert rt(fake, 1, 10, d(0.9), odd, fake, fake, N, N, N, N) == heta.HETA_ERR_INVALID_ARG
    ac = lib.heta_attention_counts
    args = [fake, fake, fake, 1, 2, 128, 4, 8, 8, 3, 3, 3, ctypes.c_float(0.1), fake, 256, fake,
            fake, fake, 1 << 30, N, N]
    no_counts = list(args)
    no_counts[15] = N
    assert ac(*no_counts) == heta.HETA_ERR_INVALID_ARG
    big_cap = list(args)
    big_cap[14] = 257
    assert ac(*big_cap) == heta.HETA_ERR_INVALID_ARG
    bad_d = list(args)
    bad_d[5] = 96
    assert ac(*bad_d) == heta.HETA_ERR_UNSUPPORTED
    small_ws = list(args)
    small_ws[18] = 16
    assert ac(*small_ws) == heta.HETA_ERR_INVALID_ARG


def test_swap_entry_point_validates_on_the_host(lib):
    N = None
    fake = ctypes.c_void_p(1 << 20)
    sw = lib.heta_route_swap
    sw.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_uint64, ctypes.c_int] + \
        [ctypes.c_void_p] * 5
    ok = [fake, 1, 100, 20, 5, 7, 0, fake, fake, N, N, N]
    for pos, bad in ((1, 0), (2, 0), (3, 101), (4, 21), (4, -1), (6, -1)):
        a = list(ok)
        a[pos] = bad
        assert sw(*a) == heta.HETA_ERR_INVALID_ARG, (pos, bad)
    big_s = list(ok)
    big_s[3], big_s[4] = 90, 11  # s > N - k
    assert sw(*big_s) == heta.HETA_ERR_INVALID_ARG
    too_big = list(ok)
    too_big[2], too_big[3], too_big[4] = 8 * 49152 + 1, 20, 5
    assert sw(*too_big) == heta.HETA_ERR_UNSUPPORTED
    no_local = list(ok)
    no_local[8] = N
    assert sw(*no_local) == heta.HETA_ERR_INVALID_ARG
    odd = list(ok)
    odd[7] = ctypes.c_void_p((1 << 20) + 4)
    assert sw(*odd) == heta.HETA_ERR_INVALID_ARG
    assert heta.swap_count(32760, 6552, 0.07) == 2294
    assert heta.swap_count(100, 5, 0.07) == 5


def test_swap_blocks_entry_point_validates_on_the_host(lib):
    """The many-block swap: block count, block range and the rule that the
    outputs of more than one block may not overlap the input."""
    N = None
    base = 1 << 20
    fake = ctypes.c_void_p(base)
    sw = lib.heta_route_swap_blocks
    sw.argtypes = [ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_uint64] + \
        [ctypes.c_int] * 2 + [ctypes.c_void_p] * 5
    # B=1, N=100, k=20, s=5; input at base, outputs far away
    far = ctypes.c_void_p(base + (1 << 24))
    ok = [fake, 1, 100, 20, 5, 7, 0, 3, far, far, N, N, N]
    for pos, bad in ((7, 0), (7, -2), (6, -1), (4, 21)):
        a = list(ok)
        a[pos] = bad
        assert sw(*a) == heta.HETA_ERR_INVALID_ARG, (pos, bad)
    a = list(ok)
    a[6] = 2 ** 31 - 2  # block0 + nblocks - 1 past INT32_MAX
    assert sw(*a) == heta.HETA_ERR_INVALID_ARG
    # dense_out overlapping dense_idx with nblocks > 1 (never launched)
    over = list(ok)
    over[8] = ctypes.c_void_p(base + 16 * 3)
    assert sw(*over) == heta.HETA_ERR_INVALID_ARG


def test_flop_model_matches_the_papers_reduction():
    """Eq. (14) at the Wan2.1-1.3B latent shape, rho = 0.2, 3x9x9 window.

    The dense/heterogeneous FLOP ratio comes out at 4.856; Table 5 prints an
    attention-FLOPs reduction of 4.87x for Wan2.1-1.3B.  Context only: the
    paper does not state which window produced its table.
    """
    N, M = 32760, 243
    k = heta.dense_count(N, 0.2)
    full = heta.attention_flops(1, 12, 128, N, N, M)
    het = heta.attention_flops(1, 12, 128, N, k, M)
    assert abs(full / het - 4.87) < 0.02
    assert het == 4 * 128 * 12 * (k * N + (N - k) * M)


def test_workspace_size(lib):
    """Whole waves of dense pairs run unsplit and need no scratch beyond the
    work counter; the pairs of a last wave at most half full (or of a first
    and only, partial wave) are cut into two key ranges whose fp32 partials
    the workspace holds."""
    # rho = 0.2: 312 pairs = 2 waves of 148 + 16 pairs cut in halves
    k = heta.dense_count(32760, 0.2)
    part = heta.attention_workspace_size(1, 12, 128, (21, 30, 52), (3, 9, 9), k)
    assert part >= 16 * 2 * 2 * 128 * (128 * 4 + 8)
    assert part < 5 * 2 ** 20
    # a last wave more than half full runs whole: counter only
    k_full = heta.dense_count(32760, 0.15)  # 240 pairs = 148 + 92
    assert heta.attention_workspace_size(1, 12, 128, (21, 30, 52), (3, 9, 9), k_full) == 256
    # one partial wave (rho = 0.05: 84 pairs) is cut in halves as well
    k_small = heta.dense_count(32760, 0.05)
    w_small = heta.attention_workspace_size(1, 12, 128, (21, 30, 52), (3, 9, 9), k_small)
    assert w_small >= 84 * 2 * 2 * 128 * (128 * 4 + 8)
    # exactly whole waves: 148 pairs of 2 tiles -> no split, counter only
    k148 = 148 * 256
    w = heta.attention_workspace_size(1, 1, 128, (37, 32, 32), (3, 9, 9), k148)
    assert w == 256
    # no dense rows, or too few key tiles to split: counter only
    assert heta.attention_workspace_size(1, 2, 64, (4, 8, 8), (3, 3, 3), 0) == 256
    assert heta.attention_workspace_size(1, 2, 64, (4, 8, 8), (3, 3, 3), 200) == 256
    with pytest.raises(heta.HetaError):
        heta.attention_workspace_size(1, 2, 96, (4, 8, 8), (3, 3, 3), 10)
    # per-sample counts: scratch for the worst remainder the device may find,
    # at most 147 pairs in halves (147 * 2 ranges * 2 tiles * 128 rows * 520 bytes)
    wc = heta.attention_counts_workspace_size(1, 12, 128, (21, 30, 52), (3, 9, 9), 32760)
    assert max(part, w_small) <= wc <= 147 * 2 * 2 * 128 * (128 * 4 + 8) + 4096
    assert wc > 32 << 20
    with pytest.raises(heta.HetaError):
        heta.attention_counts_workspace_size(1025, 1, 128, (21, 30, 52), (3, 9, 9), 100)
