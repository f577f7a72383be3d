"""fp64 CPU oracle for the heterogeneous (uncertainty-routed) attention path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  The
product (the CUDA library and its binding) never imports it, and it imports
nothing from the product: the two share only the seeded input generators.

Every function is a thin numpy wrapper around ``heta_oracle.c``, which follows
"Where Compute Matters: Heterogeneous Attention for Efficient Video Diffusion"
(HetA-DiT): Eq. (2) dense attention, Eq. (3) local attention, Eq. (7) the
per-token uncertainty, Eq. (11)-(12) the routing rule (top-k reading),
Eq. (13) the mix and Eq. (14) the dense fraction.  The readings taken where
the paper is silent are listed at the top of ``heta_oracle.c``.

Parity pins (tests/test_oracle_pins.py) tie every function here to something
other than itself; no function is "parity unpinned".
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

OK = 0
INVALID = 1
NONFINITE = 4

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_dense_count.argtypes = [ctypes.c_int, ctypes.c_double, i32p]
        lib.oracle_route.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p]
        lib.oracle_route_threshold.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_double] + [ctypes.c_void_p] * 5
        lib.oracle_philox4x32_10.argtypes = [ctypes.c_void_p] * 3
        lib.oracle_route_swap.argtypes = ([ctypes.c_void_p] + [ctypes.c_int] * 4 +
                                          [ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_void_p])
        lib.oracle_window_start.argtypes = [ctypes.c_int] * 3
        lib.oracle_window.argtypes = [ctypes.c_int] * 7 + [ctypes.c_void_p]
        lib.oracle_attention_rows.argtypes = (
            [ctypes.c_void_p] * 3 + [ctypes.c_int] * 10 + [ctypes.c_double,
             ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
             ctypes.c_void_p, ctypes.c_int])
        lib.oracle_uncertainty.argtypes = [ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_double, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int,
                                           ctypes.c_void_p, ctypes.c_int]
        lib.oracle_max_threads.argtypes = []
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__("oracle status %d" % code)
        self.code = code


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def dense_count(N: int, rho: float) -> int:
    """k = ceil(fl(rho*N)): the dense-token count per sample (Eq. (14)'s rho)."""
    k = ctypes.c_int32(0)
    rc = _load().oracle_dense_count(int(N), float(rho), ctypes.byref(k))
    if rc:
        raise OracleError(rc)
    return int(k.value)


def route(u: np.ndarray, k: int):
    """Top-k routing per sample (Eq. (11)-(12), readings R1/R2).

    u: [B,N] float32.  Returns (dense_idx [B,k], local_idx [B,N-k], mask [B,N])
    as int32/int32/uint8; mask is the paper's m_i (1 = local, 0 = dense).
    """
    u = np.ascontiguousarray(u, dtype=np.float32)
    B, N = u.shape
    dense = np.zeros((B, k), np.int32)
    local = np.zeros((B, N - k), np.int32)
    mask = np.zeros((B, N), np.uint8)
    rc = _load().oracle_route(_ptr(u), B, N, int(k), _ptr(dense), _ptr(local), _ptr(mask))
    if rc:
        raise OracleError(rc)
    return dense, local, mask


def route_threshold(u: np.ndarray, c: float):
    """Routing by the paper's threshold T = mu + c*sigma (Eq. (11)-(12), reading R10).

    u: [B,N] float32.  Returns (counts [B], dense_idx [B,N], local_idx [B,N],
    thresh [B] float64, mask [B,N]); row b of dense_idx holds counts[b]
    ascending token ids (the rest is padding), row b of local_idx the other
    N - counts[b]; mask is m_i (1 = local).
    """
    u = np.ascontiguousarray(u, dtype=np.float32)
    B, N = u.shape
    counts = np.zeros(B, np.int32)
    dense = np.full((B, N), -1, np.int32)
    local = np.full((B, N), -1, np.int32)
    thresh = np.zeros(B, np.float64)
    mask = np.zeros((B, N), np.uint8)
    rc = _load().oracle_route_threshold(_ptr(u), B, N, float(c), _ptr(counts), _ptr(dense),
                                        _ptr(local), _ptr(thresh), _ptr(mask))
    if rc:
        raise OracleError(rc)
    return counts, dense, local, thresh, mask


def philox4x32_10(ctr, key):
    """Philox4x32-10 (Salmon et al., SC 2011) of a 4-word counter and 2-word key."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, np.uint32)
    _load().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def route_swap(dense_idx: np.ndarray, N: int, s: int, seed: int, block: int):
    """One transformer block's random swap (reading R11) of a top-k routing.

    dense_idx: [B,k] int32 ascending.  Returns (dense [B,k], local [B,N-k]).
    """
    dense_idx = np.ascontiguousarray(dense_idx, dtype=np.int32)
    B, k = dense_idx.shape
    dense = np.zeros((B, k), np.int32)
    local = np.zeros((B, N - k), np.int32)
    rc = _load().oracle_route_swap(_ptr(dense_idx), B, int(N), int(k), int(s), int(seed),
                                   int(block), _ptr(dense), _ptr(local))
    if rc:
        raise OracleError(rc)
    return dense, local


def window_start(p: int, extent: int, width: int) -> int:
    return int(_load().oracle_window_start(int(p), int(extent), int(width)))


def window(grid, win, i: int) -> np.ndarray:
    """Keys of token i's clamped 3D window, ascending (Eq. (3), reading R3)."""
    Tg, Hg, Wg = grid
    wt, wh, ww = win
    out = np.zeros(wt * wh * ww, np.int32)
    n = _load().oracle_window(Tg, Hg, Wg, wt, wh, ww, int(i), _ptr(out))
    return out[:n]


def attention_rows(Q, K, V, grid, win, dense_idx, rows, scale=None, nthreads=0):
    """Output rows of the heterogeneous attention (Eq. (2), (3), (13)) in fp64.

    Q,K,V: [B,H,N,d] float32 holding the exact (bf16-rounded) inputs.
    dense_idx: [B,k] int32.  rows: flat ids (b*H + h)*N + i.  Returns [len(rows), d].
    """
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    K = np.ascontiguousarray(K, dtype=np.float32)
    V = np.ascontiguousarray(V, dtype=np.float32)
    B, H, N, d = Q.shape
    Tg, Hg, Wg = grid
    wt, wh, ww = win
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dense_idx = np.ascontiguousarray(dense_idx, dtype=np.int32).reshape(B, -1)
    k = dense_idx.shape[1]
    rows = np.ascontiguousarray(rows, dtype=np.int64).ravel()
    out = np.zeros((rows.size, d), np.float64)
    rc = _load().oracle_attention_rows(
        _ptr(Q), _ptr(K), _ptr(V), B, H, N, d, Tg, Hg, Wg, wt, wh, ww,
        float(scale), _ptr(dense_idx), k, _ptr(rows), rows.size, _ptr(out),
        int(nthreads))
    if rc:
        raise OracleError(rc)
    return out


def attention(Q, K, V, grid, win, dense_idx, scale=None, nthreads=0):
    """All rows: returns [B,H,N,d] fp64."""
    B, H, N, d = Q.shape
    rows = np.arange(B * H * N, dtype=np.int64)
    return attention_rows(Q, K, V, grid, win, dense_idx, rows, scale,
                          nthreads).reshape(B, H, N, d)


def uncertainty(X, w, bias=0.0, nthreads=0):
    """u = softplus(X . w + b) per token in fp64 (Eq. (7), reading R7).

    X: [B,N,C] float32 (exact bf16 values); w: [C] float32.  Returns [B,N] fp64.
    """
    X = np.ascontiguousarray(X, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    B, N, C = X.shape
    out = np.zeros((B, N), np.float64)
    rc = _load().oracle_uncertainty(_ptr(X), _ptr(w), float(bias), B, N, C,
                                    _ptr(out), int(nthreads))
    if rc:
        raise OracleError(rc)
    return out
