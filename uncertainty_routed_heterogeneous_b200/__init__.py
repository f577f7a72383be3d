"""B200-native heterogeneous (uncertainty-routed) attention.

Python binding over the C ABI of ``libheta.so`` (``include/heta.h``).  This
module only marshals arguments: it checks tensor placement, dtype and shape,
passes raw device pointers and the current CUDA stream, and turns status codes
into exceptions.  Every step of the path runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback -- if the library is missing, every call
raises.

The method is HetA-DiT ("Where Compute Matters: Heterogeneous Attention for
Efficient Video Diffusion"): per-sample routing of the most uncertain tokens
(Eq. (11)-(12), top-k form) to dense attention (Eq. (2)), windowed 3D local
attention for the rest (Eq. (3)), merged row by row (Eq. (13)); the
uncertainty head (Eq. (7)) produces the next step's scores.
"""
import ctypes
import math
import os

__all__ = ["load", "HetaError", "dense_count", "route", "route_threshold", "swap_count",
           "route_swap", "route_swap_blocks", "attention", "attention_counts",
           "attention_noalloc",
           "attention_workspace_size", "attention_counts_workspace_size", "uncertainty",
           "selftest_wait_timeout", "status_string", "attention_flops", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libheta.so")

HETA_OK = 0
HETA_ERR_INVALID_ARG = 1
HETA_ERR_UNSUPPORTED = 2
HETA_ERR_CUDA = 3
HETA_ERR_NONFINITE = 4
HETA_ERR_TIMEOUT = 5

_lib = None


class HetaError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = int(code)
        super().__init__("%s: heta status %d (%s)" % (what, self.code, status_string(self.code)))


def load():
    """Loads libheta.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libheta.so is not built (%s). Build it with "
            "`python -m uncertainty_routed_heterogeneous_b200.build`; "
            "there is no fallback path." % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double
    lib.heta_status_string.argtypes = [i]
    lib.heta_status_string.restype = ctypes.c_char_p
    lib.heta_version.argtypes = []
    lib.heta_version.restype = i
    lib.heta_dense_count.argtypes = [i, d, ctypes.POINTER(ctypes.c_int)]
    lib.heta_dense_count.restype = i
    lib.heta_route.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, vp]
    lib.heta_route.restype = i
    lib.heta_attention_workspace_size.argtypes = [i] * 10 + [ctypes.POINTER(ctypes.c_size_t)]
    lib.heta_attention_workspace_size.restype = i
    lib.heta_attention.argtypes = [vp, vp, vp] + [i] * 9 + [f, vp, i, vp, vp, ctypes.c_size_t,
                                                            vp, vp]
    lib.heta_attention.restype = i
    lib.heta_uncertainty.argtypes = [vp, vp, f, i, i, i, vp, vp, vp]
    lib.heta_uncertainty.restype = i
    lib.heta_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp, vp, vp]
    lib.heta_selftest_wait_timeout.restype = i
    lib.heta_route_swap.argtypes = [vp, i, i, i, i, ctypes.c_uint64, i, vp, vp, vp, vp, vp]
    lib.heta_route_swap.restype = i
    lib.heta_route_swap_blocks.argtypes = [vp, i, i, i, i, ctypes.c_uint64, i, i, vp, vp, vp,
                                           vp, vp]
    lib.heta_route_swap_blocks.restype = i
    lib.heta_route_threshold.argtypes = [vp, i, i, d, vp, vp, vp, vp, vp, vp, vp]
    lib.heta_route_threshold.restype = i
    lib.heta_attention_counts.argtypes = ([vp, vp, vp] + [i] * 9 +
                                          [f, vp, i, vp, vp, vp, ctypes.c_size_t, vp, vp])
    lib.heta_attention_counts.restype = i
    lib.heta_attention_counts_workspace_size.argtypes = ([i] * 10 +
                                                         [ctypes.POINTER(ctypes.c_size_t)])
    lib.heta_attention_counts_workspace_size.restype = i
    lib.heta_attention_noalloc.argtypes = [vp, vp, vp] + [i] * 9 + [f, vp, i, vp, vp, vp]
    lib.heta_attention_noalloc.restype = i
    _lib = lib
    return lib


def status_string(code: int) -> str:
    try:
        return load().heta_status_string(int(code)).decode()
    except RuntimeError:
        return "library not loaded"


def _check(rc, what):
    if rc != HETA_OK:
        raise HetaError(rc, what)


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t, dtype, name, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got %d" % (name, ndim, t.dim()))
    return ctypes.c_void_p(t.data_ptr())


def _opt(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def dense_count(N: int, rho: float) -> int:
    """k = ceil(rho*N) for the decimal rho stated (the dense fraction of Eq. (14))."""
    k = ctypes.c_int(0)
    _check(load().heta_dense_count(int(N), float(rho), ctypes.byref(k)), "heta_dense_count")
    return int(k.value)


def route(u, k: int, *, out=None, want_thresh=False, want_mask=False, status=None):
    """Per-sample top-k routing on the GPU (``heta_route``).

    u: [B,N] float32 CUDA.  Returns (dense_idx [B,k] int32, local_idx [B,N-k]
    int32, thresh [B] float32 or None, mask [B,N] uint8 or None).
    ``out`` may pass preallocated (dense_idx, local_idx, thresh, mask).
    """
    import torch
    pu = _dev(u, torch.float32, "u", 2)
    B, N = u.shape
    if out is None:
        dense = torch.empty((B, k), dtype=torch.int32, device=u.device)
        local = torch.empty((B, N - k), dtype=torch.int32, device=u.device)
        thresh = torch.empty(B, dtype=torch.float32, device=u.device) if want_thresh else None
        mask = torch.empty((B, N), dtype=torch.uint8, device=u.device) if want_mask else None
    else:
        dense, local, thresh, mask = out
    rc = load().heta_route(pu, B, N, int(k), _opt(dense) if k > 0 else None,
                           _opt(local) if k < N else None, _opt(thresh), _opt(mask),
                           _opt(status), _stream())
    _check(rc, "heta_route")
    return dense, local, thresh, mask


def selftest_wait_timeout(limit_ns: int, status, elapsed=None):
    """Runs the library's bounded-wait path into a timeout on purpose
    (``heta_selftest_wait_timeout``): status (int32 CUDA) receives
    HETA_ERR_TIMEOUT; elapsed (int64 CUDA, optional) the kernel's wall time."""
    import torch
    ps = _dev(status, torch.int32, "status")
    pe = _dev(elapsed, torch.int64, "elapsed") if elapsed is not None else None
    _check(load().heta_selftest_wait_timeout(int(limit_ns), ps, pe, _stream()),
           "heta_selftest_wait_timeout")


def swap_count(N: int, k: int, r: float) -> int:
    """Tokens one block's random swap moves each way: ceil(r*N) (read like
    ``dense_count``), at most min(k, N-k)."""
    return min(dense_count(N, r), k, N - k)


def route_swap(dense_idx, N: int, s: int, seed: int, block: int, *, out=None, want_mask=False,
               status=None):
    """One transformer block's random swap of a top-k routing (``heta_route_swap``).

    dense_idx: [B,k] int32 CUDA (the ``route`` output).  Returns (dense [B,k],
    local [B,N-k], mask [B,N] uint8 or None); ``out`` may pass preallocated
    (dense, local, mask), and dense may be dense_idx itself.
    """
    import torch
    pd = _dev(dense_idx, torch.int32, "dense_idx", 2)
    B, k = dense_idx.shape
    if out is None:
        dense = torch.empty((B, k), dtype=torch.int32, device=dense_idx.device)
        local = torch.empty((B, N - k), dtype=torch.int32, device=dense_idx.device)
        mask = (torch.empty((B, N), dtype=torch.uint8, device=dense_idx.device)
                if want_mask else None)
    else:
        dense, local, mask = out
    rc = load().heta_route_swap(pd if k > 0 else None, B, int(N), k, int(s),
                                int(seed) & 0xFFFFFFFFFFFFFFFF, int(block),
                                _opt(dense) if k > 0 else None, _opt(local) if k < N else None,
                                _opt(mask), _opt(status), _stream())
    _check(rc, "heta_route_swap")
    return dense, local, mask


def route_swap_blocks(dense_idx, N: int, s: int, seed: int, block0: int, nblocks: int, *,
                      out=None, want_mask=False, status=None):
    """The random swaps of nblocks consecutive transformer blocks in one launch
    (``heta_route_swap_blocks``).

    dense_idx: [B,k] int32 CUDA.  Returns (dense [nblocks,B,k], local
    [nblocks,B,N-k], mask [nblocks,B,N] uint8 or None); ``out`` may pass
    preallocated (dense, local, mask), not overlapping dense_idx.
    """
    import torch
    pd = _dev(dense_idx, torch.int32, "dense_idx", 2)
    B, k = dense_idx.shape
    nb = int(nblocks)
    if out is None:
        dev = dense_idx.device
        dense = torch.empty((nb, B, k), dtype=torch.int32, device=dev)
        local = torch.empty((nb, B, N - k), dtype=torch.int32, device=dev)
        mask = torch.empty((nb, B, N), dtype=torch.uint8, device=dev) if want_mask else None
    else:
        dense, local, mask = out
    rc = load().heta_route_swap_blocks(pd if k > 0 else None, B, int(N), k, int(s),
                                       int(seed) & 0xFFFFFFFFFFFFFFFF, int(block0), nb,
                                       _opt(dense) if k > 0 else None,
                                       _opt(local) if k < N else None, _opt(mask),
                                       _opt(status), _stream())
    _check(rc, "heta_route_swap_blocks")
    return dense, local, mask


def route_threshold(u, c: float, *, out=None, want_thresh=False, want_mask=False,
                    status=None):
    """Routing by the paper's T = mu + c*sigma rule (``heta_route_threshold``).

    u: [B,N] float32 CUDA.  Returns (counts [B] int32, dense_idx [B,N] int32,
    local_idx [B,N] int32, thresh [B] float64 or None, mask [B,N] uint8 or
    None), all on the device; row b of dense_idx holds counts[b] ids.
    ``out`` may pass preallocated (counts, dense_idx, local_idx, thresh, mask).
    """
    import torch
    pu = _dev(u, torch.float32, "u", 2)
    B, N = u.shape
    if out is None:
        counts = torch.empty(B, dtype=torch.int32, device=u.device)
        dense = torch.empty((B, N), dtype=torch.int32, device=u.device)
        local = torch.empty((B, N), dtype=torch.int32, device=u.device)
        thresh = torch.empty(B, dtype=torch.float64, device=u.device) if want_thresh else None
        mask = torch.empty((B, N), dtype=torch.uint8, device=u.device) if want_mask else None
    else:
        counts, dense, local, thresh, mask = out
    rc = load().heta_route_threshold(pu, B, N, float(c), _opt(counts), _opt(dense),
                                     _opt(local), _opt(thresh), _opt(mask), _opt(status),
                                     _stream())
    _check(rc, "heta_route_threshold")
    return counts, dense, local, thresh, mask


def attention_workspace_size(B, H, d, grid, win, k) -> int:
    """Bytes of device scratch one ``attention`` call needs for these sizes."""
    n = ctypes.c_size_t(0)
    _check(load().heta_attention_workspace_size(int(B), int(H), int(d), grid[0], grid[1],
                                                grid[2], win[0], win[1], win[2], int(k),
                                                ctypes.byref(n)),
           "heta_attention_workspace_size")
    return int(n.value)


def attention(Q, K, V, grid, win, dense_idx, *, scale=None, out=None, status=None,
              workspace=None):
    """Routed heterogeneous attention (``heta_attention``).

    Q, K, V: [B,H,N,d] bfloat16 CUDA; grid = (Tg, Hg, Wg) with N = Tg*Hg*Wg;
    win = (wt, wh, ww) odd; dense_idx: [B,k] int32 CUDA, increasing.
    ``workspace``: a uint8 CUDA tensor of at least ``attention_workspace_size``
    bytes (allocated here when omitted).  Returns out [B,H,N,d] bfloat16.
    """
    import torch
    pq = _dev(Q, torch.bfloat16, "Q", 4)
    pk = _dev(K, torch.bfloat16, "K", 4)
    pv = _dev(V, torch.bfloat16, "V", 4)
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K, V shapes differ")
    B, H, N, d = Q.shape
    Tg, Hg, Wg = grid
    if Tg * Hg * Wg != N:
        raise ValueError("grid %s does not hold N=%d tokens" % (grid, N))
    pd = _dev(dense_idx, torch.int32, "dense_idx", 2)
    if dense_idx.shape[0] != B:
        raise ValueError("dense_idx batch mismatch")
    k = dense_idx.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    po = _dev(out, torch.bfloat16, "out", 4)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attention_workspace_size(B, H, d, grid, win, k)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=Q.device)
    pw = _dev(workspace, torch.uint8, "workspace", 1)
    rc = load().heta_attention(pq, pk, pv, B, H, d, Tg, Hg, Wg, win[0], win[1], win[2],
                               float(scale), pd if k > 0 else None, k, po, pw,
                               workspace.numel(), _opt(status), _stream())
    _check(rc, "heta_attention")
    return out


def attention_noalloc(Q, K, V, grid, win, dense_idx, *, scale=None, out=None, status=None):
    """``attention`` without a workspace (``heta_attention_noalloc``): the
    library's fixed device array serves as its scratch, so nothing is
    allocated for the call (``out`` aside, when it is not passed).  Calls that
    may overlap on the GPU race on that array; see include/heta.h."""
    import torch
    pq = _dev(Q, torch.bfloat16, "Q", 4)
    pk = _dev(K, torch.bfloat16, "K", 4)
    pv = _dev(V, torch.bfloat16, "V", 4)
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K, V shapes differ")
    B, H, N, d = Q.shape
    Tg, Hg, Wg = grid
    if Tg * Hg * Wg != N:
        raise ValueError("grid %s does not hold N=%d tokens" % (grid, N))
    pd = _dev(dense_idx, torch.int32, "dense_idx", 2)
    if dense_idx.shape[0] != B:
        raise ValueError("dense_idx batch mismatch")
    k = dense_idx.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    po = _dev(out, torch.bfloat16, "out", 4)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = load().heta_attention_noalloc(pq, pk, pv, B, H, d, Tg, Hg, Wg, win[0], win[1], win[2],
                                       float(scale), pd if k > 0 else None, k, po,
                                       _opt(status), _stream())
    _check(rc, "heta_attention_noalloc")
    return out


def attention_counts_workspace_size(B, H, d, grid, win, k_cap) -> int:
    """Bytes of device scratch one ``attention_counts`` call needs."""
    n = ctypes.c_size_t(0)
    _check(load().heta_attention_counts_workspace_size(int(B), int(H), int(d), grid[0], grid[1],
                                                       grid[2], win[0], win[1], win[2],
                                                       int(k_cap), ctypes.byref(n)),
           "heta_attention_counts_workspace_size")
    return int(n.value)


def attention_counts(Q, K, V, grid, win, dense_idx, counts, *, scale=None, out=None,
                     status=None, workspace=None):
    """``attention`` with per-sample dense counts on the device
    (``heta_attention_counts``): dense_idx [B,k_cap] int32 whose row b holds
    counts[b] increasing ids (e.g. the ``route_threshold`` output, k_cap = N),
    counts [B] int32 CUDA.  Returns out [B,H,N,d] bfloat16."""
    import torch
    pq = _dev(Q, torch.bfloat16, "Q", 4)
    pk = _dev(K, torch.bfloat16, "K", 4)
    pv = _dev(V, torch.bfloat16, "V", 4)
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K, V shapes differ")
    B, H, N, d = Q.shape
    Tg, Hg, Wg = grid
    if Tg * Hg * Wg != N:
        raise ValueError("grid %s does not hold N=%d tokens" % (grid, N))
    pd = _dev(dense_idx, torch.int32, "dense_idx", 2)
    pc = _dev(counts, torch.int32, "counts", 1)
    if dense_idx.shape[0] != B or counts.shape[0] != B:
        raise ValueError("dense_idx / counts batch mismatch")
    k_cap = dense_idx.shape[1]
    if out is None:
        out = torch.empty_like(Q)
    po = _dev(out, torch.bfloat16, "out", 4)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attention_counts_workspace_size(B, H, d, grid, win, k_cap)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=Q.device)
    pw = _dev(workspace, torch.uint8, "workspace", 1)
    rc = load().heta_attention_counts(pq, pk, pv, B, H, d, Tg, Hg, Wg, win[0], win[1], win[2],
                                      float(scale), pd if k_cap > 0 else None, k_cap, pc, po, pw,
                                      workspace.numel(), _opt(status), _stream())
    _check(rc, "heta_attention_counts")
    return out


def uncertainty(X, w, bias: float = 0.0, *, out=None, status=None):
    """u = softplus(X.w + b) per token (``heta_uncertainty``).

    X: [B,N,C] bfloat16 CUDA; w: [C] float32 CUDA.  Returns u [B,N] float32.
    """
    import torch
    px = _dev(X, torch.bfloat16, "X", 3)
    pw = _dev(w, torch.float32, "w", 1)
    B, N, C = X.shape
    if w.shape[0] != C:
        raise ValueError("w has %d entries, X has C=%d" % (w.shape[0], C))
    if out is None:
        out = torch.empty((B, N), dtype=torch.float32, device=X.device)
    pu = _dev(out, torch.float32, "u_out", 2)
    rc = load().heta_uncertainty(px, pw, float(bias), B, N, C, pu, _opt(status), _stream())
    _check(rc, "heta_uncertainty")
    return out


def attention_flops(B: int, H: int, d: int, N: int, k: int, M: int) -> int:
    """Algorithmic FLOPs of one routed-attention call.

    Two matrix products (q.k and p.v) of 2*d FLOPs per (query, key) pair:
    k*N pairs for the dense rows and (N-k)*M for the local rows per (b, h) --
    the two terms of the cost model of Eq. (14).
    """
    return 4 * d * H * B * (k * N + (N - k) * M)
