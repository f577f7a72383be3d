#!/usr/bin/env python
"""Benchmark of the routed heterogeneous-attention step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl heta|reference]

One step is one pass of the whole path over one sample of the Wan2.1-1.3B
latent shape (B=1, H=12, d=128, grid 21x30x52, N=32760, rho=0.2, window
3x9x9): route the previous step's uncertainty u -> routed attention (dense
rows + windowed local rows, merged) -> uncertainty head on the step's hidden
states X (C=1536) producing the next step's u.  Inputs are seeded synthetic
data resident in HBM; Q/K/V/X (402 MB) exceed the 126 MB L2, so no flush is
needed between steps.

Rank 0 prints one JSON line.  Under torchrun each rank processes its own
independent sample (weak scaling, no data-path collective); the timed region
is bracketed by barriers and the elapsed time is the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores instead (a
deliberately slow baseline, not a target), on a bounded sample of the same
workload per step.
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from uncertainty_routed_heterogeneous_b200 import dist as D  # noqa: E402
from uncertainty_routed_heterogeneous_b200 import workloads as W  # noqa: E402

METRIC = "routed-attention tokens/s and TFLOP/s (fraction of B200 bf16 peak) at 1 GPU"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[1])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["heta", "reference"], default="heta")
    p.add_argument("--workload", default=W.WAN21.name, choices=sorted(W.ALL))
    p.add_argument("--rho", type=float, default=None,
                   help="dense fraction (default: the workload's own, 0.2)")
    p.add_argument("--window", default=None,
                   help="local window as TxHxW, odd sizes (default: the workload's own)")
    p.add_argument("--cpu-tokens", type=int, default=1536,
                   help="tokens in the oracle's bounded CPU sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-dense-compare", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-other-configs", action="store_true",
                   help="skip timing the Wan2.2 shape, the batched step with the head and "
                        "the rho sweep (uniform / clustered u)")
    p.add_argument("--no-window-sweep", action="store_true",
                   help="skip timing the 9^3 / 11^3 / 13^3 windows of the paper's ablation")
    p.add_argument("--no-threshold-mode", action="store_true",
                   help="skip timing the paper's mu + c*sigma routing (c = 0.9)")
    p.add_argument("--no-route-throughput", action="store_true",
                   help="skip timing heta_route on 512 samples in one launch")
    p.add_argument("--nvtx", action="store_true",
                   help="mark route / attention / head of every step with NVTX ranges")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="minimum host time the cpu_baseline oracle sample runs for")
    p.add_argument("--no-flex-compare", action="store_true",
                   help="skip timing PyTorch FlexAttention on the same mask (the paper's own "
                        "latency instrument; a comparison point, not part of the product)")
    p.add_argument("--shard", choices=["samples", "heads"], default="samples",
                   help="samples: each rank runs its own sample (weak scaling, the default); "
                        "heads: the ranks split one sample's heads and the head's token rows "
                        "and all-gather the next step's u (strong scaling)")
    p.add_argument("--gather-out", action="store_true",
                   help="with --shard heads: also all-gather the output along heads")
    return p.parse_args()


def chosen_workload(args):
    """The named workload, with --rho / --window applied (a renamed copy)."""
    import dataclasses
    w = W.ALL[args.workload]
    if args.rho is not None:
        if not 0.0 <= args.rho <= 1.0:
            raise SystemExit("--rho must lie in [0, 1]")
        w = dataclasses.replace(w, name="%s-rho%g" % (w.name, args.rho), rho=args.rho)
    if args.window is not None:
        win = tuple(int(x) for x in args.window.lower().split("x"))
        if len(win) != 3 or any(x < 1 or x % 2 == 0 for x in win):
            raise SystemExit("--window takes three odd sizes, e.g. 11x11x11")
        w = dataclasses.replace(w, name="%s-win%s" % (w.name, args.window), win=win)
    return w


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        pk["source"] = "measured"
        return pk
    except (OSError, ValueError):
        pk = dict(FALLBACK_PEAKS)
        pk["source"] = "fallback"
        return pk


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; no setting is changed)
# ----------------------------------------------------------------------------


class ClockSampler:
    REASONS = {  # NVML clocks-event-reason bits
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, torch_device_index, period_s=0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._on = threading.Event()
        self.handle = None
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 -- clocks are best-effort metadata
            self.error = repr(e)
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            if self._on.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    self.samples.append((mhz, rs))
                except Exception:  # noqa: BLE001
                    pass
            time.sleep(self.period)

    def start(self):
        self._on.set()

    def stop(self):
        self._on.clear()

    def close(self):
        self._stop.set()

    def summary(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "NVML unavailable: %s" % getattr(self, "error", "")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        active = set()
        for _, rs in self.samples:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    active.add(name)
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(active), "samples": len(mhz)}


# ----------------------------------------------------------------------------
# CPU side: the fp64 oracle on a bounded sample (reference arm / cpu_baseline)
# ----------------------------------------------------------------------------


class OracleSample:
    """Host copies of one sample and the oracle calls that make one 'step'."""

    def __init__(self, w, n_tokens, seed=123):
        import oracle
        self.oracle = oracle
        self.w = w
        q, k, v = W.make_qkv(w)
        self.q, self.k, self.v = W.bf16_to_f32(q), W.bf16_to_f32(k), W.bf16_to_f32(v)
        self.u = W.make_u(w)
        X, self.wv = W.make_head(w)
        self.X = W.bf16_to_f32(X)
        self.kk = oracle.dense_count(w.N, w.rho)
        self.n_tokens = min(n_tokens, w.N)
        self.rng = np.random.default_rng(seed)

    def step(self):
        """Routes the whole sample, then attention + head for a token sample."""
        o, w = self.oracle, self.w
        dense, _, _ = o.route(self.u[:1], self.kk)
        toks = self.rng.choice(w.N, size=self.n_tokens, replace=False)
        rows = (np.arange(w.H)[:, None] * w.N + toks[None, :]).ravel().astype(np.int64)
        o.attention_rows(self.q[:1], self.k[:1], self.v[:1], w.grid, w.win, dense, rows)
        o.uncertainty(self.X[:1, toks], self.wv)
        return self.n_tokens

    def describe(self):
        return ("%d of %d tokens of one sample (random), all %d heads, at the workload's own "
                "dense/local mix; routing over the full sample; head on the sampled tokens"
                % (self.n_tokens, self.w.N, self.w.H))


def run_reference(args, info):
    import oracle
    if info.rank != 0:
        return 0
    w = chosen_workload(args)
    s = OracleSample(w, n_tokens=max(16, args.cpu_tokens // 6))
    for _ in range(args.warmup):
        s.step()
    t0 = time.perf_counter()
    toks = 0
    for _ in range(args.steps):
        toks += s.step()
    dt = time.perf_counter() - t0
    value = toks / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": s.describe()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(args, w):
    """The oracle on repeated token samples until at least --cpu-seconds have passed."""
    import oracle
    s = OracleSample(w, n_tokens=args.cpu_tokens)
    s.step()  # warm: page in, build
    t0 = time.perf_counter()
    n = reps = 0
    while True:
        n += s.step()
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= args.cpu_seconds:
            break
    return {"value": n / dt, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": "%d repetitions of: %s" % (reps, s.describe()), "seconds": dt}


def profiled_traffic(workload_name):
    """DRAM bytes per launch of attn_tc_kernel from the committed ncu summary --
    only when that summary covers this workload and was taken on the current
    kernel source (else None)."""
    import hashlib
    import re
    if workload_name != W.WAN21.name:
        return None
    src = os.path.join(ROOT, "uncertainty_routed_heterogeneous_b200", "csrc", "attention_tc.cu")
    prof = os.path.join(ROOT, "profiles", "attn_tc_kernel-wan2.1-1.3b-rho0.2.md")
    try:
        text = open(prof).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    m = re.search(r"source_sha256_16: (\w+)", text)
    b = re.search(r"dram_bytes_per_launch: (\d+)", text)
    if m and b and m.group(1) == sha:
        return int(b.group(1))
    return None


def config_of(w, n_gpus):
    k = math.ceil(round(w.rho * w.N, 9))
    return {"workload": w.name, "B": w.B, "H": w.H, "d": w.d,
            "grid": "x".join(map(str, w.grid)), "N": w.N, "window": "x".join(map(str, w.win)),
            "rho": w.rho, "k": k, "head_C": w.C, "u": w.u_kind,
            "l2": "inputs larger than L2 (Q/K/V/X %.0f MB per step)" % (
                (3 * w.B * w.H * w.N * w.d * 2 + w.B * w.N * w.C * 2) / 1e6),
            "parallelism": "dp%d: one independent sample per GPU" % n_gpus}


# ----------------------------------------------------------------------------
# parity of the timed output against the fp64 oracle (after the timed region)
# ----------------------------------------------------------------------------

TOL_MAX_ABS, TOL_MEAN_ABS = 2e-2, 2e-3


def parity_rows(w, dense_np, n_per_head, seed):
    """Flat output row ids (b*H + h)*N + i to check: n_per_head seeded random
    rows of every (b, h), every border class of the window clamp (the corners,
    edges and centre of the grid on each axis) in the first and last head, and
    the first and last three dense rows there."""
    T, Hg, Wg = w.grid
    rng = np.random.default_rng(seed)
    rows = set()
    for bh in range(w.B * w.H):
        n = min(n_per_head, w.N)
        rows.update(int(bh * w.N + i) for i in rng.choice(w.N, size=n, replace=False))
    edge = []
    for t in sorted({0, 1, T // 2, T - 2, T - 1}):
        for h in sorted({0, w.win[1] // 2, Hg // 2, Hg - 1 - w.win[1] // 2, Hg - 1}):
            for x in sorted({0, w.win[2] // 2, Wg // 2, Wg - 1 - w.win[2] // 2, Wg - 1}):
                if 0 <= t < T and 0 <= h < Hg and 0 <= x < Wg:
                    edge.append((t * Hg + h) * Wg + x)
    for b in range(w.B):
        for h in sorted({0, w.H - 1}):
            base = (b * w.H + h) * w.N
            rows.update(base + i for i in edge)
            d = dense_np[b]
            rows.update(base + int(i) for i in d[:3])
            rows.update(base + int(i) for i in d[-3:])
    return np.array(sorted(rows), np.int64)


def bf16_host_f32(t):
    """A bf16 tensor (any device) as float32 numpy (exact)."""
    import torch
    return W.bf16_to_f32(t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def parity_of(w, kk, u_np, q32, k32, v32, dense_t, local_t, out_t, n_per_head, seed):
    """The routing lists bit for bit, and sampled output rows within the
    tolerance, against the oracle on the same inputs."""
    import oracle
    od, ol, _ = oracle.route(u_np, kk)
    routing_exact = bool(np.array_equal(dense_t.cpu().numpy(), od) and
                         (local_t is None or np.array_equal(local_t.cpu().numpy(), ol)))
    rows = parity_rows(w, od, n_per_head, seed)
    got = bf16_host_f32(out_t).reshape(-1, w.d)[rows]
    want = oracle.attention_rows(q32, k32, v32, w.grid, w.win, od, rows)
    err = np.abs(got.astype(np.float64) - want)
    mx = float(err.max()) if err.size else 0.0
    mean = float(err.mean()) if err.size else 0.0
    return {"max_abs": mx, "mean_abs": mean, "rows": int(rows.size),
            "rows_per_head": n_per_head, "routing_exact": routing_exact,
            "within_tolerance": bool(np.all(np.isfinite(got)) and mx <= TOL_MAX_ABS and
                                     mean <= TOL_MEAN_ABS),
            "tolerance": {"max_abs": TOL_MAX_ABS, "mean_abs": TOL_MEAN_ABS}}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------


def _time_ms(torch, fn, reps=5):
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def other_configs(heta, torch, dev, d_Q, d_K, d_V, out):
    """The Wan2.2-5B shape, the batched two-sample step with the head, the
    Wan2.1 layer at 720p (21x45x80 = 75600 tokens), and the rho sweep on
    uniform and clustered u at the Wan2.1 shape: CUDA-event times
    of the same calls as the main step (Q/K/V/X iid N(0,1) bf16 drawn on the
    device from a seeded generator; u from the workload's own generator)."""
    res = {}
    g = torch.Generator(device=dev)
    g.manual_seed(11)

    def randn_bf16(*shape):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)

    def one_step(w, Q, K, V, X, wv, u, n_check):
        kk = heta.dense_count(w.N, w.rho)
        dense = torch.empty((w.B, kk), dtype=torch.int32, device=dev)
        local = torch.empty((w.B, w.N - kk), dtype=torch.int32, device=dev)
        o = torch.empty_like(Q)
        ws = torch.empty(heta.attention_workspace_size(w.B, w.H, w.d, w.grid, w.win, kk),
                         dtype=torch.uint8, device=dev)
        u_next = torch.empty((w.B, w.N), dtype=torch.float32, device=dev)
        t_route = _time_ms(torch, lambda: heta.route(u, kk, out=(dense, local, None, None)))
        t_attn = _time_ms(torch, lambda: heta.attention(Q, K, V, w.grid, w.win, dense, out=o,
                                                         workspace=ws))
        t_head = _time_ms(torch, lambda: heta.uncertainty(X, wv, 0.0, out=u_next))
        fl = heta.attention_flops(w.B, w.H, w.d, w.N, kk, w.M)
        hbytes = 2 * w.B * w.N * w.C + 4 * w.C + 4 * w.B * w.N
        ms = t_route + t_attn + t_head
        torch.cuda.synchronize()
        par = parity_of(w, kk, u.cpu().numpy(), bf16_host_f32(Q), bf16_host_f32(K),
                        bf16_host_f32(V), dense, local, o, n_check, 5)
        return {"B": w.B, "H": w.H, "N": w.N, "k": kk, "route_ms": t_route,
                "attention_ms": t_attn, "head_ms": t_head,
                "tokens_per_s": w.B * w.N / (ms / 1e3),
                "attention_tflops": fl / (t_attn * 1e9),
                "head_gbs": hbytes / (t_head * 1e6), "parity": par}

    for w in (W.WAN22, W.BATCHED, W.WAN21_720P):
        Q, K, V = (randn_bf16(w.B, w.H, w.N, w.d) for _ in range(3))
        X = randn_bf16(w.B, w.N, w.C)
        wv = torch.from_numpy(W.make_head(W.scaled(w, B=1, grid=(1, 1, 8)))[1]).to(dev)
        u = torch.from_numpy(W.make_u(w)).to(dev)
        res[w.name] = one_step(w, Q, K, V, X, wv, u, 256)
        del Q, K, V, X
    sweep = {}
    q32, k32, v32 = bf16_host_f32(d_Q), bf16_host_f32(d_K), bf16_host_f32(d_V)
    for kind in ("uniform", "clustered"):
        # uniform u also at the two ends: LOCAL items only (rho = 0) and
        # DENSE items only (rho = 1)
        for rho in W.SWEEP_RHOS + ((0.0, 1.0) if kind == "uniform" else ()):
            w = W.sweep(rho, kind)
            kk = heta.dense_count(w.N, rho)
            u_np = W.make_u(w)
            u = torch.from_numpy(u_np).to(dev)
            dense, local, _, _ = heta.route(u, kk)
            ws = torch.empty(heta.attention_workspace_size(w.B, w.H, w.d, w.grid, w.win, kk),
                             dtype=torch.uint8, device=dev)
            t = _time_ms(torch, lambda: heta.attention(d_Q, d_K, d_V, w.grid, w.win, dense,
                                                        out=out, workspace=ws))
            fl = heta.attention_flops(w.B, w.H, w.d, w.N, kk, w.M)
            torch.cuda.synchronize()
            sweep["%s-rho%.2f" % (kind, rho)] = {
                "attention_ms": t, "algorithmic_tflops": fl / (t * 1e9),
                "parity": parity_of(w, kk, u_np, q32, k32, v32, dense, local, out, 256, 6)}
    res["rho_sweep_wan2.1"] = sweep
    return res


def flex_mask_mod(torch, perm, k, grid, win):
    """FlexAttention mask of the heterogeneous attention with the query rows
    permuted dense-first (perm = dense ids, then local ids): query position q
    attends to every key when q < k, else to the keys of the clamped window of
    its token perm[q] (start = clamp(p - w // 2, 0, extent - w) per axis)."""
    Tg, Hg, Wg = grid
    wt, wh, ww = win
    HW = Hg * Wg

    def mask_mod(b, h, q_idx, kv_idx):
        tok = perm[q_idx]
        t, hh, x = tok // HW, (tok // Wg) % Hg, tok % Wg
        tk, hk, xk = kv_idx // HW, (kv_idx // Wg) % Hg, kv_idx % Wg
        st = torch.clamp(t - wt // 2, 0, Tg - wt)
        sh = torch.clamp(hh - wh // 2, 0, Hg - wh)
        sx = torch.clamp(x - ww // 2, 0, Wg - ww)
        inwin = ((tk >= st) & (tk < st + wt) & (hk >= sh) & (hk < sh + wh) &
                 (xk >= sx) & (xk < sx + ww))
        return (q_idx < k) | inwin

    return mask_mod


def flex_compare(heta, torch, dev, w, d_Q, d_K, d_V, dense, local, ours, ours_ms):
    """The same heterogeneous mask realised with PyTorch FlexAttention, the
    paper's latency instrument (Where Compute Matters, §4 "Compute Complexity
    Assessment"; Table 5 counts the BlockMask construction in).  A comparison
    point only: the query rows are permuted so the dense ones come first (the
    dense query blocks then attend to every key block and the local ones to the
    key blocks their windows reach), the block mask is built from the routing,
    flex_attention runs the compiled block-sparse kernel, and the rows are put
    back in token order.  Returns times, the speedup of our kernel and the
    largest difference between the two outputs on the same inputs."""
    import time as _time

    from torch.nn.attention.flex_attention import create_block_mask, flex_attention
    k = dense.shape[1]
    perm = torch.cat([dense[0], local[0]]).to(torch.int64)
    mask_mod = flex_mask_mod(torch, perm, k, w.grid, w.win)
    flex = torch.compile(flex_attention, dynamic=False)
    make_mask = torch.compile(create_block_mask)
    t0 = _time.perf_counter()
    bm = make_mask(mask_mod, 1, None, w.N, w.N, device=dev)
    Qp = d_Q.index_select(2, perm)
    res = flex(Qp, d_K, d_V, block_mask=bm)
    out = torch.empty_like(d_Q)
    out.index_copy_(2, perm, res)
    torch.cuda.synchronize()
    compile_s = _time.perf_counter() - t0

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    mask_ms = timed(lambda: make_mask(mask_mod, 1, None, w.N, w.N, device=dev))
    attn_ms = timed(lambda: flex(Qp, d_K, d_V, block_mask=bm))

    def whole():
        b2 = make_mask(mask_mod, 1, None, w.N, w.N, device=dev)
        r = flex(d_Q.index_select(2, perm), d_K, d_V, block_mask=b2)
        out.index_copy_(2, perm, r)
    total_ms = timed(whole)
    diff = float((out.float() - ours.float()).abs().max())
    fl = heta.attention_flops(w.B, w.H, w.d, w.N, k, w.M)
    return {"what": "torch FlexAttention (compiled, block size 128) on the same mask, query "
                    "rows permuted dense-first; a comparison point, not the product",
            "blockmask_ms": mask_ms, "flex_attention_ms": attn_ms,
            "total_ms_with_blockmask_and_permutation": total_ms,
            "algorithmic_tflops_of_flex": fl / (attn_ms * 1e9),
            "ours_attention_ms": ours_ms, "speedup_ours_vs_flex_total": total_ms / ours_ms,
            "speedup_ours_vs_flex_kernel": attn_ms / ours_ms,
            "max_abs_diff_vs_ours": diff, "first_call_s": compile_s,
            "sparsity_of_blockmask": float(bm.sparsity()) if hasattr(bm, "sparsity") else None}


def run_heta(args, info):
    import torch

    import uncertainty_routed_heterogeneous_b200 as heta

    torch.cuda.set_device(info.local_rank)
    dev = torch.device("cuda", info.local_rank)
    D.init("nccl", info, timeout_s=300)
    heta.load()
    base = chosen_workload(args)
    w = D.rank_workload(base, info.rank)

    # ---- inputs: host (pinned) and resident device copies -------------------
    def pinned_bf16(bits):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()

    q, k, v = W.make_qkv(w)
    X, wv = W.make_head(w)
    u = W.make_u(w)
    h_Q, h_K, h_V, h_X = (pinned_bf16(a) for a in (q, k, v, X))
    del q, k, v, X
    h_u = torch.from_numpy(u).pin_memory()
    h_w = torch.from_numpy(wv)
    d_Q, d_K, d_V, d_X = (t.to(dev) for t in (h_Q, h_K, h_V, h_X))
    d_u = h_u.to(dev)
    d_w = h_w.to(dev)
    kk = heta.dense_count(w.N, w.rho)
    dense = torch.empty((w.B, kk), dtype=torch.int32, device=dev)
    local = torch.empty((w.B, w.N - kk), dtype=torch.int32, device=dev)
    out = torch.empty_like(d_Q)
    ws = torch.empty(heta.attention_workspace_size(w.B, w.H, w.d, w.grid, w.win, kk),
                     dtype=torch.uint8, device=dev)
    u_next = torch.empty((w.B, w.N), dtype=torch.float32, device=dev)
    h_out = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    h_unext = torch.empty(u_next.shape, dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()

    nvtx = torch.cuda.nvtx if args.nvtx else None

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        if nvtx:
            nvtx.range_push("heta_route")
        heta.route(d_u, kk, out=(dense, local, None, None))
        if ev is not None:
            ev[1].record()
        if nvtx:
            nvtx.range_pop()
            nvtx.range_push("heta_attention")
        heta.attention(d_Q, d_K, d_V, w.grid, w.win, dense, out=out, workspace=ws)
        if ev is not None:
            ev[2].record()
        if nvtx:
            nvtx.range_pop()
            nvtx.range_push("heta_uncertainty")
        heta.uncertainty(d_X, d_w, 0.0, out=u_next)
        if ev is not None:
            ev[3].record()
        if nvtx:
            nvtx.range_pop()

    # route, the persistent attention kernel, the head (plus one workspace memset)
    launches_per_step = 3
    flops = heta.attention_flops(w.B, w.H, w.d, w.N, kk, w.M)

    sampler = ClockSampler(info.local_rank)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    D.barrier(info, dev)
    torch.cuda.synchronize()
    sampler.start()
    t_start.record()
    for i in range(args.steps):
        step(evs[i])
    t_end.record()
    torch.cuda.synchronize()
    sampler.stop()
    D.barrier(info, dev)
    ms_local = t_start.elapsed_time(t_end)
    ms_total = D.max_over_ranks(ms_local, info, dev)
    route_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    head_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    tokens_per_step = w.B * w.N * info.world
    value = tokens_per_step * args.steps / (ms_total / 1e3)
    # the last timed step's routing and output, checked against the oracle
    # once all timing is done
    timed = (dense.cpu(), local.cpu(), out.cpu())

    # ---- the same step captured once in a CUDA graph and replayed ---------------
    graph = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        g_ms = e0.elapsed_time(e1) / args.steps
        graph = {"ms_per_step": g_ms, "tokens_per_s": w.B * w.N / (g_ms / 1e3),
                 "what": "route + attention + head captured once in a CUDA graph, replayed "
                         "%d times (the timed line above launches them eagerly)" % args.steps}
        del g
    except Exception as e:  # noqa: BLE001 -- an extra measurement never fails the bench
        graph = {"unavailable": "%s: %s" % (type(e).__name__, str(e)[:300])}
    torch.cuda.synchronize()

    # ---- the same mask through PyTorch FlexAttention (comparison point) -------
    flex = None
    if not args.no_flex_compare and info.rank == 0:
        try:
            heta.attention(d_Q, d_K, d_V, w.grid, w.win, dense, out=out, workspace=ws)
            torch.cuda.synchronize()
            flex = flex_compare(heta, torch, dev, w, d_Q, d_K, d_V, dense, local, out, attn_ms)
        except Exception as e:  # noqa: BLE001 -- a comparison leg never fails the bench
            flex = {"unavailable": "%s: %s" % (type(e).__name__, str(e)[:300])}
        torch.cuda.synchronize()

    # ---- our own full dense attention (rho = 1) at the same shape -----------
    dense_cmp = None
    if not args.no_dense_compare:
        all_idx = torch.arange(w.N, dtype=torch.int32, device=dev).repeat(w.B, 1).contiguous()
        ws_full = torch.empty(heta.attention_workspace_size(w.B, w.H, w.d, w.grid, w.win, w.N),
                              dtype=torch.uint8, device=dev)
        heta.attention(d_Q, d_K, d_V, w.grid, w.win, all_idx, out=out, workspace=ws_full)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        e0.record()
        for _ in range(reps):
            heta.attention(d_Q, d_K, d_V, w.grid, w.win, all_idx, out=out, workspace=ws_full)
        e1.record()
        torch.cuda.synchronize()
        full_ms = e0.elapsed_time(e1) / reps
        full_flops = heta.attention_flops(w.B, w.H, w.d, w.N, w.N, w.M)
        dense_cmp = {"ms": full_ms, "tflops": full_flops / (full_ms * 1e9),
                     "speedup_of_routed": full_ms / attn_ms}

    # ---- the paper's window ablation sizes (Table 7) on the same inputs -------
    win_sweep = None
    if not args.no_window_sweep:
        win_sweep = {}
        for n in W.WINDOW_CUBES:
            wn = W.window_cube(n)
            ws_n = torch.empty(heta.attention_workspace_size(w.B, w.H, w.d, w.grid, wn.win, kk),
                               dtype=torch.uint8, device=dev)
            heta.attention(d_Q, d_K, d_V, w.grid, wn.win, dense, out=out, workspace=ws_n)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            e0.record()
            for _ in range(reps):
                heta.attention(d_Q, d_K, d_V, w.grid, wn.win, dense, out=out, workspace=ws_n)
            e1.record()
            torch.cuda.synchronize()
            ms_n = e0.elapsed_time(e1) / reps
            fl_n = heta.attention_flops(w.B, w.H, w.d, w.N, kk, wn.M)
            win_sweep["x".join(map(str, wn.win))] = {
                "attention_ms": ms_n, "algorithmic_tflops": fl_n / (ms_n * 1e9),
                "speedup_vs_dense": (dense_cmp["ms"] / ms_n) if dense_cmp else None}
        del ws_n

    # ---- the other configurations, timed the same way on fresh inputs -------
    others = None
    if not args.no_other_configs and info.rank == 0 and w.name == W.WAN21.name:
        others = other_configs(heta, torch, dev, d_Q, d_K, d_V, out)

    # ---- the paper's own threshold rule, T = mu + c*sigma (Eq. (11)), c = 0.9 --
    thr = None
    if not args.no_threshold_mode:
        c = 0.9
        t_counts = torch.empty(w.B, dtype=torch.int32, device=dev)
        t_dense = torch.empty((w.B, w.N), dtype=torch.int32, device=dev)
        t_local = torch.empty((w.B, w.N), dtype=torch.int32, device=dev)
        ws_t = torch.empty(heta.attention_counts_workspace_size(w.B, w.H, w.d, w.grid, w.win,
                                                                w.N),
                           dtype=torch.uint8, device=dev)

        def thr_step(ev=None):
            if ev is not None:
                ev[0].record()
            heta.route_threshold(d_u, c, out=(t_counts, t_dense, t_local, None, None))
            if ev is not None:
                ev[1].record()
            heta.attention_counts(d_Q, d_K, d_V, w.grid, w.win, t_dense, t_counts, out=out,
                                  workspace=ws_t)
            if ev is not None:
                ev[2].record()

        for _ in range(3):
            thr_step()
        torch.cuda.synchronize()
        tev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(10)]
        for ev in tev:
            thr_step(ev)
        torch.cuda.synchronize()
        cnt = t_counts.cpu().tolist()
        r_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in tev)
        a_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in tev)
        fl_t = sum(heta.attention_flops(1, w.H, w.d, w.N, kb, w.M) for kb in cnt)
        thr = {"c": c, "dense_counts": cnt, "dense_fraction": sum(cnt) / (w.B * w.N),
               "route_ms": r_ms, "attention_ms": a_ms,
               "algorithmic_tflops": fl_t / (a_ms * 1e9),
               "tokens_per_s": w.B * w.N / ((r_ms + a_ms) / 1e3)}
        del ws_t

    # ---- the per-block random swap (Table 8: r = 7% of N) on this routing -----
    swap = None
    if not args.no_threshold_mode:
        s_sw = heta.swap_count(w.N, kk, 0.07)
        sw_d = torch.empty_like(dense)
        sw_l = torch.empty_like(local)
        heta.route(d_u, kk, out=(dense, local, None, None))
        for _ in range(3):
            heta.route_swap(dense, w.N, s_sw, 2024, 0, out=(sw_d, sw_l, None))
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 20
        e0.record()
        for blk in range(reps):
            heta.route_swap(dense, w.N, s_sw, 2024, blk, out=(sw_d, sw_l, None))
        e1.record()
        torch.cuda.synchronize()
        us_one = 1e3 * e0.elapsed_time(e1) / reps
        # all 30 blocks of a step (Wan2.1-1.3B has 30) in one launch
        nb = 30
        bd = torch.empty((nb,) + tuple(dense.shape), dtype=torch.int32, device=dev)
        bl = torch.empty((nb,) + tuple(local.shape), dtype=torch.int32, device=dev)
        for _ in range(3):
            heta.route_swap_blocks(dense, w.N, s_sw, 2024, 0, nb, out=(bd, bl, None))
        torch.cuda.synchronize()
        e0.record()
        for _ in range(5):
            heta.route_swap_blocks(dense, w.N, s_sw, 2024, 0, nb, out=(bd, bl, None))
        e1.record()
        torch.cuda.synchronize()
        us_all = 1e3 * e0.elapsed_time(e1) / 5
        swap = {"r": 0.07, "s": s_sw, "us_per_block": us_one,
                "blocks_in_one_launch": nb, "us_all_blocks": us_all,
                "us_per_block_batched": us_all / nb}
        del bd, bl

    # ---- routing in throughput mode: many samples of this N in one launch ------
    # 512 samples, and a whole number of samples per SM (4 x the SM count), so
    # that no SM runs a last sample alone
    route_tp = None
    if not args.no_route_throughput:
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        hbm = load_peaks()["hbm_gbs"]
        g = torch.Generator(device=dev)
        g.manual_seed(7)
        runs = {}
        for Bt in (512, 4 * sms):
            u_tp = (d_u[:1].repeat(Bt, 1) +
                    1e-3 * torch.randn((Bt, w.N), generator=g, device=dev)).contiguous()
            dn_tp = torch.empty((Bt, kk), dtype=torch.int32, device=dev)
            lc_tp = torch.empty((Bt, w.N - kk), dtype=torch.int32, device=dev)
            for _ in range(3):
                heta.route(u_tp, kk, out=(dn_tp, lc_tp, None, None))
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 20
            e0.record()
            for _ in range(reps):
                heta.route(u_tp, kk, out=(dn_tp, lc_tp, None, None))
            e1.record()
            torch.cuda.synchronize()
            us = 1e3 * e0.elapsed_time(e1) / reps
            nbytes = Bt * w.N * 4 * 2  # read u once, write both index lists
            runs[Bt] = {"B": Bt, "N": w.N, "k": kk, "us": us, "bytes": nbytes,
                        "GB/s": nbytes / (us * 1e3), "frac_of_hbm": nbytes / (us * 1e3) / hbm}
            del u_tp, dn_tp, lc_tp
        route_tp = dict(runs[512])
        route_tp["full_waves"] = runs[4 * sms]
        route_tp["peak_source"] = "measured copy bandwidth"

    # ---- end to end through the public API with host buffers ----------------
    # Every step copies its inputs from pinned host memory and reads its
    # results (out, next u) back.  Three streams pipeline the steps: the
    # inputs of step i+1 travel while step i computes and step i-1's results
    # come back; two device copies of the inputs and outputs alternate.
    e2e = None
    if not args.no_e2e:
        ke = max(2, min(args.steps, 20))
        s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
        sets = [dict(Q=d_Q, K=d_K, V=d_V, X=d_X, u=d_u, out=out, un=u_next)]
        sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
        h_outs = [h_out, torch.empty_like(h_out).pin_memory()]
        h_uns = [h_unext, torch.empty_like(h_unext).pin_memory()]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            j = i % 2
            bs = sets[j]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[j])  # step i-2 has read these inputs
                for n, h in (("Q", h_Q), ("K", h_K), ("V", h_V), ("X", h_X), ("u", h_u)):
                    bs[n].copy_(h, non_blocking=True)
                ev_in[j].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[j])
                if i >= 2:
                    s_cmp.wait_event(ev_out[j])  # step i-2's results are back
                heta.route(bs["u"], kk, out=(dense, local, None, None))
                heta.attention(bs["Q"], bs["K"], bs["V"], w.grid, w.win, dense, out=bs["out"],
                               workspace=ws)
                heta.uncertainty(bs["X"], d_w, 0.0, out=bs["un"])
                ev_cmp[j].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[j])
                h_outs[j].copy_(bs["out"], non_blocking=True)
                h_uns[j].copy_(bs["un"], non_blocking=True)
                ev_out[j].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        D.barrier(info, dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(ke):
            e2e_step(i)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = D.max_over_ranks(e0.elapsed_time(e1), info, dev)
        h2d = sum(t.numel() * t.element_size() for t in (h_Q, h_K, h_V, h_X, h_u))
        d2h = sum(t.numel() * t.element_size() for t in (h_out, h_unext))
        e2e = {"value": tokens_per_step * ke / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ke,
               "pipelined": "inputs of the next step copied while this one computes"}
        del sets

    cpu = None
    if info.rank == 0 and info.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, base)
    parity = None
    if info.rank == 0:
        parity = parity_of(w, kk, u, bf16_host_f32(h_Q), bf16_host_f32(h_K), bf16_host_f32(h_V),
                           *timed, 4096, 1)
        parity["checked"] = ("the last timed step: dense/local lists bit for bit; %d output "
                             "rows (4096 random per head, every border class and the first "
                             "and last dense rows) against the fp64 oracle" % parity["rows"])

    sampler.close()
    if info.rank != 0:
        return 0
    peaks = load_peaks()
    tflops = flops / (attn_ms * 1e9)
    # the timed region (tens of ms) runs at the full SM clock (see "clocks"),
    # so the burst GEMM figure is the peak; the power-capped sustained one is
    # reported beside it
    peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": info.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; Wan2.1-1.3B latent shape; no model weights)",
        "config": config_of(base, info.world),
        "attention_tflops": tflops,
        "kernel_ms": {"route": route_ms, "attention": attn_ms, "head": head_ms},
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (persistent; dense + local items)",
                     "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak,
                     "frac_of_sustained": tflops / peaks["bf16_tflops_sustained"],
                     "peak_source": "%s burst bf16 (cuBLAS)" % peaks["source"],
                     "traffic": profiled_traffic(base.name), "traffic_unit": "bytes/launch",
                     "algorithmic_flops": flops},
        "head_roofline": {"bound": "hbm",
                          "achieved": (w.B * w.N * w.C * 2 + w.C * 4 + w.B * w.N * 4) /
                          (head_ms * 1e6),
                          "peak": peaks["hbm_gbs"], "unit": "GB/s"},
        "dense_compare": dense_cmp,
        "flex_compare": flex,
        "graph_replay": graph,
        "window_sweep": win_sweep,
        "other_configs": others,
        "threshold_mode": thr,
        "route_throughput": route_tp,
        "route_swap": swap,
        "parity": parity,
        "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
        "cpu_baseline": cpu, "clocks": sampler.summary(),
    }
    line["head_roofline"]["frac"] = line["head_roofline"]["achieved"] / peaks["hbm_gbs"]
    print(json.dumps(line), flush=True)
    return 0


def run_heta_heads(args, info):
    """One sample split over the ranks by heads (strong scaling): every rank
    routes the sample's full u itself, runs attention on its head block and
    the uncertainty head on its block of token rows; the next step's u, which
    every rank needs, is all-gathered (NCCL); optionally the output too."""
    import torch

    import uncertainty_routed_heterogeneous_b200 as heta

    torch.cuda.set_device(info.local_rank)
    dev = torch.device("cuda", info.local_rank)
    D.init("nccl", info, timeout_s=300)
    heta.load()
    w = chosen_workload(args)
    if w.B != 1:
        raise SystemExit("--shard heads takes one sample (B = 1)")
    if (w.B * w.N) % info.world:
        raise SystemExit("--shard heads needs the token count divisible by the rank count")
    h0, h1 = D.head_range(w.H, info.world, info.rank)
    r0, r1 = D.row_range(w.B * w.N, info.world, info.rank)

    def dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    q, k, v = W.make_qkv(w)
    d_Q, d_K, d_V = (dev_bf16(a[:, h0:h1]) for a in (q, k, v))
    del q, k, v
    X, wv = W.make_head(w)
    d_X = dev_bf16(X.reshape(1, w.B * w.N, w.C)[:, r0:r1])
    del X
    d_w = torch.from_numpy(wv).to(dev)
    d_u = torch.from_numpy(W.make_u(w)).to(dev)
    kk = heta.dense_count(w.N, w.rho)
    Hl = h1 - h0
    dense = torch.empty((w.B, kk), dtype=torch.int32, device=dev)
    local = torch.empty((w.B, w.N - kk), dtype=torch.int32, device=dev)
    out = torch.empty_like(d_Q)
    ws = torch.empty(max(256, heta.attention_workspace_size(w.B, Hl, w.d, w.grid, w.win, kk)),
                     dtype=torch.uint8, device=dev)
    u_rows = torch.empty((1, r1 - r0), dtype=torch.float32, device=dev)
    gather_out = args.gather_out and w.H % info.world == 0

    def step():
        heta.route(d_u, kk, out=(dense, local, None, None))
        if Hl > 0:
            heta.attention(d_Q, d_K, d_V, w.grid, w.win, dense, out=out, workspace=ws)
        heta.uncertainty(d_X, d_w, 0.0, out=u_rows)
        u_next = D.all_gather_equal(u_rows, info)
        if gather_out:
            D.all_gather_equal(out, info)
        return u_next

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(info.local_rank)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier(info, dev)
    torch.cuda.synchronize()
    sampler.start()
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    sampler.stop()
    D.barrier(info, dev)
    ms_total = D.max_over_ranks(t0.elapsed_time(t1), info, dev)
    sampler.close()
    if info.rank != 0:
        return 0
    value = w.B * w.N * args.steps / (ms_total / 1e3)
    cfg = config_of(w, info.world)
    cfg["parallelism"] = ("heads%d: one sample's %d heads split over %d GPUs, u of the next "
                          "step all-gathered%s" % (info.world, w.H, info.world,
                                                    ", output all-gathered" if gather_out
                                                    else ""))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": info.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded; Wan2.1-1.3B latent shape)",
            "config": cfg, "gpu_launches": (3 if Hl > 0 else 2) * args.steps,
            "clocks": sampler.summary()}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    info = D.rank_info()
    if args.impl == "reference":
        return run_reference(args, info)
    if args.shard == "heads":
        rc = run_heta_heads(args, info)
    else:
        rc = run_heta(args, info)
    if info.world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
