"""bench.py's reference arm keeps the one-JSON-line contract, on the host.

The reference arm times the fp64 oracle on the host cores, so it runs here
without a GPU: at N = 1 it prints one line with the contract's keys, on the
same metric, unit and workload as the GPU arm; under torchrun with two ranks
rank 0 alone prints it and every rank exits 0.
"""
import json
import os
import socket
import subprocess
import sys

from uncertainty_routed_heterogeneous_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REQUIRED = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
            "cpu_baseline", "e2e"}


def _json_lines(text):
    return [json.loads(line) for line in text.splitlines() if line.startswith("{")]


def _bench_constants():
    consts = {}
    with open(os.path.join(ROOT, "bench.py")) as f:
        for line in f:
            for name in ("METRIC", "UNIT"):
                if line.startswith(name + " = "):
                    consts[name] = json.loads(line.split(" = ", 1)[1])
    return consts


def test_reference_line_at_one_rank():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "1", "--cpu-tokens", "96"],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert REQUIRED <= set(d)
    c = _bench_constants()
    assert d["impl"] == "reference"
    assert d["metric"] == c["METRIC"] and d["unit"] == c["UNIT"]
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 1, 1)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["config"]["workload"] == W.WAN21.name  # the GPU arm's default workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_line_under_torchrun_comes_from_rank_0_only():
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1",
                        "--workload", W.TINY.name],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
    assert lines[0]["config"]["workload"] == W.TINY.name


def test_flex_comparison_mask_is_the_oracles_mask():
    """The FlexAttention comparison in bench.py realises the same mask: run
    eagerly on CPU on a tiny grid (dense query rows first, as bench.py
    permutes them), put back in token order, it equals the fp64 oracle."""
    import numpy as np
    import torch
    from torch.nn.attention.flex_attention import create_block_mask, flex_attention

    import oracle
    sys.path.insert(0, ROOT)
    import bench
    w = W.scaled(W.WAN21, H=2, d=64, grid=(4, 6, 10), win=(3, 3, 5), u_kind="uniform",
                 u_seeds=(13,))
    q, k, v = (W.bf16_to_f32(a) for a in W.make_qkv(w))
    kk = oracle.dense_count(w.N, w.rho)
    dense, local, _ = oracle.route(W.make_u(w), kk)
    perm = torch.from_numpy(np.concatenate([dense[0], local[0]]).astype(np.int64))
    mask_mod = bench.flex_mask_mod(torch, perm, kk, w.grid, w.win)
    bm = create_block_mask(mask_mod, 1, None, w.N, w.N, device="cpu", BLOCK_SIZE=16)
    Q, K, V = (torch.from_numpy(a).double() for a in (q, k, v))
    res = flex_attention(Q.index_select(2, perm), K, V, block_mask=bm)
    out = torch.empty_like(Q)
    out.index_copy_(2, perm, res)
    want = oracle.attention(q, k, v, w.grid, w.win, dense)
    assert np.abs(out.numpy() - want).max() < 1e-9
