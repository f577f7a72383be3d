"""The plain-C program examples/heta_run.c on the GPU: one step of the path
(route -> attention -> head) driven through include/heta.h and libheta.so
alone, its outputs against the fp64 oracle on the same inputs.

"Where Compute Matters: Heterogeneous Attention for Efficient Video
Diffusion": Eq. (11)-(12) routing (bit for bit), Eq. (2), (3), (13)
attention (max abs <= 2e-2, mean abs <= 2e-3), Eq. (7) head
(|u - u_oracle| <= 1e-5 (1 + |u|)).
"""
import dataclasses
import subprocess

import numpy as np
import pytest

import oracle
from helpers import assert_close
from uncertainty_routed_heterogeneous_b200 import build as heta_build
from uncertainty_routed_heterogeneous_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_c_program_step_matches_the_oracle(gpu_lib, tmp_path):
    w = dataclasses.replace(W.scaled(W.WAN21, B=2, H=2, grid=(5, 12, 20), u_kind="uniform",
                                     u_seeds=(5, 6), C=512), name="c-example")
    q, k, v = W.make_qkv(w)
    u = W.make_u(w)
    X, wv = W.make_head(w)
    (tmp_path / "meta.txt").write_text("%d %d %d %d %d %d %d %d %d %d %r\n" % (
        w.B, w.H, w.d, *w.grid, *w.win, w.C, w.rho))
    for name, a in (("q", q), ("k", k), ("v", v), ("x", X)):
        np.ascontiguousarray(a, np.uint16).tofile(tmp_path / (name + ".bin"))
    np.ascontiguousarray(u, np.float32).tofile(tmp_path / "u.bin")
    np.ascontiguousarray(wv, np.float32).tofile(tmp_path / "w.bin")

    exe = heta_build.build_example()
    r = subprocess.run([exe, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr

    kk = gpu_lib.dense_count(w.N, w.rho)
    od, ol, _ = oracle.route(u, kk)
    dense = np.fromfile(tmp_path / "dense.bin", np.int32).reshape(w.B, kk)
    local = np.fromfile(tmp_path / "local.bin", np.int32).reshape(w.B, w.N - kk)
    assert np.array_equal(dense, od) and np.array_equal(local, ol)

    got = W.bf16_to_f32(np.fromfile(tmp_path / "out.bin", np.uint16)).reshape(-1, w.d)
    assert not np.isnan(got).any()
    want = oracle.attention(W.bf16_to_f32(q), W.bf16_to_f32(k), W.bf16_to_f32(v), w.grid,
                            w.win, od).reshape(-1, w.d)
    assert_close(got, want, w.name)

    un = np.fromfile(tmp_path / "u_next.bin", np.float32).reshape(w.B, w.N)
    uref = oracle.uncertainty(W.bf16_to_f32(X), wv, 0.0)
    assert np.max(np.abs(un - uref) / (1 + np.abs(uref))) <= 1e-5
