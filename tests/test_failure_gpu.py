"""Failure detection on the GPU without a fault.

Every wait inside the library's kernels is bounded: it gives up after a
wall-time limit, or as soon as another thread of the CTA has raised the abort
flag, and the kernel reports HETA_ERR_TIMEOUT through status_dev and returns.
heta_selftest_wait_timeout drives that path on purpose (a barrier nothing
completes), so these tests check the status, the abort hand-off between
warps, and that the context stays usable afterwards.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports(gpu_lib):
    import torch
    heta = gpu_lib
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    el = torch.zeros(1, dtype=torch.int64, device="cuda")
    heta.selftest_wait_timeout(50_000_000, st, el)  # 50 ms
    torch.cuda.synchronize()
    assert int(st.item()) == heta.HETA_ERR_TIMEOUT
    ns = int(el.item())
    # the first wait ran its limit out; the second (5 s limit) was released
    # by the abort flag right after
    assert 50_000_000 <= ns < 2_000_000_000, ns


def test_context_usable_after_timeout(gpu_lib):
    import torch
    heta = gpu_lib
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    heta.selftest_wait_timeout(10_000_000, st)
    torch.cuda.synchronize()
    assert int(st.item()) == heta.HETA_ERR_TIMEOUT
    # the next launches work and report nothing
    u = torch.rand((1, 4096), device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    dense, local, _, _ = heta.route(u, 800, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    want = torch.topk(u[0].double(), 800).indices.sort().values.to(torch.int32)
    assert torch.equal(dense[0], want)


def test_selftest_rejects_bad_limits(gpu_lib):
    import torch
    heta = gpu_lib
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, 11_000_000_000):
        with pytest.raises(heta.HetaError):
            heta.selftest_wait_timeout(bad, st)
