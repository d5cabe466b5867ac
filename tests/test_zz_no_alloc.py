"""The allocation-free GEMV entry point (hgd_gemv_bf16_static_ws).

It serves callers that cannot allocate device memory, for instance a plugin whose
host framework owns every device allocation, or a decode loop that cannot afford
the device synchronisation a cudaMalloc brings.  Its split-K scratch is an array
built into the library instead of a caller workspace.  These checks call it
through the C ABI and compare it with hgd_gemv_bf16 (which takes a workspace) on
two calls in a row, since every call reuses the same built-in array.  This file
is collected last, so that a run stopping at its first failure has already run
every other test.
"""
import ctypes as C

import numpy as np
import pytest

import hgd_synth as syn
from helpers import assert_bf16_close, dev_bf16, fp32_dot_bound, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hgd():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import __graft_entry__ as g
    g.build()
    import hybrid_gated_delta_b200 as m
    return m


def _static(hgd, W, x, y, fp32):
    import torch
    M, K = x.shape
    N = W.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    return hgd._lib.hgd_gemv_bf16_static_ws(W.data_ptr(), x.data_ptr(), y.data_ptr(), int(fp32), M, N, K,
                                            stream)


@pytest.mark.parametrize("N,K,M", [(1024, 2048, 1), (1024, 3584, 8), (1500, 1024, 3), (8224, 1024, 1)])
def test_static_scratch_matches_workspace_entry_point(hgd, N, K, M):
    import torch
    c = syn.gemv_case(N, K, M, seed=21)
    W, x = dev_bf16(c["W"]), dev_bf16(c["x"])
    ws = hgd.make_workspace(M, N, K)
    assert ws is not None  # these shapes spread K over SMs, so the scratch is really used
    ref32 = hgd.gemv_bf16(W, x, workspace=ws)
    ref16 = hgd.gemv_bf16(W, x, y_is_fp32=False, workspace=ws)
    for _ in range(2):  # the built-in array keeps the previous call's contents
        y32 = torch.full((M, N), float("nan"), device="cuda")
        y16 = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
        assert _static(hgd, W, x, y32, True) == 0
        assert _static(hgd, W, x, y16, False) == 0
        torch.cuda.synchronize()
        bound = fp32_dot_bound(c["W"], c["x"])
        assert np.all(np.abs(host(y32) - host(ref32)) <= 2 * bound + 1e-30)
        assert_bf16_close(host(y16), host(ref16), "static scratch bf16")
        # the same arithmetic as the workspace entry point: equal bits
        assert torch.equal(y32, ref32) and torch.equal(y16.view(torch.int16), ref16.view(torch.int16))


def test_static_scratch_rejects_shapes_beyond_its_size(hgd):
    import torch
    N, K, M = 32752, 4096, 8   # 2047 row blocks x 16 slabs: about 16.8 MB of split-K scratch
    n = C.c_size_t()
    assert hgd._lib.hgd_gemv_workspace_bytes(M, N, K, 0, C.byref(n)) == 0
    assert n.value > (4 << 20)
    # buffers of the declared shape (W is 268 MB), so that even if the size check
    # ever stopped rejecting this shape, the launch would stay inside them
    W = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.full((M, N), 7.0, device="cuda")
    rc = hgd._lib.hgd_gemv_bf16_static_ws(W.data_ptr(), x.data_ptr(), y.data_ptr(), 1, M, N, K,
                                          torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 9  # HGD_ERR_BUFFER_TOO_SMALL
    assert bool((y == 7.0).all())  # a rejected call writes nothing
