"""GPU parity of the tensor-core (tcgen05) GEMM for windows of token rows
against the CPU oracle's GEMV: every output within twice Higham's fp32
dot-product bound (both sides are fp32 sums of exact bf16 products), at shapes
that span several 128-row weight tiles and 64-wide K blocks with ragged N and M,
split K, and the window projections of the 24-layer stack at 128 token rows."""
import numpy as np
import pytest

import hgd_synth as syn
from helpers import dev_bf16, fp32_dot_bound, host

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


def _run(hgd, W, x, N, guard=64):
    """y through the C ABI into a NaN-guarded buffer; returns (y, guard intact)."""
    import torch
    M = x.shape[0]
    Wp = hgd.gemm_tc_pack_weight(W)
    torch.cuda.synchronize()
    buf = torch.full((M * N + guard,), float("nan"), device="cuda")
    y = buf[:M * N].view(M, N)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hgd.gemm_tc_bf16(Wp, x, N, y=y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y, bool(torch.isnan(buf[M * N:]).all().item()), Wp, status


SMALL = [(1000, 128, 1), (257, 1024, 16), (129, 3584, 128), (300, 640, 200), (2048, 2048, 256),
         (64, 64, 17), (4096, 1536, 33)]


@pytest.mark.parametrize("N,K,M", SMALL)
def test_gemm_tc_small(hgd, orc, N, K, M):
    import torch
    c = syn.gemv_case(N, K, M, seed=11)
    y, guard_ok, Wp, status = _run(hgd, dev_bf16(c["W"]), dev_bf16(c["x"]), N)
    assert guard_ok, "wrote past y"
    got = host(y)
    assert np.isfinite(got).all()
    ref = orc.gemv(c["W"], c["x"])
    bound = fp32_dot_bound(c["W"], c["x"])
    err = np.abs(got - ref)
    assert np.all(err <= 2 * bound + 1e-30), (err.max(), (err / (bound + 1e-30)).max())
    # the same call again: the same bits (fixed split, fixed order)
    y2 = torch.empty_like(y)
    hgd.gemm_tc_bf16(Wp, dev_bf16(c["x"]), N, y=y2, status=status)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


def test_gemm_tc_identity_is_exact(hgd):
    """W = I (one nonzero product per output): y = x exactly, every row and tile."""
    import torch
    K, M = 384, 144
    x = syn.gemv_case(K, K, M, seed=12)["x"]
    W = np.zeros((K, K), np.uint16)
    W[np.arange(K), np.arange(K)] = 0x3F80  # bf16 1.0
    y, guard_ok, _, _ = _run(hgd, dev_bf16(W), dev_bf16(x), K)
    assert guard_ok
    assert np.array_equal(host(y), syn.from_bf16(x).astype(np.float32))


def test_gemm_tc_rejects_bad_shapes(hgd):
    import torch
    W = torch.zeros((128, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hgd.HgdError):
        hgd.gemm_tc_pack_weight(W)  # K % 64
    Wp = hgd.gemm_tc_pack_weight(torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda"))
    x = torch.zeros((257, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hgd.HgdError):
        hgd.gemm_tc_bf16(Wp, x, 128)  # M > 256
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(hgd.HgdError):
        hgd.gemm_tc_bf16(Wp, x[:16], 128, workspace=small)


# the projections of an 8-stream x 16-row window of the 24-layer stack
WINDOW = {"gdn_in": (8224, 1024), "attn_in": (5120, 1024), "gdn_out": (1024, 2048), "gate_up": (7168, 1024),
          "down": (1024, 3584), "lm_head": (248320, 1024)}


@pytest.mark.parametrize("name", list(WINDOW))
def test_gemm_tc_window_shapes(hgd, orc, name):
    """M = 128 at full size; the oracle checks a sample of 512 output features
    (all of them below 2048)."""
    N, K = WINDOW[name]
    M = 128
    c = syn.gemv_case(N, K, M, seed=13)
    y, guard_ok, _, _ = _run(hgd, dev_bf16(c["W"]), dev_bf16(c["x"]), N)
    assert guard_ok
    cols = np.arange(N) if N <= 2048 else np.sort(syn.rng(6).choice(N, 512, replace=False))
    Ws = np.ascontiguousarray(c["W"][cols])
    ref = orc.gemv(Ws, c["x"])
    got = host(y)[:, cols]
    err = np.abs(got - ref)
    bound = fp32_dot_bound(Ws, c["x"])
    assert np.all(err <= 2 * bound + 1e-30), (name, err.max(), (err / (bound + 1e-30)).max())


@pytest.mark.parametrize("name", ["lm_head", "down", "gdn_in"])
def test_gemm_tc_rows_independent_of_m(hgd, name):
    """Each token row's result does not depend on how many rows the call carries
    (the property a window equal to its one-row steps rests on): the first M rows
    of a 200-row call, bit for bit, at M = 1 .. 128.  At 200 rows the LM-head
    shape runs one weight block per CTA, at 128 rows or fewer two blocks per CTA
    for its first waves and one for the rest: the same bits either way.  The split
    shapes (down: 8 splits in a cluster, gdn_in: 2) keep their split at every M."""
    import torch
    N, K = WINDOW[name]
    c = syn.gemv_case(N, K, 200, seed=17)
    W, x = dev_bf16(c["W"]), dev_bf16(c["x"])
    y_all, guard_ok, Wp, status = _run(hgd, W, x, N)
    assert guard_ok
    for M in (1, 8, 16, 100, 128):
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        hgd.gemm_tc_bf16(Wp, x[:M].contiguous(), N, y=y, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(y, y_all[:M]), (name, M)


def test_stuck_wait_reports_timeout_and_context_survives(hgd, orc):
    """A bounded in-kernel wait that nothing completes ends after its limit with
    HGD_ERR_TIMEOUT in the status word; the next calls still compute correctly."""
    import time
    import torch
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    hgd.check_bounded_wait(status)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status[0].item()) == 5  # HGD_ERR_TIMEOUT
    assert 1.0 < elapsed < 30.0, elapsed
    c = syn.gemv_case(257, 1024, 16, seed=14)
    y, guard_ok, _, _ = _run(hgd, dev_bf16(c["W"]), dev_bf16(c["x"]), 257)
    assert guard_ok
    err = np.abs(host(y) - orc.gemv(c["W"], c["x"]))
    assert np.all(err <= 2 * fp32_dot_bound(c["W"], c["x"]) + 1e-30)
