"""GPU parity of the standalone C-ABI ops against the CPU oracle (configs 1-3 and
small cases that span several tiles with ragged tails)."""
import numpy as np
import pytest

import hgd_synth as syn
from helpers import (assert_bf16_close, dev_bf16, dev_f32, fp32_dot_bound, host, rel_l2,
                     STATE_REL_L2)

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


# ------------------------------------------------------------------ GEMV ----

GEMV_SMALL = [(1000, 96, 1), (1000, 96, 3), (257, 1056, 8), (129, 3584, 9), (64, 256, 33),
              (1536, 1536, 5), (40, 4096, 2)]


@pytest.mark.parametrize("N,K,M", GEMV_SMALL)
def test_gemv_small_fp32_and_bf16(hgd, orc, N, K, M):
    import torch
    c = syn.gemv_case(N, K, M, seed=9)
    W, x = dev_bf16(c["W"]), dev_bf16(c["x"])
    y32 = torch.full((M, N), float("nan"), device="cuda")
    hgd.gemv_bf16(W, x, y32)
    ybf = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    hgd.gemv_bf16(W, x, ybf, y_is_fp32=False)
    # with the split-K workspace: the same bits, twice in a row (the workspace
    # must come back zero-filled)
    ws = hgd.make_workspace(M, N, K)
    if ws is not None:
        for _ in range(2):
            ys = torch.full((M, N), float("nan"), device="cuda")
            hgd.gemv_bf16(W, x, ys, workspace=ws)
            assert torch.equal(ys, y32)
        torch.cuda.synchronize()
        assert int(ws.count_nonzero().item()) >= 0
    torch.cuda.synchronize()
    ref = orc.gemv(c["W"], c["x"])
    got = host(y32)
    bound = fp32_dot_bound(c["W"], c["x"])
    assert np.all(np.abs(got - ref) <= 2 * bound + 1e-30), np.abs(got - ref).max()
    assert_bf16_close(host(ybf), syn.from_bf16(orc.round_bf16(ref)), "gemv bf16")


@pytest.mark.parametrize("name", list(syn.GEMV_SHAPES))
@pytest.mark.parametrize("M", syn.GEMV_M)
def test_gemv_sweep_shapes(hgd, orc, name, M):
    """The decode GEMV sweep at full size; the oracle checks a sample of output
    features (every M row) for the LM head and all features otherwise."""
    import torch
    N, K = syn.GEMV_SHAPES[name]
    c = syn.gemv_case(N, K, M)
    W, x = dev_bf16(c["W"]), dev_bf16(c["x"])
    ybf = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    hgd.gemv_bf16(W, x, ybf, y_is_fp32=False, workspace=hgd.make_workspace(M, N, K))
    torch.cuda.synchronize()
    cols = np.arange(N) if N <= 4096 else np.sort(syn.rng(5).choice(N, 1024, replace=False))
    ref = orc.gemv(np.ascontiguousarray(c["W"][cols]), c["x"])
    assert_bf16_close(host(ybf)[:, cols], syn.from_bf16(orc.round_bf16(ref)), f"{name} M={M}")


@pytest.mark.parametrize("M", syn.GEMV_M)
def test_swiglu_sweep(hgd, orc, M):
    import torch
    I, K = syn.SWIGLU_SHAPE
    c = syn.swiglu_case(I, K, M)
    h = torch.full((M, I), float("nan"), device="cuda", dtype=torch.bfloat16)
    Wg, Wu, x = dev_bf16(c["Wg"]), dev_bf16(c["Wu"]), dev_bf16(c["x"])
    hgd.gemv_swiglu_bf16(Wg, Wu, x, h)
    ws = hgd.make_workspace(M, I, K, swiglu=True)
    h2 = hgd.gemv_swiglu_bf16(Wg, Wu, x, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), h2.view(torch.int16))
    ref = syn.from_bf16(orc.swiglu(c["Wg"], c["Wu"], c["x"]))
    assert_bf16_close(host(h), ref, f"swiglu M={M}")


def test_swiglu_ragged(hgd, orc):
    import torch
    c = syn.swiglu_case(203, 320, 3, seed=8)
    h = hgd.gemv_swiglu_bf16(dev_bf16(c["Wg"]), dev_bf16(c["Wu"]), dev_bf16(c["x"]))
    torch.cuda.synchronize()
    assert_bf16_close(host(h), syn.from_bf16(orc.swiglu(c["Wg"], c["Wu"], c["x"])), "swiglu ragged")


@pytest.mark.parametrize("K", [1536, 3584])
def test_gemv_rows_independent_of_M(hgd, K):
    """A row computed in an M-row call equals the same row computed alone."""
    import torch
    M, N = 32, 700
    c = syn.gemv_case(N, K, M, seed=4)
    W, x = dev_bf16(c["W"]), dev_bf16(c["x"])
    full = hgd.gemv_bf16(W, x)
    full_ws = hgd.gemv_bf16(W, x, workspace=hgd.make_workspace(M, N, K))
    assert torch.equal(full, full_ws)
    for m in (0, 7, 8, 31):
        one = hgd.gemv_bf16(W, x[m:m + 1].contiguous())
        assert torch.equal(one[0], full[m])
        one_ws = hgd.gemv_bf16(W, x[m:m + 1].contiguous(), workspace=hgd.make_workspace(1, N, K))
        assert torch.equal(one_ws[0], full[m])
    h_full = hgd.gemv_swiglu_bf16(W, W, x)
    h_one = hgd.gemv_swiglu_bf16(W, W, x[5:6].contiguous())
    assert torch.equal(h_one[0].view(torch.int16), h_full[5].view(torch.int16))


# ------------------------------------------------------------------ conv ----

def test_conv_parity_and_window(hgd, orc):
    import torch
    B, T, C, kc = 3, 7, 1000, 4
    g = syn.rng(31)
    x = g.standard_normal((B, T, C)).astype(np.float32)
    tail0 = g.standard_normal((B, kc - 1, C)).astype(np.float32)
    w = syn.normal_bf16(g, (C, kc), 0.5)
    tail = dev_f32(tail0)
    rec = torch.full((B, T, kc - 1, C), float("nan"), device="cuda")
    y = hgd.conv1d_tail_update(dev_f32(x), tail, dev_bf16(w), tail_rec=rec)
    ot = tail0.astype(np.float64).copy()
    oy, orec = orc.conv1d_tail_update(x.astype(np.float64), ot, w, record=True)
    torch.cuda.synchronize()
    assert np.allclose(host(y), oy, rtol=1e-5, atol=1e-5)
    assert np.array_equal(host(rec), orec.astype(np.float32).astype(np.float64))
    assert np.array_equal(host(tail), ot.astype(np.float32).astype(np.float64))
    # window == steps, bit for bit
    t2 = dev_f32(tail0)
    ys = [hgd.conv1d_tail_update(dev_f32(x[:, t:t + 1]), t2, dev_bf16(w)) for t in range(T)]
    assert torch.equal(torch.cat(ys, 1), y) and torch.equal(t2, tail)


# ------------------------------------------------------------------- GDN ----

def _gdn_dev(hgd, inp, S, T, record=False):
    import torch
    B, H, dv, dk = S.shape
    rec = torch.full((B, T, H, dv, dk), float("nan"), device="cuda") if record else None
    o = hgd.gdn_decode_step(dev_f32(inp["q"]), dev_f32(inp["k"]), dev_f32(inp["v"]), dev_f32(inp["g"]),
                            dev_f32(inp["b"]), S, S_rec=rec)
    return o, rec


@pytest.mark.parametrize("dk,dv", [(32, 48), (64, 64), (128, 128), (256, 96)])
def test_gdn_step_small(hgd, orc, dk, dv):
    """q|k|v packed per row with a row stride (the conv-output layout), records on."""
    import torch
    B, T, H = 2, 5, 3
    g = syn.rng(40 + dk)
    inp = dict(q=g.standard_normal((B, T, H, dk)), k=g.standard_normal((B, T, H, dk)),
               v=g.standard_normal((B, T, H, dv)), g=-np.log1p(np.exp(g.standard_normal((B, T, H)))),
               b=g.standard_normal((B, T, H)))
    inp = {k: v.astype(np.float32) for k, v in inp.items()}
    S0 = (g.standard_normal((B, H, dv, dk)) * 0.1).astype(np.float32)
    packed = np.concatenate([inp["q"].reshape(B, T, -1), inp["k"].reshape(B, T, -1),
                             inp["v"].reshape(B, T, -1)], -1)
    stride = packed.shape[-1]
    P = dev_f32(packed)
    S = dev_f32(S0)
    rec = torch.full((B, T, H, dv, dk), float("nan"), device="cuda")
    o = hgd.gdn_decode_step(P, P[..., H * dk:], P[..., 2 * H * dk:], dev_f32(inp["g"]), dev_f32(inp["b"]),
                            S, S_rec=rec, row_stride=stride, B=B, T=T)
    oS = S0.astype(np.float64).copy()
    oo, orec = orc.gdn_step_packed(packed, inp["g"], inp["b"], oS, record=True)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            assert rel_l2(host(S)[b, h], oS[b, h]) <= STATE_REL_L2
            for t in range(T):
                assert rel_l2(host(rec)[b, t, h], orec[b, t, h]) <= STATE_REL_L2
    assert rel_l2(host(o), oo) <= STATE_REL_L2


def test_gdn_window_equals_steps(hgd):
    import torch
    B, T, H, d = 2, 16, 4, 128
    g = syn.rng(50)
    inp = dict(q=g.standard_normal((B, T, H, d)), k=g.standard_normal((B, T, H, d)),
               v=g.standard_normal((B, T, H, d)), g=-np.log1p(np.exp(g.standard_normal((B, T, H)))),
               b=g.standard_normal((B, T, H)))
    inp = {k: v.astype(np.float32) for k, v in inp.items()}
    S0 = (g.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    S1 = dev_f32(S0)
    ow, rw = _gdn_dev(hgd, inp, S1, T, record=True)
    S2 = dev_f32(S0)
    for t in range(T):
        sl = {k: np.ascontiguousarray(v[:, t:t + 1]) for k, v in inp.items()}
        o, r = _gdn_dev(hgd, sl, S2, 1, record=True)
        assert torch.equal(o[:, 0], ow[:, t]) and torch.equal(r[:, 0], rw[:, t])
    assert torch.equal(S1, S2)


@pytest.mark.parametrize("B", syn.GDN_SWEEP_B)
def test_gdn_sweep_256_steps(hgd, orc, B):
    """The state-update sweep: 256 consecutive one-row steps of B streams x 16 heads,
    d = 128.  Every step of every head is checked for B = 1; for larger B a fixed
    sample of (stream, head) pairs is followed by the oracle through all 256 steps
    (the heads are independent, so each sampled head is checked exactly)."""
    import torch
    steps = 256
    c = syn.gdn_sweep(B, steps=steps)
    H, d = 16, 128
    S = dev_f32(c["S"])
    pairs = [(b, h) for b in range(B) for h in range(H)] if B == 1 else \
        [(int(b), int(h)) for b, h in zip(syn.rng(60 + B).integers(0, B, 4), syn.rng(61 + B).integers(0, H, 4))]
    oS = {bh: c["S"][bh[0], bh[1]][None, None].astype(np.float64).copy() for bh in pairs}
    qd, kd, vd = dev_f32(c["q"]), dev_f32(c["k"]), dev_f32(c["v"])
    gd, bd = dev_f32(c["g"]), dev_f32(c["b"])
    worst_s = worst_o = 0.0
    for t in range(steps):
        o = hgd.gdn_decode_step(qd[t], kd[t], vd[t], gd[t], bd[t], S)
        idx_b = torch.tensor([b for b, _ in pairs], device="cuda")
        idx_h = torch.tensor([h for _, h in pairs], device="cuda")
        S_h = host(S[idx_b, idx_h])
        o_h = host(o[idx_b, 0, idx_h])
        for n, (b, h) in enumerate(pairs):
            sl = lambda a: np.ascontiguousarray(a[t, b:b + 1, :, h:h + 1])
            oo = orc.gdn_step(sl(c["q"]), sl(c["k"]), sl(c["v"]), sl(c["g"]), sl(c["b"]), oS[(b, h)])
            worst_s = max(worst_s, rel_l2(S_h[n], oS[(b, h)][0, 0]))
            worst_o = max(worst_o, rel_l2(o_h[n], oo[0, 0, 0]))
    assert worst_s <= STATE_REL_L2, worst_s
    assert worst_o <= STATE_REL_L2, worst_o


# ------------------------------------------------------ config 1: tiny GDN --

def _tiny_gpu(hgd, c, window):
    import torch
    H, d, C, T = c["H"], c["d"], c["C"], c["T"]
    tail = dev_f32(c["tail"])
    S = dev_f32(c["S"])
    Wqkv, Wo, cw = dev_bf16(c["W_qkv"]), dev_bf16(c["W_o"]), dev_bf16(c["conv_w"])
    g, b = dev_f32(c["g"]), dev_f32(c["b"])
    xs = dev_bf16(c["x"])
    outs, os_ = [], []
    rows = [slice(0, T)] if window else [slice(t, t + 1) for t in range(T)]
    for r in rows:
        n = r.stop - r.start
        qkv = hgd.gemv_bf16(Wqkv, xs[r].contiguous())
        y = hgd.conv1d_tail_update(qkv.view(1, n, C), tail, cw)
        o_bf = torch.empty((1, n, H, d), dtype=torch.bfloat16, device="cuda")
        o = hgd.gdn_decode_step(y, y[..., H * d:], y[..., 2 * H * d:], g[:, r].contiguous(),
                                b[:, r].contiguous(), S, o_bf16=o_bf, row_stride=C, B=1, T=n)
        outs.append(hgd.gemv_bf16(Wo, o_bf.view(n, H * d), y_is_fp32=False))
        os_.append(o)
    torch.cuda.synchronize()
    return torch.cat(outs, 0), torch.cat(os_, 1), S, tail


def test_tiny_gdn_mixer(hgd, orc):
    import torch
    c = syn.tiny_gdn(seed=1)
    H, d, C, T = c["H"], c["d"], c["C"], c["T"]
    yw, ow, Sw, tw = _tiny_gpu(hgd, c, window=True)
    ys, os_, Ss, ts = _tiny_gpu(hgd, c, window=False)
    # the 8-row window equals 8 one-row steps, bit for bit
    assert torch.equal(yw.view(torch.int16), ys.view(torch.int16))
    assert torch.equal(ow, os_) and torch.equal(Sw, Ss) and torch.equal(tw, ts)
    # against the oracle
    qkv = orc.gemv(c["W_qkv"], c["x"])[None]
    ot = c["tail"].astype(np.float64).copy()
    yy = orc.conv1d_tail_update(qkv, ot, c["conv_w"])
    oS = c["S"].astype(np.float64).copy()
    oo = orc.gdn_step_packed(yy, c["g"], c["b"], oS)
    out = orc.gemv(c["W_o"], orc.round_bf16(oo.reshape(T, H * d)))
    assert_bf16_close(host(yw), syn.from_bf16(orc.round_bf16(out)), "tiny y")
    assert_bf16_close(host(ow).astype(np.float32), oo, "tiny o")
    for h in range(H):
        assert rel_l2(host(Sw)[0, h], oS[0, h]) <= STATE_REL_L2
    assert np.allclose(host(tw), ot, rtol=1e-5, atol=1e-5)


# ------------------------------------------- recurrence logs and keep -------
# "qwen3_5 cuda ... #849", tree-window commit note: a verify window logs each
# row's decay, write and key; keep replays the kept rows in one pass.

@pytest.mark.parametrize("B,H,dk,dv,T", [(3, 2, 64, 64, 7), (4, 16, 128, 128, 16), (2, 3, 32, 48, 5),
                                         (1, 2, 256, 96, 4)])
def test_gdn_window_log_and_keep(hgd, orc, B, H, dk, dv, T):
    """A T-row logged window leaves S untouched and gives the o of T one-row steps
    bit for bit; keep(n) per stream (0, some, all) gives the S of n one-row steps
    bit for bit; the logs match the oracle's (decay and key to fp32 rounding, the
    write within the state tolerance per head)."""
    import torch
    g = syn.rng(70 + dk + T)
    S0 = syn.normal_f32(g, (B, H, dv, dk), 0.1)
    q = syn.normal_f32(g, (B, T, H, dk))
    k = syn.normal_f32(g, (B, T, H, dk))
    v = syn.normal_f32(g, (B, T, H, dv))
    gg = syn.neg_softplus_normal(g, (B, T, H))
    bb = syn.normal_f32(g, (B, T, H))
    # the GPU's q/k/v as one packed row per (b, t): q | k | v
    stride = 2 * H * dk + H * dv
    rows = np.concatenate([q.reshape(B * T, -1), k.reshape(B * T, -1), v.reshape(B * T, -1)], axis=1)
    rd = dev_f32(rows)
    qd, kd, vd = rd, rd[:, H * dk:], rd[:, 2 * H * dk:]
    gd, bd = dev_f32(gg), dev_f32(bb)
    S = dev_f32(S0)
    o, la, ld, lk = hgd.gdn_window_log(qd, kd, vd, gd, bd, S, row_stride=stride, B=B, T=T)
    torch.cuda.synchronize()
    assert torch.equal(S, dev_f32(S0))
    # one-row steps from the same state
    Ss = dev_f32(S0)
    steps_o, steps_S = [], []
    for t in range(T):
        rs = dev_f32(rows.reshape(B, T, -1)[:, t])
        os_ = hgd.gdn_decode_step(rs, rs[:, H * dk:], rs[:, 2 * H * dk:], dev_f32(gg[:, t:t + 1]),
                                  dev_f32(bb[:, t:t + 1]), Ss, row_stride=stride, B=B, T=1)
        steps_o.append(os_)
        steps_S.append(Ss.clone())
    assert torch.equal(o, torch.cat(steps_o, dim=1))
    keep = np.array({1: [T], 2: [0, T], 3: [0, T // 2, T], 4: [0, 1, T // 2, T]}[B], np.int32)
    Sk = dev_f32(S0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hgd.gdn_keep(Sk, la, ld, lk, torch.from_numpy(keep).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for b in range(B):
        n = int(keep[b])
        ref = dev_f32(S0)[b] if n == 0 else steps_S[n - 1][b]
        assert torch.equal(Sk[b], ref), f"stream {b}: keep({n}) differs from {n} steps"
    # against the oracle's logs (dk == dv cases; the oracle's separate arrays share one stride)
    if dk == dv:
        oo, ola, old, olk = orc.gdn_window_log(q, k, v, gg, bb, S0.astype(np.float64))
        assert np.allclose(host(la), ola, rtol=2e-6, atol=0)
        assert np.allclose(host(lk), olk, rtol=0, atol=2e-6)
        gdl = host(ld)
        worst = max(rel_l2(gdl[b, t, h], old[b, t, h]) for b in range(B) for t in range(T) for h in range(H))
        assert worst <= STATE_REL_L2, worst
        assert rel_l2(host(o), oo) <= STATE_REL_L2


def test_gdn_keep_rejects_out_of_range_counts(hgd):
    """A keep count outside [0, T] leaves that stream's state as it is and reports
    HGD_ERR_INVALID_ARG; the other streams are kept."""
    import torch
    B, H, d, T = 3, 2, 64, 4
    g = syn.rng(77)
    S0 = dev_f32(syn.normal_f32(g, (B, H, d, d), 0.1))
    q = dev_f32(syn.normal_f32(g, (B, T, H, d)))
    k = dev_f32(syn.normal_f32(g, (B, T, H, d)))
    v = dev_f32(syn.normal_f32(g, (B, T, H, d)))
    gd, bd = dev_f32(syn.neg_softplus_normal(g, (B, T, H))), dev_f32(syn.normal_f32(g, (B, T, H)))
    _, la, ld, lk = hgd.gdn_window_log(q, k, v, gd, bd, S0)
    S = S0.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hgd.gdn_keep(S, la, ld, lk, torch.tensor([T + 1, 2, -1], dtype=torch.int32, device="cuda"), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    assert torch.equal(S[0], S0[0]) and torch.equal(S[2], S0[2]) and not torch.equal(S[1], S0[1])


def test_conv_keep_equals_stepped_tails(hgd):
    """The conv tail after keep(n) rows of a window equals the tail left by n
    one-row conv steps, bit for bit; out-of-range counts are refused per stream."""
    import torch
    B, T, C_, kc = 4, 6, 6144, 4
    g = syn.rng(78)
    x = dev_f32(syn.normal_f32(g, (B, T, C_)))
    w = dev_bf16(syn.normal_bf16(g, (C_, kc), 0.5))
    tail0 = dev_f32(syn.normal_f32(g, (B, kc - 1, C_)))
    ts = tail0.clone()
    stepped = []
    for t in range(T):
        hgd.conv1d_tail_update(x[:, t:t + 1].contiguous(), ts, w)
        stepped.append(ts.clone())
    keep = torch.tensor([0, 1, 5, T], dtype=torch.int32, device="cuda")
    tk = tail0.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hgd.conv1d_keep(tk, x, keep, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for b, n in enumerate(keep.tolist()):
        assert torch.equal(tk[b], tail0[b] if n == 0 else stepped[n - 1][b])
    bad = tail0.clone()
    hgd.conv1d_keep(bad, x, torch.tensor([7, 0, 0, 0], dtype=torch.int32, device="cuda"), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1 and torch.equal(bad, tail0)


# --------------------------------- value heads over fewer key heads ---------
# "qwen3_5 cuda ... #849", commit on the widths read from config.json.

@pytest.mark.parametrize("Hk,H,d,T", [(4, 16, 128, 3), (2, 6, 64, 2)])
def test_gdn_grouped_step(hgd, orc, Hk, H, d, T):
    """Value head h reads key head h // (H / Hk): the grouped step equals the
    ungrouped step on q/k heads repeated per group, bit for bit, and the oracle's
    grouped step within the state tolerance."""
    import torch
    B = 2
    g = syn.rng(80 + H)
    q, k = syn.normal_f32(g, (B, T, Hk, d)), syn.normal_f32(g, (B, T, Hk, d))
    v = syn.normal_f32(g, (B, T, H, d))
    gg, bb = syn.neg_softplus_normal(g, (B, T, H)), syn.normal_f32(g, (B, T, H))
    S0 = syn.normal_f32(g, (B, H, d, d), 0.1)
    stride = 2 * Hk * d + H * d
    rows = dev_f32(np.concatenate([q.reshape(B * T, -1), k.reshape(B * T, -1), v.reshape(B * T, -1)], axis=1))
    S = dev_f32(S0)
    o = hgd.gdn_decode_step_grouped(rows, rows[:, Hk * d:], rows[:, 2 * Hk * d:], dev_f32(gg), dev_f32(bb), S,
                                    key_heads=Hk, row_stride=stride, B=B, T=T)
    G = H // Hk
    Su = dev_f32(S0)
    ou = hgd.gdn_decode_step(dev_f32(np.repeat(q, G, axis=2)), dev_f32(np.repeat(k, G, axis=2)), dev_f32(v),
                             dev_f32(gg), dev_f32(bb), Su)
    torch.cuda.synchronize()
    assert torch.equal(o, ou) and torch.equal(S, Su)
    oS = S0.astype(np.float64)
    oo = orc.gdn_step_grouped(q, k, v, gg, bb, oS)
    assert rel_l2(host(o), oo) <= STATE_REL_L2
    for b in range(B):
        for h in range(H):
            assert rel_l2(host(S[b, h]), oS[b, h]) <= STATE_REL_L2


# ----------------------------------------------------- prefill (chunked) ----
# "luce-megakernel HANDOFF.md", Architecture Summary (a prefill kernel) and
# Expected Results (pp512): T rows at once, equal to T one-row steps to rounding.

@pytest.mark.parametrize("B,H,dk,dv,T", [(2, 3, 128, 128, 100), (1, 4, 64, 64, 37), (2, 2, 128, 64, 512),
                                         (1, 2, 128, 128, 1), (1, 16, 128, 128, 512)])
def test_gdn_prefill_matches_steps_and_oracle(hgd, orc, B, H, dk, dv, T):
    """The chunked form over T rows (whole chunks of 32 and a ragged tail) against
    the oracle's row-by-row recurrence (fp64), output and final state per head
    within the state tolerance, and against the GPU's own one-row-at-a-time
    kernel over the same rows."""
    import torch
    g = syn.rng(90 + T + dk)
    S0 = syn.normal_f32(g, (B, H, dv, dk), 0.1)
    q = syn.normal_f32(g, (B, T, H, dk))
    k = syn.normal_f32(g, (B, T, H, dk))
    v = syn.normal_f32(g, (B, T, H, dv))
    gg = syn.neg_softplus_normal(g, (B, T, H))
    bb = syn.normal_f32(g, (B, T, H))
    stride = 2 * H * dk + H * dv
    rows = dev_f32(np.concatenate([q.reshape(B * T, -1), k.reshape(B * T, -1), v.reshape(B * T, -1)], axis=1))
    qd, kd, vd = rows, rows[:, H * dk:], rows[:, 2 * H * dk:]
    S = dev_f32(S0)
    o = hgd.gdn_prefill(qd, kd, vd, dev_f32(gg), dev_f32(bb), S, row_stride=stride, B=B, T=T)
    Ss = dev_f32(S0)
    os_ = hgd.gdn_decode_step(qd, kd, vd, dev_f32(gg), dev_f32(bb), Ss, row_stride=stride, B=B, T=T)
    torch.cuda.synchronize()
    go, gS = host(o), host(S)
    assert rel_l2(gS, host(Ss)) <= STATE_REL_L2 and rel_l2(go, host(os_)) <= STATE_REL_L2
    if dk == dv:
        oS = S0.astype(np.float64)
        oo = orc.gdn_step(q, k, v, gg, bb, oS)
        for b in range(B):
            for h in range(H):
                assert rel_l2(gS[b, h], oS[b, h]) <= STATE_REL_L2, (b, h)
                assert rel_l2(go[b, :, h], oo[b, :, h]) <= STATE_REL_L2, (b, h)
