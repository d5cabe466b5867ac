"""Pins for the CPU oracle: each check ties it to something other than itself.

Closed forms, invariants, exact rational arithmetic on tiny inputs, and special
cases that reduce to a library routine (torch's bf16 cast, numpy.correlate,
scipy's softmax).  Every check here is chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a stale
state) fails at least one of them.  No GPU is used.
"""
from fractions import Fraction as Fr
import math

import numpy as np
import pytest

import hgd_synth as syn

EPS_D = 2.0 ** -53
EPS_F = 2.0 ** -24


def bfv(h):
    return syn.from_bf16(h).astype(np.float64)


def bf16_ulp(v):
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return 2.0 ** (e - 7)


# ---------------------------------------------------------------- bf16 -----

def test_round_bf16_matches_torch_cast(orc):
    torch = pytest.importorskip("torch")
    g = syn.rng(11)
    vals = np.concatenate([
        g.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (g.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 3.4e38, -3.4e38, np.inf, -np.inf,
                  1.00390625, 1.01171875, 1.0078125], np.float32),  # ties and overflow
    ])
    ours = orc.round_bf16(vals.astype(np.float64))
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert orc.round_bf16(np.array([np.nan]))[0] & 0x7FFF > 0x7F80


def test_round_bf16_double_input_is_nearest(orc):
    # doubles just above / below a bf16 midpoint must round by the exact value
    mid = 1.0 + 2.0 ** -8            # midpoint between 1 and 1+2^-7
    out = orc.round_bf16(np.array([mid, mid + 2.0 ** -40, mid - 2.0 ** -40]))
    assert list(out) == [0x3F80, 0x3F81, 0x3F80]


# ---------------------------------------------------------------- GEMV -----

def test_gemv_permutation_is_exact(orc):
    g = syn.rng(12)
    K, N, M = 96, 64, 3
    perm = g.permutation(K)[:N]
    W = np.zeros((N, K), np.uint16)
    W[np.arange(N), perm] = 0x3F80  # 1.0
    x = syn.normal_bf16(g, (M, K), 1.0)
    y = orc.gemv(W, x)
    assert np.array_equal(y, bfv(x)[:, perm])


def test_gemv_exact_rational_bound(orc, orc32):
    g = syn.rng(13)
    M, N, K = 2, 5, 37
    W = syn.normal_bf16(g, (N, K), 1.0)
    x = syn.normal_bf16(g, (M, K), 1.0)
    Wf, xf = bfv(W), bfv(x)
    for o, eps in ((orc, EPS_D), (orc32, EPS_F)):
        y = o.gemv(W, x).astype(np.float64)
        gam = K * eps / (1 - K * eps)
        for m in range(M):
            for n in range(N):
                exact = sum(Fr(float(Wf[n, k])) * Fr(float(xf[m, k])) for k in range(K))
                bound = gam * float(np.sum(np.abs(Wf[n]) * np.abs(xf[m])))
                assert abs(Fr(float(y[m, n])) - exact) <= Fr(bound) + Fr(1, 10 ** 30)


def test_swiglu_is_nearest_bf16_of_definition(orc):
    g = syn.rng(14)
    M, I, K = 2, 9, 40
    Wg = syn.normal_bf16(g, (I, K), 0.3)
    Wu = syn.normal_bf16(g, (I, K), 0.3)
    x = syn.normal_bf16(g, (M, K), 1.0)
    h = bfv(orc.swiglu(Wg, Wu, x))
    for m in range(M):
        for i in range(I):
            gv = float(sum(Fr(float(a)) * Fr(float(b)) for a, b in zip(bfv(Wg)[i], bfv(x)[m])))
            uv = float(sum(Fr(float(a)) * Fr(float(b)) for a, b in zip(bfv(Wu)[i], bfv(x)[m])))
            v = gv / (1.0 + math.exp(-gv)) * uv
            assert abs(h[m, i] - v) <= 0.5 * bf16_ulp(v) * (1 + 1e-9) + 1e-300
    # silu(0) = 0: a zero gate matrix gives exactly zero
    assert not np.any(orc.swiglu(np.zeros_like(Wg), Wu, x) & 0x7FFF)


# ---------------------------------------------------------------- conv -----

def test_conv_impulse_response(orc):
    C, kc, T = 6, 4, 6
    g = syn.rng(15)
    w = syn.normal_bf16(g, (C, kc), 1.0)
    tail = np.zeros((1, kc - 1, C))
    x = np.zeros((1, T, C))
    x[0, 0, :] = 1.0
    y = orc.conv1d_tail_update(x, tail, w, apply_silu=True)
    wf = bfv(w)
    silu = lambda t: t / (1 + np.exp(-t))
    for t in range(kc):
        assert np.allclose(y[0, t], silu(wf[:, kc - 1 - t]), rtol=1e-15, atol=0)
    assert np.all(y[0, kc:] == 0)
    # no silu: plain taps, exactly
    tail = np.zeros((1, kc - 1, C))
    y = orc.conv1d_tail_update(x, tail, w, apply_silu=False)
    for t in range(kc):
        assert np.array_equal(y[0, t], wf[:, kc - 1 - t])


def test_conv_is_correlation_over_history(orc):
    B, T, C, kc = 2, 7, 5, 4
    g = syn.rng(16)
    w = syn.normal_bf16(g, (C, kc), 1.0)
    tail0 = g.standard_normal((B, kc - 1, C))
    x = g.standard_normal((B, T, C))
    tail = tail0.copy()
    y, rec = orc.conv1d_tail_update(x, tail, w, apply_silu=False, record=True)
    wf = bfv(w)
    for b in range(B):
        for c in range(C):
            hist = np.concatenate([tail0[b, :, c], x[b, :, c]])
            ref = np.correlate(hist, wf[c], mode="valid")
            assert np.allclose(y[b, :, c], ref, rtol=1e-13, atol=1e-13)
            for t in range(T):  # the recorded tail is the last kc-1 inputs
                assert np.array_equal(rec[b, t, :, c], hist[t + 1:t + kc])
        assert np.array_equal(tail[b], rec[b, -1])


def test_conv_window_equals_steps(orc):
    B, T, C, kc = 2, 8, 7, 4
    g = syn.rng(17)
    w = syn.normal_bf16(g, (C, kc), 1.0)
    tail0 = g.standard_normal((B, kc - 1, C))
    x = g.standard_normal((B, T, C))
    t1 = tail0.copy()
    yw = orc.conv1d_tail_update(x, t1, w)
    t2 = tail0.copy()
    ys = np.concatenate([orc.conv1d_tail_update(np.ascontiguousarray(x[:, t:t + 1]), t2, w)
                         for t in range(T)], axis=1)
    assert np.array_equal(yw, ys) and np.array_equal(t1, t2)


# ---------------------------------------------------------- gated delta -----

def _gdn_inputs(g, B, T, H, dk, dv):
    return dict(q=g.standard_normal((B, T, H, dk)), k=g.standard_normal((B, T, H, dk)),
                v=g.standard_normal((B, T, H, dv)),
                g=-np.log1p(np.exp(g.standard_normal((B, T, H)))),
                b=g.standard_normal((B, T, H)))


def test_gdn_beta0_identity_state(orc):
    """P1: S = I and beta = 0 leave S = alpha I and o = alpha q, exactly."""
    d, H, T = 16, 3, 4
    g = syn.rng(21)
    S = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    inp = _gdn_inputs(g, 1, T, H, d, d)
    inp["b"][:] = -1000.0  # sigmoid(-1000) == 0 in double
    o = orc.gdn_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], S, l2norm=False)
    alpha = np.exp(inp["g"])                      # [1,T,H]
    cum = np.cumprod(alpha, axis=1)
    assert np.array_equal(S, np.eye(d)[None, None] * cum[0, -1][None, :, None, None])
    assert np.allclose(o, cum[..., None] * inp["q"], rtol=1e-15, atol=0)
    # with L2 normalisation the output is alpha q / sqrt(|q|^2 + 1e-6)
    S = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    o = orc.gdn_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], S, l2norm=True)
    qn = inp["q"] / np.sqrt(np.sum(inp["q"] ** 2, -1, keepdims=True) + 1e-6)
    assert np.allclose(o, cum[..., None] * qn, rtol=1e-13, atol=0)


@pytest.mark.parametrize("fp32", [False, True])
def test_gdn_delta_rule_write_and_retrieve(orc, orc32, fp32):
    """P2: with |k| = 1, S_t k = alpha(1-beta) S_{t-1} k + beta v; beta = 1
    retrieves v; directions orthogonal to k only decay by alpha."""
    o_ = orc32 if fp32 else orc
    tol = 2e-6 if fp32 else 1e-12
    d, H = 32, 2
    g = syn.rng(22)
    S0 = g.standard_normal((1, H, d, d)) * 0.3
    inp = _gdn_inputs(g, 1, 1, H, d, d)
    k = inp["k"] / np.linalg.norm(inp["k"], axis=-1, keepdims=True)
    u = g.standard_normal((H, d))
    u -= np.sum(u * k[0, 0], -1, keepdims=True) * k[0, 0]      # u orthogonal to k
    for braw in (1000.0, 0.7):
        bb = np.full((1, 1, H), braw)
        S = o_._r(S0).copy()
        o_.gdn_step(inp["q"], k, inp["v"], inp["g"], bb, S, l2norm=False)
        S = S.astype(np.float64)
        alpha = np.exp(inp["g"][0, 0])
        beta = 1.0 / (1.0 + np.exp(-braw))
        for h in range(H):
            lhs = S[0, h] @ k[0, 0, h]
            rhs = alpha[h] * (1 - beta) * (S0[0, h] @ k[0, 0, h]) + beta * inp["v"][0, 0, h]
            assert np.allclose(lhs, rhs, rtol=0, atol=tol * (1 + np.abs(rhs).max()))
            if braw == 1000.0:
                assert np.allclose(lhs, inp["v"][0, 0, h], rtol=0, atol=tol * 4)
            assert np.allclose(S[0, h] @ u[h], alpha[h] * (S0[0, h] @ u[h]), rtol=0,
                               atol=tol * (1 + np.abs(S0[0, h] @ u[h]).max()))


def test_gdn_frobenius_stability_bound(orc):
    """P3: |S_t|_F <= alpha |S_{t-1}|_F + beta |v| for every step (beta in [0,1])."""
    d, H, T = 24, 2, 64
    g = syn.rng(23)
    S = g.standard_normal((1, H, d, d)) * 0.1
    inp = _gdn_inputs(g, 1, T, H, d, d)
    _, rec = orc.gdn_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], S.copy(),
                          record=True)
    prev = S[0]
    for t in range(T):
        a = np.exp(inp["g"][0, t])
        be = 1 / (1 + np.exp(-inp["b"][0, t]))
        for h in range(H):
            lhs = np.linalg.norm(rec[0, t, h])
            rhs = a[h] * np.linalg.norm(prev[h]) + be[h] * np.linalg.norm(inp["v"][0, t, h])
            assert lhs <= rhs * (1 + 1e-12)
        prev = rec[0, t]


def test_gdn_exact_rational_tiny(orc):
    """P4: alpha = 1 (g = 0) and beta = 1/2 (b = 0) make every step rational; compare
    with exact Fraction arithmetic of the dense definition on the given doubles."""
    d, T = 3, 3
    g = syn.rng(24)
    S0 = g.standard_normal((d, d))
    ks = [g.standard_normal(d) for _ in range(T)]
    vs = [g.standard_normal(d) for _ in range(T)]
    qs = [g.standard_normal(d) for _ in range(T)]
    S = S0[None, None].copy()
    o = orc.gdn_step(np.array(qs)[None, :, None], np.array(ks)[None, :, None],
                     np.array(vs)[None, :, None], np.zeros((1, T, 1)), np.zeros((1, T, 1)), S,
                     l2norm=False)
    Sx = [[Fr(float(S0[i, j])) for j in range(d)] for i in range(d)]
    half = Fr(1, 2)
    for t in range(T):
        k = [Fr(float(a)) for a in ks[t]]
        v = [Fr(float(a)) for a in vs[t]]
        q = [Fr(float(a)) for a in qs[t]]
        A = [[(1 if i == j else 0) - half * k[i] * k[j] for j in range(d)] for i in range(d)]
        Sx = [[sum(Sx[i][l] * A[l][j] for l in range(d)) + half * v[i] * k[j]
               for j in range(d)] for i in range(d)]
        ox = [sum(Sx[i][j] * q[j] for j in range(d)) for i in range(d)]
        for i in range(d):
            assert abs(float(ox[i]) - o[0, t, 0, i]) <= 1e-13 * (1 + abs(float(ox[i])))
    for i in range(d):
        for j in range(d):
            assert abs(float(Sx[i][j]) - S[0, 0, i, j]) <= 1e-13 * (1 + abs(float(Sx[i][j])))


def test_gdn_matches_rank1_and_unrolled_forms(orc):
    """P4: the oracle's dense form equals two algebraically different forms:
    the rank-1 update S + beta (v - alpha S k) k^T (after scaling S by alpha), and the
    unrolled product S_T = S_0 prod(alpha A) + sum_t beta v k^T prod_{s>t}(alpha A)."""
    for d, T in ((4, 4), (8, 3), (5, 2)):
        g = syn.rng(25 + d)
        H = 2
        S0 = g.standard_normal((1, H, d, d))
        inp = _gdn_inputs(g, 1, T, H, d, d)
        S = S0.copy()
        o = orc.gdn_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], S)
        for h in range(H):
            R = S0[0, h].copy()
            terms = []
            P = np.eye(d)
            for t in range(T):
                q = inp["q"][0, t, h] / np.sqrt(np.sum(inp["q"][0, t, h] ** 2) + 1e-6)
                k = inp["k"][0, t, h] / np.sqrt(np.sum(inp["k"][0, t, h] ** 2) + 1e-6)
                a = np.exp(inp["g"][0, t, h])
                be = 1 / (1 + np.exp(-inp["b"][0, t, h]))
                R = a * R + be * np.outer(inp["v"][0, t, h] - a * (R @ k), k)
                assert np.allclose(R @ q, o[0, t, h], rtol=1e-12, atol=1e-12)
                M = a * (np.eye(d) - be * np.outer(k, k))
                terms = [X @ M for X in terms] + [be * np.outer(inp["v"][0, t, h], k)]
                P = P @ M
            unrolled = S0[0, h] @ P + sum(terms)
            assert np.allclose(S[0, h], R, rtol=1e-12, atol=1e-12)
            assert np.allclose(S[0, h], unrolled, rtol=1e-12, atol=1e-12)


# ------------------------------------------- recurrence logs and keep -----
# "qwen3_5 cuda ... #849", tree-window commit note: a verify window logs each
# row's decay, write and key, and keep replays the kept rows in one pass.

def test_gdn_log_exact_rational_tiny(orc):
    """alpha = 1 (g = 0), beta = 1/2 (b = 0), no normalisation: every quantity is
    rational.  The logged write delta_t = beta (v_t - alpha S_{t-1} k_t), the logged
    key and decay, and the replay S_t = alpha S_{t-1} + delta_t k_t^T are compared
    with exact Fraction arithmetic of the dense definition (which the replay must
    reproduce exactly in rationals); S itself stays untouched by the window."""
    d, T = 3, 3
    g = syn.rng(61)
    S0 = g.standard_normal((d, d))
    ks, vs, qs = (g.standard_normal((T, d)) for _ in range(3))
    S = S0[None, None].copy()
    o, la, ld, lk = orc.gdn_window_log(qs[None, :, None], ks[None, :, None], vs[None, :, None],
                                       np.zeros((1, T, 1)), np.zeros((1, T, 1)), S, l2norm=False)
    assert np.array_equal(S[0, 0], S0)
    Sx = [[Fr(float(S0[i, j])) for j in range(d)] for i in range(d)]
    half = Fr(1, 2)
    for t in range(T):
        k = [Fr(float(a)) for a in ks[t]]
        v = [Fr(float(a)) for a in vs[t]]
        q = [Fr(float(a)) for a in qs[t]]
        delta = [half * (v[i] - sum(Sx[i][j] * k[j] for j in range(d))) for i in range(d)]
        A = [[(1 if i == j else 0) - half * k[i] * k[j] for j in range(d)] for i in range(d)]
        dense = [[sum(Sx[i][l] * A[l][j] for l in range(d)) + half * v[i] * k[j] for j in range(d)]
                 for i in range(d)]
        replay = [[Sx[i][j] + delta[i] * k[j] for j in range(d)] for i in range(d)]
        assert dense == replay  # the identity the logs rest on, exactly
        Sx = dense
        assert la[0, t, 0] == 1.0 and np.array_equal(lk[0, t, 0], ks[t])
        for i in range(d):
            assert abs(float(delta[i]) - ld[0, t, 0, i]) <= 1e-13 * (1 + abs(float(delta[i])))
            ox = sum(Sx[i][j] * q[j] for j in range(d))
            assert abs(float(ox) - o[0, t, 0, i]) <= 1e-13 * (1 + abs(float(ox)))
    Sk = S0[None, None].copy()
    orc.gdn_keep(Sk, la, ld, lk, np.array([T], np.int32))
    for i in range(d):
        for j in range(d):
            assert abs(float(Sx[i][j]) - Sk[0, 0, i, j]) <= 1e-13 * (1 + abs(float(Sx[i][j])))


def test_gdn_keep_equals_steps(orc):
    """With gates and normalisation: o of the logged window equals the stepped o bit
    for bit (same dense rows on a copy); keep(n) per stream equals n steps to
    rounding (the replay is the rank-1 form, the steps the dense form); keep(0)
    leaves S untouched; a keep count outside [0, T] is refused."""
    B, T, H, d = 3, 6, 2, 8
    g = syn.rng(62)
    S0 = g.standard_normal((B, H, d, d))
    inp = _gdn_inputs(g, B, T, H, d, d)
    S = S0.copy()
    o, la, ld, lk = orc.gdn_window_log(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], S)
    assert np.array_equal(S, S0)
    assert np.allclose(np.sum(lk ** 2, axis=-1), 1.0, rtol=1e-6)
    assert np.allclose(la, np.exp(inp["g"]), rtol=1e-15, atol=0)
    So = S0.copy()
    ostep = orc.gdn_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], So)
    assert np.array_equal(o, ostep)
    keep = np.array([0, 4, T], np.int32)
    Sk = S0.copy()
    orc.gdn_keep(Sk, la, ld, lk, keep)
    assert np.array_equal(Sk[0], S0[0])
    for b in (1, 2):
        n = int(keep[b])
        Sn = S0[b:b + 1].copy()
        orc.gdn_step(inp["q"][b:b + 1, :n], inp["k"][b:b + 1, :n], inp["v"][b:b + 1, :n],
                     inp["g"][b:b + 1, :n], inp["b"][b:b + 1, :n], Sn)
        assert np.allclose(Sk[b], Sn[0], rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        orc.gdn_keep(S0.copy(), la, ld, lk, np.array([0, 1, T + 1], np.int32))


def test_conv_keep_equals_recorded_tails(orc):
    """The tail after keep(n) rows equals the tail the stepped conv records after
    row n-1 (and the untouched tail for n = 0), bit for bit."""
    B, T, C_, kc = 3, 5, 12, 4
    g = syn.rng(63)
    x = g.standard_normal((B, T, C_))
    w = syn.normal_bf16(g, (C_, kc), 0.5)
    tail0 = g.standard_normal((B, kc - 1, C_))
    t1 = tail0.copy()
    _, rec = orc.conv1d_tail_update(x, t1, w, record=True)
    keep = np.array([0, 2, T], np.int32)
    tk = tail0.copy()
    orc.conv1d_keep(tk, x, keep)
    assert np.array_equal(tk[0], tail0[0])
    assert np.array_equal(tk[1], rec[1, 1])
    assert np.array_equal(tk[2], rec[2, T - 1])
    with pytest.raises(ValueError):
        orc.conv1d_keep(tail0.copy(), x, np.array([-1, 0, 0], np.int32))


def test_gdn_window_equals_steps(orc):
    """P5: a T-row call equals T one-row calls bit for bit (state carried row to row)."""
    B, T, H, d = 2, 8, 3, 16
    g = syn.rng(26)
    S0 = g.standard_normal((B, H, d, d)) * 0.1
    inp = _gdn_inputs(g, B, T, H, d, d)
    S1 = S0.copy()
    ow, rw = orc.gdn_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], S1, record=True)
    S2 = S0.copy()
    for t in range(T):
        sl = {k: np.ascontiguousarray(v[:, t:t + 1]) for k, v in inp.items()}
        o, r = orc.gdn_step(sl["q"], sl["k"], sl["v"], sl["g"], sl["b"], S2, record=True)
        assert np.array_equal(o[:, 0], ow[:, t]) and np.array_equal(r[:, 0], rw[:, t])
    assert np.array_equal(S1, S2)


def test_gdn_packed_rows_match_separate(orc):
    B, T, H, d = 1, 3, 2, 8
    g = syn.rng(27)
    S0 = g.standard_normal((B, H, d, d))
    inp = _gdn_inputs(g, B, T, H, d, d)
    qkv = np.concatenate([inp["q"].reshape(B, T, -1), inp["k"].reshape(B, T, -1),
                          inp["v"].reshape(B, T, -1)], -1)
    S1, S2 = S0.copy(), S0.copy()
    o1 = orc.gdn_step(inp["q"], inp["k"], inp["v"], inp["g"], inp["b"], S1)
    o2 = orc.gdn_step_packed(qkv, inp["g"], inp["b"], S2)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


# --------------------------------------------------------------- norms -----

# --------------------------------------------------------- GDN gates -----
# The gated delta rule decays the state by alpha_t = exp(g_t).  The stack's
# log-decay is g = -exp(A_log) * softplus(a + dt_bias) (A_log per head, stored as
# bf16: "qwen3_5 cuda: mixed-width MLX checkpoints ... #849", the commit on widths
# read from config.json) with the stable softplus max(x,0) + log1p(exp(-|x|))
# ("nvfp4-megamoe-kernel commit log", activation_topk).
# The references below are evaluated with mpmath at 50 digits from the closed
# form log(1 + e^x), not from the oracle's formula.

def _mp_softplus(x):
    import mpmath
    mpmath.mp.dps = 50
    return mpmath.log1p(mpmath.exp(mpmath.mpf(x)))


def _mp_gate(a, A_log, dt):
    import mpmath
    mpmath.mp.dps = 50
    return -mpmath.exp(mpmath.mpf(A_log)) * _mp_softplus(mpmath.mpf(a) + mpmath.mpf(dt))


def test_softplus_closed_forms(orc):
    pytest.importorskip("mpmath")
    assert abs(orc.softplus(0.0) - math.log(2.0)) <= 2 * EPS_D * math.log(2.0)
    # softplus(x) - softplus(-x) = x, and the limits at both ends: the unstable
    # log(1 + exp(x)) gives 0 at -40 (1 + e^-40 rounds to 1) and inf past 709,
    # the stable form e^x and x to full relative precision
    for x in (-700.0, -40.0, -7.25, -1.0, -1e-3, 1e-3, 0.5, 3.0, 40.0, 700.0):
        ref = float(_mp_softplus(x))
        got = orc.softplus(x)
        assert got > 0 and abs(got - ref) <= 4 * EPS_D * ref, (x, got, ref)
        assert abs((orc.softplus(x) - orc.softplus(-x)) - x) <= 8 * EPS_D * max(1.0, abs(x))
    assert orc.softplus(800.0) == 800.0


def test_gdn_gates_match_closed_form(orc):
    """g = -exp(A_log) softplus(a + dt_bias) per head, against the closed form in
    50-digit arithmetic: a dropped exp on A_log, a wrong sign or a missing
    dt_bias each miss by far more than the tolerance."""
    pytest.importorskip("mpmath")
    g = syn.rng(41)
    H = 64
    a = g.standard_normal(H) * 3.0
    A_log = syn.to_bf16((g.standard_normal(H) * 0.7).astype(np.float32))
    dt = syn.to_bf16((g.standard_normal(H) * 1.5).astype(np.float32))
    got = orc.gdn_gates(a, A_log, dt)
    ref = np.array([float(_mp_gate(a[h], bfv(A_log[h]), bfv(dt[h]))) for h in range(H)])
    assert np.all(got < 0)
    assert np.all(np.abs(got - ref) <= 8 * EPS_D * np.abs(ref))
    # special cases: A_log = 0, dt_bias = 0 give g = -softplus(a); A_log = bf16(ln 2)
    # scales |g| by exp(bf16(ln 2)) (= 1.9965, the bf16 value of ln 2 being 0.69140625)
    z = np.zeros(H, np.uint16)
    g0 = orc.gdn_gates(a, z, z)
    assert np.all(np.abs(g0 + np.array([float(_mp_softplus(v)) for v in a])) <= 4 * EPS_D * np.abs(g0))
    ln2 = np.full(H, syn.to_bf16(np.array([math.log(2.0)], np.float32))[0], np.uint16)
    assert bfv(ln2[0]) == 0.69140625
    g2 = orc.gdn_gates(a, ln2, z)
    assert np.all(np.abs(g2 / g0 - math.exp(0.69140625)) <= 8 * EPS_D)
    # dt_bias enters as a shift of a
    gd = orc.gdn_gates(a, z, dt)
    assert np.allclose(gd, orc.gdn_gates(a + bfv(dt), z, z), rtol=8 * EPS_D, atol=0)


def test_stack_gdn_decay_follows_the_gates(orc):
    """One GDN layer of the stack with its key rows zeroed and zero conv tails: the
    key is 0, so the layer's update reduces to S <- alpha S with
    alpha = exp(-exp(A_log[h]) softplus(a_h + dt_bias[h])).  The a-row of head h is
    the unit vector e_{j_h}, so a_h is the normalised input's element j_h (from the
    oracle's RMSNorm, pinned above).  The recorded state after the row is compared
    with alpha * S0 per head, alpha from the closed form in 50-digit arithmetic:
    this ties the stack to the gate formula, to its a/b row order and to the
    per-head A_log and dt_bias."""
    pytest.importorskip("mpmath")
    cfg = dict(syn.SMALL_CFG, n_layers=1, attn_every=8)
    w = syn.stack_weights(cfg, seed=42)
    H, dk, dv, D = cfg["gdn_heads"], cfg["gdn_dk"], cfg["gdn_dv"], cfg["hidden"]
    Cc = 2 * H * dk + H * dv
    lw = w["layers"][0]
    w_in = lw["w_in"].copy()
    w_in[H * dk:2 * H * dk] = 0                        # key rows: k = conv(0) = silu(0) = 0
    cols = [3, 200]
    for h in range(H):
        w_in[Cc + H * dv + h] = 0
        w_in[Cc + H * dv + h, cols[h]] = 0x3F80          # a_h = 1.0 * hnorm[cols[h]]
    lw["w_in"] = w_in
    lw["A_log"] = syn.to_bf16(np.array([0.6, -0.9], np.float32))
    lw["dt_bias"] = syn.to_bf16(np.array([-1.25, 2.0], np.float32))
    m = orc.make_model(cfg, w)
    st = syn.stack_state(cfg, 1, 8, prefill=0, seed=43)
    st["S"] = st["S"].astype(orc.real)
    st["tail"] = np.zeros_like(st["tail"], dtype=orc.real)
    S0 = st["S"].copy()
    tok = np.array([[17]], np.int32)
    r = orc.decode_stack(m, st, tok, record=True)
    hn = bfv(orc.rmsnorm(w["embed"][17][None], lw["in_norm"]))[0]
    for h in range(H):
        alpha = float(__import__("mpmath").exp(_mp_gate(hn[cols[h]], bfv(lw["A_log"][h]),
                                                           bfv(lw["dt_bias"][h]))))
        ratio = r["S_rec"][0, 0, 0, h] / S0[0, 0, h]
        assert 0 < alpha < 1
        assert np.all(np.abs(ratio - alpha) <= 4 * EPS_D * alpha), (h, ratio.min(), ratio.max(), alpha)


def test_rmsnorm_unit_gain_gives_unit_rms(orc):
    g = syn.rng(31)
    x = syn.normal_bf16(g, (5, 512), 3.0)
    y = bfv(orc.rmsnorm(x, np.full(512, 0x3F80, np.uint16)))
    rms = np.sqrt(np.mean(y ** 2, -1))
    assert np.all(np.abs(rms - 1) < 2.0 ** -8)
    # y is the bf16 nearest to x / rms(x) elementwise (eps negligible here)
    xf = bfv(x)
    ref = xf / np.sqrt(np.mean(xf ** 2, -1, keepdims=True) + 1e-6)
    assert np.all(np.abs(y - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-6))
    # gains multiply elementwise: a gain of 2 doubles every output exactly
    y2 = bfv(orc.rmsnorm(x, np.full(512, 0x4000, np.uint16)))
    assert np.array_equal(y2, 2 * y)


def test_gated_rmsnorm_closed_forms(orc):
    g = syn.rng(32)
    M, nh, d = 3, 4, 32
    o = g.standard_normal((M, nh * d)) * 5
    w1 = np.full(d, 0x3F80, np.uint16)
    z0 = np.zeros((M, nh * d), np.uint16)
    assert not np.any(orc.gated_rmsnorm(o, z0, w1, nh) & 0x7FFF)  # silu(0) = 0
    z = syn.normal_bf16(g, (M, nh * d), 2.0)
    u = bfv(orc.gated_rmsnorm(o, z, w1, nh))
    zf = bfv(z)
    sil = zf / (1 + np.exp(-zf))
    ratio = (u / sil).reshape(M, nh, d)  # per-head normalised o
    on = o.reshape(M, nh, d)
    ref = on / np.sqrt(np.mean(on ** 2, -1, keepdims=True) + 1e-6)
    assert np.allclose(ratio, ref, rtol=2.0 ** -8, atol=1e-6)
    # heads are normalised separately: scaling one head of o leaves u unchanged
    o2 = o.copy()
    o2[:, :d] *= 8.0
    assert np.array_equal(orc.gated_rmsnorm(o2, z, w1, nh)[:, d:], orc.gated_rmsnorm(o, z, w1, nh)[:, d:])


# ----------------------------------------------------------- attention -----

def test_rope_closed_forms(orc):
    g = syn.rng(41)
    hd = 64
    x = g.standard_normal(hd)
    assert np.array_equal(orc.rope(x, 0), x)
    for pos in (1, 7, 513):
        r = orc.rope(x, pos)
        half = hd // 2
        # pair 0 turns by pos radians, pair hd/4 by pos * base^-1/2
        assert np.isclose(r[0], x[0] * math.cos(pos) - x[half] * math.sin(pos), rtol=1e-14, atol=1e-14)
        th = pos * 10000.0 ** -0.5
        i = hd // 4
        assert np.isclose(r[i + half], x[i + half] * math.cos(th) + x[i] * math.sin(th), rtol=1e-14, atol=1e-14)
        # every pair keeps its length
        assert np.allclose(r[:half] ** 2 + r[half:] ** 2, x[:half] ** 2 + x[half:] ** 2, rtol=1e-13)
    # relative position: <R(p) q, R(p') k> depends on p - p' only
    q, k = g.standard_normal(hd), g.standard_normal(hd)
    a = orc.rope(q, 600) @ orc.rope(k, 590)
    b = orc.rope(q, 10) @ orc.rope(k, 0)
    assert np.isclose(a, b, rtol=1e-11)


def _attn_case(g, nq, nkv, hd, L):
    q = g.standard_normal((nq, hd))
    gate = g.standard_normal((nq, hd))
    K = syn.normal_bf16(g, (nkv, L, hd), 1.0)
    V = syn.normal_bf16(g, (nkv, L, hd), 1.0)
    return q, gate, K, V


def test_attention_one_key_and_identical_keys(orc):
    g = syn.rng(42)
    nq, nkv, hd, L = 4, 2, 32, 16
    q, gate, K, V = _attn_case(g, nq, nkv, hd, L)
    sig = 1 / (1 + np.exp(-gate))
    out = bfv(orc.attention_row(q, gate, K, V, 1))
    for i in range(nq):
        ref = bfv(V)[i // 2, 0] * sig[i]
        assert np.all(np.abs(out[i] - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-9) + 1e-300)
    # identical keys: the output is the mean of the values
    K2 = np.broadcast_to(K[:, :1], K.shape).copy()
    out = bfv(orc.attention_row(q, gate, K2, V, 11))
    for i in range(nq):
        ref = bfv(V)[i // 2, :11].mean(0) * sig[i]
        assert np.all(np.abs(out[i] - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-9) + 1e-300)


def test_attention_gqa_head_map(orc):
    g = syn.rng(43)
    nq, nkv, hd, L = 8, 2, 16, 8
    q, gate, K, _ = _attn_case(g, nq, nkv, hd, L)
    V = np.zeros((nkv, L, hd), np.uint16)
    V[0] = 0x3F80  # 1.0
    V[1] = 0x4040  # 3.0
    gate = np.full((nq, hd), 50.0)  # sigmoid(50) rounds to 1 in bf16
    out = bfv(orc.attention_row(q, gate, K, V, L))
    assert np.all(out[:4] == 1.0) and np.all(out[4:] == 3.0)


def test_attention_matches_library_softmax(orc):
    sp = pytest.importorskip("scipy.special")
    g = syn.rng(44)
    nq, nkv, hd, L = 4, 2, 64, 300
    q, gate, K, V = _attn_case(g, nq, nkv, hd, L)
    n = 257
    out = bfv(orc.attention_row(q, gate, K, V, n))
    Kf, Vf = bfv(K), bfv(V)
    for i in range(nq):
        p = sp.softmax(Kf[i // 2, :n] @ q[i] / math.sqrt(hd))
        ref = (p @ Vf[i // 2, :n]) / (1 + np.exp(-gate[i]))
        assert np.all(np.abs(out[i] - ref) <= 0.5 * bf16_ulp(ref) * (1 + 1e-6) + 1e-30)


# --------------------------------------------------------------- stack -----

@pytest.fixture(scope="module")
def small():
    cfg = dict(syn.SMALL_CFG)
    return cfg, syn.stack_weights(cfg, seed=5)


def _state(orc, cfg, B, Lmax=40, prefill=16):
    st = syn.stack_state(cfg, B, Lmax, prefill=prefill, seed=6)
    st["S"] = st["S"].astype(orc.real)
    st["tail"] = st["tail"].astype(orc.real)
    return st


def _copy(st):
    return {k: v.copy() for k, v in st.items()}


def test_stack_window_equals_steps(orc, small):
    cfg, w = small
    m = orc.make_model(cfg, w)
    B, T = 2, 5
    st0 = _state(orc, cfg, B)
    toks = syn.stack_tokens(cfg, B, T, seed=7)
    a = _copy(st0)
    rw = orc.decode_stack(m, a, toks, record=True)
    b = _copy(st0)
    for t in range(T):
        r = orc.decode_stack(m, b, toks[:, t:t + 1], record=True)
        assert np.array_equal(r["logits"][:, 0], rw["logits"][:, t])
        assert np.array_equal(r["argmax"][:, 0], rw["argmax"][:, t])
        assert np.array_equal(r["S_rec"][:, :, 0], rw["S_rec"][:, :, t])
        assert np.array_equal(r["tail_rec"][:, :, 0], rw["tail_rec"][:, :, t])
    for k in a:
        assert np.array_equal(a[k], b[k])
    assert np.all(a["pos"] == 16 + T)


def test_stack_resume_equals_continuous(orc, small):
    cfg, w = small
    m = orc.make_model(cfg, w)
    st = _state(orc, cfg, 1)
    toks = syn.stack_tokens(cfg, 1, 6, seed=8)
    full = orc.decode_stack(m, _copy(st), toks)
    s2 = _copy(st)
    orc.decode_stack(m, s2, toks[:, :3])
    saved = _copy(s2)
    r = orc.decode_stack(m, saved, toks[:, 3:])
    assert np.array_equal(r["logits"], full["logits"][:, 3:])


def test_stack_zero_mixers_is_norm_and_tied_head(orc, small):
    """With every output projection zero the residual stream stays the embedding, so
    logits = E . bf16(RMSNorm(E[tok]) * final_norm) exactly as the tied head defines."""
    cfg, w = small
    w0 = {"embed": w["embed"], "final_norm": w["final_norm"],
          "layers": [{k: (np.zeros_like(v) if k in ("w_out", "w_down") else v)
                      for k, v in lw.items()} for lw in w["layers"]]}
    m = orc.make_model(cfg, w0)
    st = _state(orc, cfg, 1)
    toks = syn.stack_tokens(cfg, 1, 2, seed=9)
    r = orc.decode_stack(m, st, toks)
    for t in range(2):
        h = orc.rmsnorm(w["embed"][toks[0, t]][None], w["final_norm"])
        ref = bfv(w["embed"]) @ bfv(h)[0]
        assert np.allclose(r["logits"][0, t], ref, rtol=1e-12, atol=1e-12)
        assert r["argmax"][0, t] == int(np.argmax(ref.astype(np.float32)))


def test_stack_argmax_ties_take_lowest_index(orc, small):
    cfg, w = small
    w2 = dict(w)
    emb = w["embed"].copy()
    emb[:] = emb[3]  # every row identical: all logits tie
    w2["embed"] = emb
    m = orc.make_model(cfg, w2)
    st = _state(orc, cfg, 1)
    r = orc.decode_stack(m, st, np.array([[5, 9]], np.int32))
    assert np.all(r["argmax"] == 0)


def test_stack_rejects_out_of_range(orc, small):
    cfg, w = small
    m = orc.make_model(cfg, w)
    st = _state(orc, cfg, 1, Lmax=20, prefill=19)
    with pytest.raises(ValueError):
        orc.decode_stack(m, st, np.array([[1, 2]], np.int32))


# ------------------------------------ value heads over key heads, untied head
# "qwen3_5 cuda ... #849", commit on the widths read from config.json: linear
# value heads over fewer key heads, an untied head.

def test_gdn_grouped_equals_repeated_key_heads(orc):
    """Value head h reads key head h // (H / Hk): a grouped step equals the
    ungrouped step whose q and k heads are repeated per group, bit for bit, and
    differs from it when the key heads are mapped any other way (interleaved)."""
    B, T, Hk, H, d = 2, 3, 2, 6, 8
    g = syn.rng(64)
    q, k = g.standard_normal((B, T, Hk, d)), g.standard_normal((B, T, Hk, d))
    v = g.standard_normal((B, T, H, d))
    gg, bb = -np.log1p(np.exp(g.standard_normal((B, T, H)))), g.standard_normal((B, T, H))
    S0 = g.standard_normal((B, H, d, d))
    Sg = S0.copy()
    og = orc.gdn_step_grouped(q, k, v, gg, bb, Sg)
    Su = S0.copy()
    ou = orc.gdn_step(np.repeat(q, H // Hk, axis=2), np.repeat(k, H // Hk, axis=2), v, gg, bb, Su)
    assert np.array_equal(og, ou) and np.array_equal(Sg, Su)
    Si = S0.copy()
    oi = orc.gdn_step(np.tile(q, (1, 1, H // Hk, 1)), np.tile(k, (1, 1, H // Hk, 1)), v, gg, bb, Si)
    assert not np.allclose(oi, og)


def _expand_grouped(cfg_g, w_g, st_g):
    """The ungrouped model (Hk = H) equivalent to a grouped one: the q and k rows of
    the in-projection, the q and k channels of the conv weights and conv tails
    repeated once per value head of each group."""
    Hk, H = syn.gdn_heads(cfg_g)
    dk, dv, D = cfg_g["gdn_dk"], cfg_g["gdn_dv"], cfg_g["hidden"]
    G = H // Hk
    rep = lambda a, axis: np.repeat(a.reshape(a.shape[:axis] + (Hk, dk) + a.shape[axis + 1:]), G,
                                    axis=axis).reshape(a.shape[:axis] + (H * dk,) + a.shape[axis + 1:])
    cfg_u = dict(cfg_g, gdn_heads=H, gdn_v_heads=H)
    w_u = {kk: vv for kk, vv in w_g.items() if kk != "layers"}
    w_u["layers"] = []
    for lw in w_g["layers"]:
        lu = dict(lw)
        if "conv_w" in lw:
            wi, cw = lw["w_in"], lw["conv_w"]
            lu["w_in"] = np.concatenate([rep(wi[:Hk * dk], 0), rep(wi[Hk * dk:2 * Hk * dk], 0),
                                         wi[2 * Hk * dk:]], axis=0)
            lu["conv_w"] = np.concatenate([rep(cw[:Hk * dk], 0), rep(cw[Hk * dk:2 * Hk * dk], 0),
                                           cw[2 * Hk * dk:]], axis=0)
        w_u["layers"].append(lu)
    tl = st_g["tail"]
    st_u = dict(st_g, tail=np.ascontiguousarray(np.concatenate(
        [rep(tl[..., :Hk * dk], tl.ndim - 1), rep(tl[..., Hk * dk:2 * Hk * dk], tl.ndim - 1),
         tl[..., 2 * Hk * dk:]], axis=-1)))
    return cfg_u, w_u, st_u


def test_stack_grouped_heads_equal_expanded_model(orc):
    """A stack with 4 GDN value heads over 2 key heads equals, bit for bit (logits,
    argmax, recorded state), the 4-head stack whose q/k projection rows, conv
    weights and conv tails are the grouped ones repeated per value head."""
    cfg = dict(syn.SMALL_CFG, gdn_heads=2, gdn_v_heads=4)
    w = syn.stack_weights(cfg, seed=65)
    st = syn.stack_state(cfg, 2, 40, prefill=16, seed=66)
    cfg_u, w_u, st_u = _expand_grouped(cfg, w, st)
    toks = syn.stack_tokens(cfg, 2, 3, seed=67)
    res = []
    for c, ww, s0 in ((cfg, w, st), (cfg_u, w_u, st_u)):
        s1 = {kk: (vv.astype(orc.real) if vv.dtype == np.float32 else vv).copy() for kk, vv in s0.items()}
        r = orc.decode_stack(orc.make_model(c, ww), s1, toks, record=True)
        res.append((r, s1))
    (rg, sg), (ru, su) = res
    assert np.array_equal(rg["logits"], ru["logits"]) and np.array_equal(rg["argmax"], ru["argmax"])
    assert np.array_equal(rg["S_rec"], ru["S_rec"]) and np.array_equal(sg["S"], su["S"])
    assert rg["S_rec"].shape[3] == 4 and rg["tail_rec"].shape[-1] == 2 * 2 * 64 + 4 * 64


def test_stack_untied_head(orc):
    """The untied head (its own [V, D] matrix): equal to the tied stack when it holds
    the embedding, and with all mixers' and MLPs' output projections zero, the
    logits are lm_head . bf16(RMSNorm(E[tok]) * final_norm) (numpy's product)."""
    cfg = dict(syn.SMALL_CFG, untied_head=1)
    w = syn.stack_weights(cfg, seed=68)
    st = syn.stack_state(cfg, 1, 40, prefill=16, seed=69)
    toks = syn.stack_tokens(cfg, 1, 2, seed=70)
    fresh = lambda: {kk: (vv.astype(orc.real) if vv.dtype == np.float32 else vv).copy() for kk, vv in st.items()}
    w_same = dict(w, lm_head=w["embed"])
    r_same = orc.decode_stack(orc.make_model(cfg, w_same), fresh(), toks)
    w_tied = {kk: vv for kk, vv in w.items() if kk != "lm_head"}
    r_tied = orc.decode_stack(orc.make_model(syn.SMALL_CFG, w_tied), fresh(), toks)
    assert np.array_equal(r_same["logits"], r_tied["logits"])
    w0 = dict(w, layers=[{kk: (np.zeros_like(vv) if kk in ("w_out", "w_down") else vv) for kk, vv in lw.items()}
                         for lw in w["layers"]])
    r0 = orc.decode_stack(orc.make_model(cfg, w0), fresh(), toks)
    for t in range(2):
        h = orc.rmsnorm(w["embed"][toks[0, t]][None], w["final_norm"])
        ref = bfv(w["lm_head"]) @ bfv(h)[0]
        assert np.allclose(r0["logits"][0, t], ref, rtol=1e-12, atol=1e-12)
        assert not np.allclose(ref, bfv(w["embed"]) @ bfv(h)[0], rtol=1e-3, atol=1e-3)


def test_all_cores_build_equals_default_build(orc):
    """The OpenMP build (the all-cores CPU baseline) shares out output elements
    only; every sum keeps its order, so a stack call gives the same bits."""
    from oracle import Oracle
    omp = Oracle(all_cores=True)
    cfg = syn.SMALL_CFG
    w = syn.stack_weights(cfg, seed=5)
    out = []
    for o in (orc, omp):
        st = _state(o, cfg, 2)
        r = o.decode_stack(o.make_model(cfg, w), st, syn.stack_tokens(cfg, 2, 3, seed=7), record=True)
        out.append((r["logits"], r["S_rec"], st["S"], st["kv"]))
    for a, b in zip(*out):
        assert np.array_equal(a, b)


def test_fp32_build_agrees_with_fp64(orc, orc32):
    """The float build (the pages' fp32 reference) stays within the fp32 state
    tolerance of the double build on the tiny GDN case."""
    c = syn.tiny_gdn()
    outs = []
    for o in (orc, orc32):
        qkv = o.gemv(c["W_qkv"], c["x"])[None]
        tail = o._r(c["tail"]).copy()
        y = o.conv1d_tail_update(qkv, tail, c["conv_w"])
        S = o._r(c["S"]).copy()
        oo = o.gdn_step_packed(y, c["g"], c["b"], S)
        outs.append((oo.astype(np.float64), S.astype(np.float64)))
    (o64, S64), (o32, S32) = outs
    assert np.linalg.norm(S32 - S64) / np.linalg.norm(S64) < 1e-5
    assert np.linalg.norm(o32 - o64) / np.linalg.norm(o64) < 1e-5
