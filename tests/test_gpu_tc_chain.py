"""The tensor-core decode chain (hgd_decode_layer_stack_tc) against itself and the oracle.

"qwen3_5 cuda: mixed-width MLX checkpoints ... #849", PR body: windows of up to
16 rows of several streams per call, a window's rows equal to one-row steps bit
for bit.  Through the tensor-core chain (every projection a tcgen05 GEMM over
all of a call's rows):
* a window equals its one-row steps bit for bit (logits, argmax, per-row state and
  conv-tail records, final state, cache, positions), in the reduced geometry and
  for the 8-stream x 16-row window at full size;
* the results follow the oracle: within the bf16 tolerance in the reduced
  geometry, and at full size within the oracle's own fp32 deviation end to end
  (GDN layer 0, which sees exact inputs, within the state tolerance).
"""
import functools
import threading

import numpy as np
import pytest

import hgd_synth as syn
from helpers import BF16_REL_L2, host, rel_l2
from stack_common import compare_argmax, compare_logits, compare_state_rel, oracle_state, weights

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


def _call(hgd, model, state, toks, T, V):
    import torch
    cfg = model.cfg_dict
    B = state.B
    n_gdn, _ = syn.layer_counts(cfg)
    Hk, H = syn.gdn_heads(cfg)
    dk, dv, kc = cfg["gdn_dk"], cfg["gdn_dv"], cfg["conv_k"]
    Cc = 2 * Hk * dk + H * dv
    lg = torch.full((B * T, V), float("nan"), device="cuda")
    sr = torch.full((n_gdn, B, T, H, dv, dk), float("nan"), device="cuda")
    tr = torch.full((n_gdn, B, T, kc - 1, Cc), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    am = hgd.decode_layer_stack_tc(model, state, toks, T, logits=lg, S_rec=sr, tail_rec=tr, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, hgd.status_string(int(status.item()))
    return am, lg, sr, tr


def _window_vs_steps(hgd, model, cfg, B, T, Lmax, prefill, seed):
    import torch
    V = cfg["vocab"]
    init = syn.stack_state(cfg, B, Lmax, prefill=prefill, seed=seed)
    toks = syn.stack_tokens(cfg, B, T, seed=seed)
    sw = hgd.State(model, B, T, Lmax, init)
    amw, lw, srw, trw = _call(hgd, model, sw, torch.from_numpy(toks).cuda(), T, V)
    ss = hgd.State(model, B, 1, Lmax, init)
    for t in range(T):
        am, lg, sr, tr = _call(hgd, model, ss, torch.from_numpy(np.ascontiguousarray(toks[:, t:t + 1])).cuda(), 1, V)
        rows = [b * T + t for b in range(B)]
        assert torch.equal(lg, lw[rows]), f"row {t}: logits differ"
        assert torch.equal(am, amw[rows])
        assert torch.equal(sr[:, :, 0], srw[:, :, t]) and torch.equal(tr[:, :, 0], trw[:, :, t]), f"row {t}"
        del lg, sr, tr
    for a, b in ((sw.S, ss.S), (sw.conv, ss.conv), (sw.kv, ss.kv), (sw.pos, ss.pos)):
        assert torch.equal(a, b)
    return init, toks, amw, lw, srw, trw, sw


def test_tc_chain_small_window_equals_steps_and_oracle(hgd, orc):
    cfg, w = syn.SMALL_CFG, weights("small", 5)
    model = hgd.Model(cfg, w, tc=True)
    B, T, Lmax = 2, 5, 40
    init, toks, amw, lw, srw, trw, sw = _window_vs_steps(hgd, model, cfg, B, T, Lmax, 16, 51)
    V = cfg["vocab"]
    m = orc.make_model(cfg, w)
    ost = oracle_state(orc, init)
    r = orc.decode_stack(m, ost, toks, record=True)
    compare_logits(host(lw), r["logits"].reshape(B * T, V), "tensor-core chain, small window")
    compare_argmax(host(amw), r["logits"].reshape(B * T, V), "tensor-core chain, small window")
    compare_state_rel(host(srw)[0], r["S_rec"][0], "tensor-core chain, GDN layer 0 records")
    compare_state_rel(host(trw)[0], r["tail_rec"][0], "tensor-core chain, layer 0 conv tails")
    assert rel_l2(host(sw.S), ost["S"]) <= BF16_REL_L2


@functools.lru_cache(maxsize=1)
def _full_oracle(T, seed):
    from oracle import Oracle
    cfg = syn.STACK_CFG
    w = weights("stack", 4)
    init = syn.stack_state(cfg, 8, 768, prefill=512, seed=seed)
    toks = syn.stack_tokens(cfg, 8, T, seed=seed)
    res = {}

    def run(o):
        st = oracle_state(o, init, streams=slice(0, 1))
        rr = o.decode_stack(o.make_model(cfg, w), st, toks[0:1], logits=True, record=True)
        res[o.real] = (rr["logits"][0].astype(np.float64), rr["S_rec"].astype(np.float64))

    th = [threading.Thread(target=run, args=(o,)) for o in (Oracle(), Oracle(fp32=True))]
    for t in th:
        t.start()
    for t in th:
        t.join()
    return res


def test_tc_chain_config5_window_equals_steps_and_oracle(hgd):
    """8 streams x 16-row window, the full stack: the window equals 16 one-row steps
    of the 8 streams bit for bit; stream 0 follows the oracle."""
    cfg = syn.STACK_CFG
    model = hgd.Model(cfg, weights("stack", 4), tc=True)
    B, T, Lmax = 8, 16, 768
    init, toks, amw, lw, srw, trw, sw = _window_vs_steps(hgd, model, cfg, B, T, Lmax, 512, 52)
    res = _full_oracle(T, 52)
    l64, sr64 = res[np.float64]
    l32, sr32 = res[np.float32]
    g = host(lw[:T])
    for t in range(T):
        assert rel_l2(g[t], l64[t]) <= 1.5 * rel_l2(l32[t], l64[t]) + 1e-3, f"row {t} logits"
    gs = host(srw[:, 0:1])
    compare_state_rel(gs[0], sr64[0], "tensor-core chain, GDN layer 0 records")
    assert rel_l2(gs, sr64) <= 1.5 * rel_l2(sr32, sr64) + BF16_REL_L2


# value heads over fewer key heads and an untied head ("qwen3_5 cuda ... #849",
# the commit on widths read from config.json): the reduced geometry, and hidden
# 1024 with 16 value heads over 8 key heads of 128 (the head-per-CTA GDN kernel
# with the gated norm fused and the conv separate), both through the tensor cores
GROUPED_SMALL = dict(syn.SMALL_CFG, gdn_heads=2, gdn_v_heads=4, untied_head=1)
GROUPED_WIDE = dict(syn.STACK_CFG, n_layers=4, vocab=8192, gdn_heads=8, gdn_v_heads=16, untied_head=1)


@pytest.mark.parametrize("which", ["small", "wide"])
def test_tc_chain_grouped_untied(hgd, orc, orc32, which):
    """A window equals its one-row steps bit for bit; the window's logits follow the
    oracle within its own fp32 deviation (the end-to-end reading: at most 1.5x the
    fp32 oracle's deviation from fp64, over the window; a single row within 3x, since
    a bf16 rounding flip upstream in one evaluation and not the other moves one row
    by about that much), and in the reduced geometry within the bf16 tolerance.  The
    mma.sync chain on the same inputs agrees to the same fp32 noise (a wrong head or
    row mapping would not)."""
    import torch
    cfg = GROUPED_SMALL if which == "small" else GROUPED_WIDE
    w = syn.stack_weights(cfg, seed=92)
    model = hgd.Model(cfg, w, tc=True)
    B, T, Lmax, pre = (2, 5, 40, 16) if which == "small" else (4, 8, 640, 512)
    init, toks, amw, lw, srw, trw, sw = _window_vs_steps(hgd, model, cfg, B, T, Lmax, pre, 93)
    V = cfg["vocab"]
    refs = {}
    for o in (orc, orc32):
        ost = oracle_state(o, init)
        r = o.decode_stack(o.make_model(cfg, w), ost, toks, logits=True)
        refs[o.real] = r["logits"].reshape(B * T, V).astype(np.float64)
    l64, l32 = refs[np.float64], refs[np.float32]
    g = host(lw)
    assert rel_l2(g, l64) <= 1.5 * rel_l2(l32, l64) + 1e-3, which
    for row in range(B * T):
        assert rel_l2(g[row], l64[row]) <= 3 * rel_l2(l32[row], l64[row]) + 2e-3, f"{which}: row {row} logits"
    model_m = hgd.Model(cfg, w)
    sm = hgd.State(model_m, B, T, Lmax, init)
    lg_m = torch.empty((B * T, V), device="cuda")
    hgd.decode_layer_stack(model_m, sm, torch.from_numpy(toks).cuda(), T, logits=lg_m)
    torch.cuda.synchronize()
    assert rel_l2(g, host(lg_m)) <= 2 * rel_l2(l32, l64) + 1e-3, f"{which}: tensor-core vs mma.sync chain"
    if which == "small":
        compare_logits(g, l64, "tensor-core chain, grouped small")


# attention geometries of the tensor-core partials: head dims 128 and 32, eight
# query heads over one kv head with 12-row windows (96 query vectors of a stream
# per chunk: two passes of the 64-vector tiles), and a window that starts 7 keys
# before a chunk boundary (its first rows see only the chunk before it)
ATTN_GEOMS = {
    "hd128_group8": (dict(syn.SMALL_CFG, attn_q_heads=8, attn_kv_heads=1, attn_head_dim=128), 2, 12, 64, 25),
    "hd32": (dict(syn.SMALL_CFG, attn_head_dim=32), 3, 5, 48, 30),
}


@pytest.mark.parametrize("which", list(ATTN_GEOMS))
def test_tc_chain_attention_geometries(hgd, orc, which):
    """A window equals its one-row steps bit for bit and follows the oracle within
    the bf16 tolerance, at attention geometries the stack's own shape does not reach."""
    cfg, B, T, Lmax, pre = ATTN_GEOMS[which]
    w = syn.stack_weights(cfg, seed=94)
    model = hgd.Model(cfg, w, tc=True)
    init, toks, amw, lw, srw, trw, sw = _window_vs_steps(hgd, model, cfg, B, T, Lmax, pre, 95)
    V = cfg["vocab"]
    r = orc.decode_stack(orc.make_model(cfg, w), oracle_state(orc, init), toks, logits=True)
    compare_logits(host(lw), r["logits"].reshape(B * T, V), f"tensor-core chain, {which}")
    compare_argmax(host(amw), r["logits"].reshape(B * T, V), f"tensor-core chain, {which}")
