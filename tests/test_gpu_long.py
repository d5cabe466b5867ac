"""The 24-layer configurations at the lengths they are stated at, against the oracle.

The method of "qwen3_5 cuda: mixed-width MLX checkpoints ... #849" (PR body:
logits compared with an fp32 reference at every position of a token check), on
this stack:
* batch 1, 128 decode tokens: the fp64 oracle decodes greedily on its own tokens;
  the GPU (one persistent launch per token) is teacher-forced on those tokens;
* 8 streams x 16-row windows, four windows in a row (64 rows per stream): the
  GPU's window launches on seeded tokens, streams 0 and 1 followed by the oracle.
Data flows oracle -> GPU only.  Through 24 bf16-rounded layers no fp32
evaluation stays within the per-stage bf16 tolerance end to end, so every
position is held to the bound the oracle sets for itself: the GPU's deviation
from the fp64 oracle is at most 1.5 times (plus a small floor) the deviation of
the oracle's own fp32 build, on the logits and on the final recurrent state;
argmax must match the fp64 oracle's on rows whose fp64 top-1/top-2 gap exceeds
four times that noise, and overall the GPU must pick the fp64 oracle's token at
least as often as the oracle's fp32 build does (less 5% of the rows): with
random-init weights most gaps are near-ties, where any fp32 evaluation may
pick either token.  Each oracle is run once per session (threads: the oracle releases the
interpreter lock while it computes).
"""
import functools
import queue
import threading

import numpy as np
import pytest

import hgd_synth as syn
from helpers import host, rel_l2
from stack_common import oracle_state, weights

pytestmark = pytest.mark.gpu

STEPS4 = 128            # config 4: greedy tokens at batch 1
B5, T5, WIN5 = 8, 16, 4  # config 5: streams, rows per window, windows in a row
FOLLOWED5 = (0, 1)      # streams followed by the oracle


@pytest.fixture(scope="module")
def hgd():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import __graft_entry__ as g
    g.build()
    import hybrid_gated_delta_b200 as m
    return m


@functools.lru_cache(maxsize=1)
def _oracles():
    from oracle import Oracle
    return Oracle(), Oracle(fp32=True)


@functools.lru_cache(maxsize=1)
def _config4_oracle():
    """fp64 oracle greedy on its own tokens (T = 1 per call), and the fp32 oracle
    teacher-forced on the same tokens as they appear (a second thread)."""
    cfg = syn.STACK_CFG
    w = weights("stack", 4)
    o64, o32 = _oracles()
    init = syn.stack_state(cfg, 1, 640, prefill=512, seed=4)
    tok0 = int(syn.stack_tokens(cfg, 1, 1, seed=4)[0, 0])
    q: "queue.Queue[int]" = queue.Queue()
    out = {"tok": [tok0], "l64": [], "l32": []}

    def run64():
        m = o64.make_model(cfg, w)
        st = oracle_state(o64, init)
        tok = tok0
        q.put(tok)
        for s in range(STEPS4):
            r = o64.decode_stack(m, st, np.array([[tok]], np.int32))
            out["l64"].append(r["logits"][0, 0].copy())
            tok = int(r["argmax"][0, 0])
            if s + 1 < STEPS4:
                out["tok"].append(tok)
                q.put(tok)
        out["S64"] = st["S"].copy()

    def run32():
        m = o32.make_model(cfg, w)
        st = oracle_state(o32, init)
        for _ in range(STEPS4):
            tok = q.get()
            r = o32.decode_stack(m, st, np.array([[tok]], np.int32))
            out["l32"].append(r["logits"][0, 0].astype(np.float64))
        out["S32"] = st["S"].astype(np.float64)

    th = [threading.Thread(target=run64), threading.Thread(target=run32)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert len(out["l64"]) == STEPS4 and len(out["l32"]) == STEPS4
    return init, out


def _within_noise(got, r64, r32, what, floor_rel=1e-3, floor_abs=1e-2):
    noise_rel = rel_l2(r32, r64)
    noise_max = float(np.abs(r32 - r64).max())
    got_rel = rel_l2(got, r64)
    got_max = float(np.abs(got - r64).max())
    assert got_rel <= 1.5 * noise_rel + floor_rel, f"{what}: relL2 {got_rel:.3g} vs fp32-oracle noise {noise_rel:.3g}"
    assert got_max <= 1.5 * noise_max + floor_abs, f"{what}: max|err| {got_max:.3g} vs noise {noise_max:.3g}"
    return noise_max


def _argmax_ok(got_logits, r64, r32, noise_max, what):
    """(rows checked strictly, GPU == fp64 token, fp32 oracle == fp64 token)."""
    lf = r64.astype(np.float32)
    ref = int(np.argmax(lf))
    g = int(np.argmax(got_logits))
    top2 = np.sort(lf)[-2:]
    strict = 0
    if top2[1] - top2[0] > 4 * noise_max:
        assert g == ref, what
        strict = 1
    return np.array([strict, int(g == ref), int(int(np.argmax(r32.astype(np.float32))) == ref)])


def _agreement_ok(counts, n, what):
    strict, gpu_same, f32_same = (int(v) for v in counts)
    assert gpu_same >= f32_same - 0.05 * n, (
        f"{what}: GPU picks the fp64 token at {gpu_same} of {n} rows, the fp32 oracle at {f32_same}")
    return strict, gpu_same, f32_same


def test_config4_128_greedy_tokens_vs_oracle(hgd):
    """24 layers, hidden 1024, vocab 248320, batch 1, KV context 512: all 128
    decode tokens of the configuration, every position's logits and argmax."""
    import torch
    cfg = syn.STACK_CFG
    init, r = _config4_oracle()
    model = hgd.Model(cfg, weights("stack", 4))
    st = hgd.State(model, 1, 1, 640, init)
    assert model.launches(1, 1) == 1
    V = cfg["vocab"]
    lg = torch.empty((1, V), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    counts = np.zeros(3, np.int64)
    for s in range(STEPS4):
        tok = torch.tensor([[r["tok"][s]]], dtype=torch.int32, device="cuda")
        hgd.decode_layer_stack(model, st, tok, 1, logits=lg, status=status)
        got = host(lg)[0]
        assert int(status.item()) == 0
        nm = _within_noise(got, r["l64"][s], r["l32"][s], f"token {s}")
        counts += _argmax_ok(got, r["l64"][s], r["l32"][s], nm, f"token {s} argmax")
    print("config 4 argmax (strict rows, GPU == fp64, fp32 == fp64):", _agreement_ok(counts, STEPS4, "config 4"))
    # the recurrent state after 128 tokens, every GDN layer and head together
    _within_noise(host(st.S), r["S64"], r["S32"], "state after 128 tokens", floor_rel=1e-4, floor_abs=1e-3)
    assert host(st.pos).tolist() == [512 + STEPS4]


@functools.lru_cache(maxsize=1)
def _config5_oracle():
    cfg = syn.STACK_CFG
    w = weights("stack", 4)
    o64, o32 = _oracles()
    init = syn.stack_state(cfg, B5, 768, prefill=512, seed=5)
    toks = syn.stack_tokens(cfg, B5, T5 * WIN5, seed=5)
    res = {}

    def run(o, b):
        m = o.make_model(cfg, w)
        st = oracle_state(o, init, streams=slice(b, b + 1))
        rr = o.decode_stack(m, st, toks[b:b + 1], logits=True)
        res[(o.real, b)] = (rr["logits"][0].astype(np.float64), st["S"].astype(np.float64))

    th = [threading.Thread(target=run, args=(o, b)) for o in (o64, o32) for b in FOLLOWED5]
    for t in th:
        t.start()
    for t in th:
        t.join()
    return init, toks, res


def test_config5_four_windows_vs_oracle(hgd):
    """8 streams x 16-row windows, four consecutive windows (64 rows per stream):
    streams 0 and 1 against the oracle at every row (logits, argmax) and in their
    recurrent state after the last window."""
    import torch
    cfg = syn.STACK_CFG
    init, toks, res = _config5_oracle()
    model = hgd.Model(cfg, weights("stack", 4))
    st = hgd.State(model, B5, T5, 768, init)
    V = cfg["vocab"]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = {b: [] for b in FOLLOWED5}
    for wi in range(WIN5):
        tk = torch.from_numpy(np.ascontiguousarray(toks[:, wi * T5:(wi + 1) * T5])).cuda()
        lg = torch.empty((B5 * T5, V), device="cuda")
        hgd.decode_layer_stack(model, st, tk, T5, logits=lg, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for b in FOLLOWED5:
            got[b].append(host(lg[b * T5:(b + 1) * T5]))
    counts = np.zeros(3, np.int64)
    for b in FOLLOWED5:
        g = np.concatenate(got[b], axis=0)
        l64, S64 = res[(np.float64, b)]
        l32, S32 = res[(np.float32, b)]
        for t in range(T5 * WIN5):
            nm = _within_noise(g[t], l64[t], l32[t], f"stream {b} row {t}")
            counts += _argmax_ok(g[t], l64[t], l32[t], nm, f"stream {b} row {t} argmax")
        _within_noise(host(st.S[:, b:b + 1]), S64, S32, f"stream {b} state after 64 rows",
                      floor_rel=1e-4, floor_abs=1e-3)
    print("config 5 argmax (strict rows, GPU == fp64, fp32 == fp64):",
          _agreement_ok(counts, T5 * WIN5 * len(FOLLOWED5), "config 5"))
    assert host(st.pos).tolist() == [512 + T5 * WIN5] * B5
