"""Shared set-up of the stack parity tests: seeded weights/state for both sides,
GPU model/state construction, oracle runs and the comparisons."""
import functools

import numpy as np

import hgd_synth as syn
from helpers import BF16_MAX_ABS, BF16_REL_L2, STATE_REL_L2, host, rel_l2

ARGMAX_MARGIN = 2e-2  # rows whose oracle top-1/top-2 gap is below this are reported, not failed


@functools.lru_cache(maxsize=2)
def weights(cfg_key: str, seed: int):
    cfg = syn.STACK_CFG if cfg_key == "stack" else syn.SMALL_CFG
    return syn.stack_weights(cfg, seed=seed)


def oracle_state(orc, init, streams=None):
    sel = slice(None) if streams is None else streams
    st = {"S": init["S"][:, sel].astype(orc.real).copy(), "tail": init["tail"][:, sel].astype(orc.real).copy(),
          "kv": np.ascontiguousarray(init["kv"][:, :, sel]).copy(), "pos": init["pos"][sel].copy()}
    return st


def compare_logits(got, ref, what):
    """got, ref [rows, V]: bf16-class tolerance on the logits."""
    mx = np.abs(got - ref).max()
    rl = rel_l2(got, ref)
    assert mx <= BF16_MAX_ABS and rl <= BF16_REL_L2, f"{what}: logits max|err|={mx:.3g} relL2={rl:.3g}"
    return mx, rl


def compare_argmax(got, ref_logits, what):
    """Identical argmax on every row whose oracle top-1/top-2 gap exceeds the margin."""
    lf = ref_logits.astype(np.float32)
    close = []
    for r in range(lf.shape[0]):
        top2 = np.partition(lf[r], -2)[-2:]
        gap = float(top2[1] - top2[0])
        ref = int(np.argmax(lf[r]))
        if gap > ARGMAX_MARGIN:
            assert int(got[r]) == ref, f"{what}: row {r} argmax {int(got[r])} != {ref} (gap {gap:.3g})"
        else:
            close.append((r, gap))
    return close


def compare_state_rel(got, ref, what, heads_axis=True):
    """fp32 recurrent state, relative L2 <= 1e-4 per trailing 2-D block: per head
    for S [..., H, dv, dk], per row record for conv tails [..., kc-1, C]."""
    g = got.reshape(-1, got.shape[-2] * got.shape[-1])
    r = ref.reshape(-1, ref.shape[-2] * ref.shape[-1])
    worst = 0.0
    for i in range(g.shape[0]):
        worst = max(worst, rel_l2(g[i], r[i]))
    assert worst <= STATE_REL_L2, f"{what}: worst per-head relL2 {worst:.3g}"
    return worst
