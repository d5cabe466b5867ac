"""Seeded synthetic inputs for the hybrid gated-delta decode step.

This module only draws random numbers: it holds none of the method's arithmetic
and is shared, read-only, by the oracle side and the CUDA side of every test and
by the benchmark.  Every array is host numpy; bf16 tensors are uint16 bit
patterns obtained by rounding float32 draws to nearest-even.

Distribution readings (the configurations write N(0, s)):
  * "N(0,1/K)" is a variance (LeCun fan-in init), std = 1/sqrt(K);
  * a decimal such as N(0,0.02) or N(0,0.1) is a standard deviation, as in
    the usual initializer_range convention;
  * norm gains are 1 + N(0,0.02) (a literal N(0,0.02) gain would zero the stream).
"""
from __future__ import annotations

import numpy as np

# ------------------------------------------------------------------ helpers --


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (nearest-even).  Input generation only."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    r = ((u.astype(np.uint64) + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def from_bf16(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(g: np.random.Generator, shape, std: float, mean: float = 0.0) -> np.ndarray:
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if mean != 0.0:
        a += np.float32(mean)
    return to_bf16(a)


def normal_f32(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def neg_softplus_normal(g: np.random.Generator, shape) -> np.ndarray:
    """g = -softplus(N(0,1)) in float32 (the log-decay input of the GDN configs).
    The draw is transformed in float64 and stored as float32; both sides then read
    the same float32 values."""
    z = g.standard_normal(size=shape).astype(np.float64)
    return (-(np.maximum(z, 0) + np.log1p(np.exp(-np.abs(z))))).astype(np.float32)


# ------------------------------------------------------ config 1: tiny GDN --

TINY = dict(D=256, H=4, d=64, kc=4, T=8)


def tiny_gdn(seed: int = 1, T: int = 8) -> dict:
    """One GDN mixer without norm/z-gate: hidden 256, 4 heads, d=64, conv over
    3*256 channels, T steps of one stream."""
    D, H, d, kc = TINY["D"], TINY["H"], TINY["d"], TINY["kc"]
    C = 3 * H * d
    g = rng(seed)
    return dict(
        x=normal_bf16(g, (T, D), 1.0),
        W_qkv=normal_bf16(g, (C, D), 1.0 / np.sqrt(D)),
        W_o=normal_bf16(g, (D, H * d), 1.0 / np.sqrt(H * d)),
        conv_w=normal_bf16(g, (C, kc), 1.0 / np.sqrt(kc)),
        S=normal_f32(g, (1, H, d, d), 0.1),
        tail=normal_f32(g, (1, kc - 1, C), 1.0),
        g=neg_softplus_normal(g, (1, T, H)),
        b=normal_f32(g, (1, T, H), 1.0),
        D=D, H=H, d=d, kc=kc, C=C, T=T,
    )


# ------------------------------------------------------ config 2: GEMV sweep --

GEMV_SHAPES = {
    # name: (N, K)  -- hidden 1536, MLP 4096, vocab 100000
    "qkvo": (1536, 1536),
    "down": (1536, 4096),
    "lm_head": (100000, 1536),
}
SWIGLU_SHAPE = (4096, 1536)  # (I, K): up/gate fused
GEMV_M = (1, 2, 4, 8, 16, 32)


def gemv_case(N: int, K: int, M: int, seed: int = 2) -> dict:
    g = rng(seed * 1000003 + N * 7 + K * 13 + M)
    return dict(W=normal_bf16(g, (N, K), 1.0 / np.sqrt(K)), x=normal_bf16(g, (M, K), 1.0))


def swiglu_case(I: int, K: int, M: int, seed: int = 2) -> dict:
    g = rng(seed * 1000033 + I * 7 + K * 13 + M)
    return dict(Wg=normal_bf16(g, (I, K), 1.0 / np.sqrt(K)),
                Wu=normal_bf16(g, (I, K), 1.0 / np.sqrt(K)),
                x=normal_bf16(g, (M, K), 1.0))


# ------------------------------------------------------ config 3: GDN sweep --

GDN_SWEEP_B = (1, 4, 16, 64)


def gdn_sweep(B: int, steps: int = 256, H: int = 16, d: int = 128, seed: int = 3) -> dict:
    """Initial state and per-step inputs of the state-update sweep."""
    g = rng(seed * 7919 + B)
    return dict(
        S=normal_f32(g, (B, H, d, d), 0.1),
        q=normal_f32(g, (steps, B, 1, H, d)),
        k=normal_f32(g, (steps, B, 1, H, d)),
        v=normal_f32(g, (steps, B, 1, H, d)),
        g=neg_softplus_normal(g, (steps, B, 1, H)),
        b=normal_f32(g, (steps, B, 1, H)),
    )


# ---------------------------------------------------- configs 4/5: the stack --

STACK_CFG = dict(n_layers=24, hidden=1024, vocab=248320, gdn_heads=16, gdn_dk=128, gdn_dv=128,
                 conv_k=4, attn_q_heads=8, attn_kv_heads=2, attn_head_dim=256, mlp_inter=3584,
                 attn_every=4, norm_eps=1e-6, rope_base=10000.0)

# A reduced geometry of the same family for fast tests (every code path, small sizes).
SMALL_CFG = dict(n_layers=4, hidden=256, vocab=1000, gdn_heads=2, gdn_dk=64, gdn_dv=64,
                 conv_k=4, attn_q_heads=4, attn_kv_heads=2, attn_head_dim=64, mlp_inter=512,
                 attn_every=4, norm_eps=1e-6, rope_base=10000.0)


def is_attn(cfg: dict, l: int) -> bool:
    return l % cfg["attn_every"] == cfg["attn_every"] - 1


def layer_counts(cfg: dict) -> tuple[int, int]:
    n_attn = sum(is_attn(cfg, l) for l in range(cfg["n_layers"]))
    return cfg["n_layers"] - n_attn, n_attn


def stack_weights(cfg: dict, seed: int = 4, std: float = 0.02) -> dict:
    """Random-init bf16 weights N(0, std) with gains 1 + N(0, std).
    Returns {"embed", "final_norm", "layers": [dict per layer]}; the per-layer keys
    match the oracle's layer struct (in_norm, w_in, conv_w, A_log, dt_bias, gnorm_w,
    w_out, post_norm, w_gate, w_up, w_down)."""
    D, V, H = cfg["hidden"], cfg["vocab"], cfg["gdn_heads"]
    dk, dv, kc = cfg["gdn_dk"], cfg["gdn_dv"], cfg["conv_k"]
    nq, nkv, hd, I = cfg["attn_q_heads"], cfg["attn_kv_heads"], cfg["attn_head_dim"], cfg["mlp_inter"]
    Cc = 2 * H * dk + H * dv
    g = rng(seed)
    w = {"embed": normal_bf16(g, (V, D), std), "final_norm": normal_bf16(g, (D,), std, 1.0),
         "layers": []}
    for l in range(cfg["n_layers"]):
        lw = {"in_norm": normal_bf16(g, (D,), std, 1.0)}
        if not is_attn(cfg, l):
            lw["w_in"] = normal_bf16(g, (Cc + H * dv + 2 * H, D), std)
            lw["conv_w"] = normal_bf16(g, (Cc, kc), std)
            lw["A_log"] = normal_bf16(g, (H,), std)
            lw["dt_bias"] = normal_bf16(g, (H,), std)
            lw["gnorm_w"] = normal_bf16(g, (dv,), std, 1.0)
            lw["w_out"] = normal_bf16(g, (D, H * dv), std)
        else:
            lw["w_in"] = normal_bf16(g, (2 * nq * hd + 2 * nkv * hd, D), std)
            lw["w_out"] = normal_bf16(g, (D, nq * hd), std)
        lw["post_norm"] = normal_bf16(g, (D,), std, 1.0)
        lw["w_gate"] = normal_bf16(g, (I, D), std)
        lw["w_up"] = normal_bf16(g, (I, D), std)
        lw["w_down"] = normal_bf16(g, (D, I), std)
        w["layers"].append(lw)
    return w


def stack_state(cfg: dict, B: int, Lmax: int, prefill: int = 512, seed: int = 4) -> dict:
    """Initial decode state: S ~ N(0,0.1) fp32, conv tails ~ N(0,1) fp32, KV cache
    rows 0..prefill-1 ~ N(0,1) bf16 (keys taken as already rotated), rows past it
    zero; every stream starts at position `prefill`."""
    n_gdn, n_attn = layer_counts(cfg)
    H, dk, dv, kc = cfg["gdn_heads"], cfg["gdn_dk"], cfg["gdn_dv"], cfg["conv_k"]
    nkv, hd = cfg["attn_kv_heads"], cfg["attn_head_dim"]
    Cc = 2 * H * dk + H * dv
    g = rng(seed * 31 + 17 + B)
    kv = np.zeros((n_attn, 2, B, nkv, Lmax, hd), np.uint16)
    if prefill > 0:
        kv[..., :prefill, :] = normal_bf16(g, (n_attn, 2, B, nkv, prefill, hd), 1.0)
    return dict(
        S=normal_f32(g, (n_gdn, B, H, dv, dk), 0.1),
        tail=normal_f32(g, (n_gdn, B, kc - 1, Cc), 1.0),
        kv=kv,
        pos=np.full((B,), prefill, np.int32),
    )


def stack_tokens(cfg: dict, B: int, n: int, seed: int = 4) -> np.ndarray:
    """Token ids uniform in [0, vocab), [B, n]."""
    return rng(seed * 131 + 7 + B).integers(0, cfg["vocab"], size=(B, n), dtype=np.int32)
