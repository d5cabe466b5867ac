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

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_CHUNK = 1 << 22
_POOL: ThreadPoolExecutor | None = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1))
    return _POOL

# ------------------------------------------------------------------ helpers --


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (nearest-even).  Input generation only."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = ((u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def keyed_normal_bf16(key: tuple, shape, std: float, mean: float = 0.0) -> np.ndarray:
    """N(mean, std) bf16 draws for a large tensor, generated in fixed 4M-element
    chunks, chunk i from PCG64(SeedSequence(key + (i,))): the values depend on the
    key only, never on the number of threads that fill them."""
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16)

    def fill(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key) + [i])))
        a = g.standard_normal(size=hi - lo, dtype=np.float32)
        if std != 1.0:
            a *= np.float32(std)
        if mean != 0.0:
            a += np.float32(mean)
        out[lo:hi] = to_bf16(a)

    nch = (n + _CHUNK - 1) // _CHUNK
    if nch <= 1:
        fill(0) if n else None
    else:
        list(_pool().map(fill, range(nch)))
    return out.reshape(shape)


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


_NAMES = ("in_norm", "w_in", "conv_w", "A_log", "dt_bias", "gnorm_w", "w_out", "post_norm", "w_gate",
          "w_up", "w_down")


def gdn_heads(cfg: dict) -> tuple[int, int]:
    """(key heads Hk, value heads H) of the GDN layers; gdn_v_heads 0 or absent: H = Hk."""
    Hk = cfg["gdn_heads"]
    return Hk, (cfg.get("gdn_v_heads") or Hk)


def stack_weights(cfg: dict, seed: int = 4, std: float = 0.02) -> dict:
    """Random-init bf16 weights N(0, std) with gains 1 + N(0, std).
    Returns {"embed", "final_norm", "layers": [dict per layer]} and, with
    cfg["untied_head"], "lm_head" [V, D]; the per-layer keys match the oracle's
    layer struct (in_norm, w_in, conv_w, A_log, dt_bias, gnorm_w, w_out,
    post_norm, w_gate, w_up, w_down).  Tensor (layer l, name) is drawn from the
    key (seed, l, name index); the model-level tensors use l = -1.  With Hk key
    and H value heads the GDN in-projection has rows q (Hk*dk) | k (Hk*dk) |
    v (H*dv) | z (H*dv) | a (H) | b (H)."""
    D, V = cfg["hidden"], cfg["vocab"]
    Hk, H = gdn_heads(cfg)
    dk, dv, kc = cfg["gdn_dk"], cfg["gdn_dv"], cfg["conv_k"]
    nq, nkv, hd, I = cfg["attn_q_heads"], cfg["attn_kv_heads"], cfg["attn_head_dim"], cfg["mlp_inter"]
    Cc = 2 * Hk * dk + H * dv

    def w_(l, name, shape, mean=0.0):
        return keyed_normal_bf16((seed, l + 1, _NAMES.index(name) if name in _NAMES else 99 + len(name)),
                                 shape, std, mean)

    w = {"embed": w_(-1, "embed", (V, D)), "final_norm": w_(-1, "final_norm", (D,), 1.0), "layers": []}
    if cfg.get("untied_head"):
        w["lm_head"] = w_(-1, "lm_head", (V, D))
    for l in range(cfg["n_layers"]):
        lw = {"in_norm": w_(l, "in_norm", (D,), 1.0)}
        if not is_attn(cfg, l):
            lw["w_in"] = w_(l, "w_in", (Cc + H * dv + 2 * H, D))
            lw["conv_w"] = w_(l, "conv_w", (Cc, kc))
            lw["A_log"] = w_(l, "A_log", (H,))
            lw["dt_bias"] = w_(l, "dt_bias", (H,))
            lw["gnorm_w"] = w_(l, "gnorm_w", (dv,), 1.0)
            lw["w_out"] = w_(l, "w_out", (D, H * dv))
        else:
            lw["w_in"] = w_(l, "w_in", (2 * nq * hd + 2 * nkv * hd, D))
            lw["w_out"] = w_(l, "w_out", (D, nq * hd))
        lw["post_norm"] = w_(l, "post_norm", (D,), 1.0)
        lw["w_gate"] = w_(l, "w_gate", (I, D))
        lw["w_up"] = w_(l, "w_up", (I, D))
        lw["w_down"] = w_(l, "w_down", (D, I))
        w["layers"].append(lw)
    return w


def stack_state(cfg: dict, B: int, Lmax: int, prefill: int = 512, seed: int = 4) -> dict:
    """Initial decode state: S ~ N(0,0.1) fp32, conv tails ~ N(0,1) fp32, KV cache
    rows 0..prefill-1 ~ N(0,1) bf16 (keys taken as already rotated), rows past it
    zero; every stream starts at position `prefill`."""
    n_gdn, n_attn = layer_counts(cfg)
    Hk, H = gdn_heads(cfg)
    dk, dv, kc = cfg["gdn_dk"], cfg["gdn_dv"], cfg["conv_k"]
    nkv, hd = cfg["attn_kv_heads"], cfg["attn_head_dim"]
    Cc = 2 * Hk * dk + H * dv
    g = rng(seed * 31 + 17 + B)
    kv = np.zeros((n_attn, 2, B, nkv, Lmax, hd), np.uint16)
    if prefill > 0:
        kv[..., :prefill, :] = keyed_normal_bf16((seed, 7001, B), (n_attn, 2, B, nkv, prefill, hd), 1.0)
    return dict(
        S=normal_f32(g, (n_gdn, B, H, dv, dk), 0.1),
        tail=normal_f32(g, (n_gdn, B, kc - 1, Cc), 1.0),
        kv=kv,
        pos=np.full((B,), prefill, np.int32),
    )


def stack_tokens(cfg: dict, B: int, n: int, seed: int = 4) -> np.ndarray:
    """Token ids uniform in [0, vocab), [B, n]."""
    return rng(seed * 131 + 7 + B).integers(0, cfg["vocab"], size=(B, n), dtype=np.int32)
