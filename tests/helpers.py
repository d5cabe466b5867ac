"""Shared helpers of the GPU parity tests (host <-> device marshalling and the
tolerances).  Tolerances: bf16 outputs max-abs <= 2e-2 and relative L2 <= 5e-3;
the fp32 recurrent state relative L2 <= 1e-4 per step and per head."""
import numpy as np

import hgd_synth as syn

BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
STATE_REL_L2 = 1e-4


def dev_bf16(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


def dev_f32(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return syn.from_bf16(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (den if den > 0 else 1.0)


def bf16_quantum(v):
    """Spacing of bf16 values at |v| (2^(e-7) for 2^e <= |v| < 2^(e+1))."""
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_bf16_close(got, ref, what=""):
    """bf16 outputs: relative L2 <= 5e-3, and every element within 2e-2 of the
    reference or, where one bf16 rounding quantum of the reference is larger than
    2e-2 (|ref| >= 4), within one quantum: a correctly rounded bf16 result is off
    by one quantum when its fp32 value and the reference straddle a midpoint."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    allow = np.maximum(BF16_MAX_ABS, bf16_quantum(ref))
    mx = err.max() if got.size else 0.0
    over = (err - allow).max() if got.size else 0.0
    rl = rel_l2(got, ref)
    assert over <= 0 and rl <= BF16_REL_L2, f"{what}: max|err|={mx:.3g} (over bound {over:.3g}) relL2={rl:.3g}"
    return mx, rl


def fp32_dot_bound(W, x):
    """|fp32 dot - exact| <= gamma_K * sum|w||x| (products exact); elementwise [M,N]."""
    K = W.shape[1]
    g = K * 2.0 ** -24 / (1 - K * 2.0 ** -24)
    return g * (np.abs(syn.from_bf16(x)).astype(np.float64) @ np.abs(syn.from_bf16(W)).astype(np.float64).T)
