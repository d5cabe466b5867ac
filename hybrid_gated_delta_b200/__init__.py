"""Python binding of libhgd, the sm_100a hybrid gated-delta decode library.

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libhgd.so; PyTorch supplies device memory and streams.  The entry
points have the names of the C ABI in include/hgd.h.  If the library is not
built, importing this package raises instead of falling back to anything.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhgd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libhgd.so is not built ({LIB_PATH}); run "
                      "`python -c 'import __graft_entry__ as g; g.build()'`")

_lib = C.CDLL(LIB_PATH)

HGD_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "misaligned",
          4: "CUDA error", 5: "timeout", 6: "not co-resident", 7: "NaN logit",
          8: "unsupported device", 9: "buffer too small"}

MAX_LAYERS = 64
W_IN_NORM, W_IN, W_CONV, W_A_LOG, W_DT_BIAS, W_GNORM, W_OUT, W_POST_NORM, W_GATE, W_UP, W_DOWN = range(11)
W_LAYER_COUNT = 11
W_EMBED, W_FINAL_NORM, W_LM_HEAD = 100, 101, 102
LAYER_TENSORS = {"in_norm": W_IN_NORM, "w_in": W_IN, "conv_w": W_CONV, "A_log": W_A_LOG,
                 "dt_bias": W_DT_BIAS, "gnorm_w": W_GNORM, "w_out": W_OUT, "post_norm": W_POST_NORM,
                 "w_gate": W_GATE, "w_up": W_UP, "w_down": W_DOWN}
S_GDN, S_CONV, S_KV, S_POS, S_RESID = range(5)


class HgdError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({STATUS.get(code, 'unknown')})")
        self.code = code


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("hidden", C.c_int32), ("vocab", C.c_int32),
                ("gdn_heads", C.c_int32), ("gdn_dk", C.c_int32), ("gdn_dv", C.c_int32),
                ("conv_k", C.c_int32), ("attn_q_heads", C.c_int32), ("attn_kv_heads", C.c_int32),
                ("attn_head_dim", C.c_int32), ("mlp_inter", C.c_int32), ("attn_every", C.c_int32),
                ("norm_eps", C.c_float), ("rope_base", C.c_float), ("gdn_v_heads", C.c_int32),
                ("untied_head", C.c_int32)]


class _Model(C.Structure):
    _fields_ = [("cfg", Config), ("embed", C.c_void_p), ("final_norm", C.c_void_p),
                ("w", (C.c_void_p * W_LAYER_COUNT) * MAX_LAYERS), ("arena_bytes", C.c_size_t),
                ("lm_head", C.c_void_p), ("tcw", (C.c_void_p * 4) * MAX_LAYERS), ("tc_head", C.c_void_p)]


class _State(C.Structure):
    _fields_ = [("B", C.c_int32), ("Tmax", C.c_int32), ("Lmax", C.c_int32),
                ("arena", C.c_void_p), ("arena_bytes", C.c_size_t), ("off", C.c_size_t * 32)]


_p, _i, _i64, _sz = C.c_void_p, C.c_int, C.c_int64, C.c_size_t
_SIGS = {
    "hgd_status_string": ([_i], C.c_char_p),
    "hgd_version": ([], _i),
    "hgd_gemv_bf16": ([_p, _p, _p, _i, _i, _i, _i, _p, _sz, _p], _i),
    "hgd_gemv_workspace_bytes": ([_i, _i, _i, _i, C.POINTER(_sz)], _i),
    "hgd_gemv_bf16_static_ws": ([_p, _p, _p, _i, _i, _i, _i, _p], _i),
    "hgd_gemv_swiglu_bf16": ([_p, _p, _p, _p, _i, _i, _i, _p, _sz, _p], _i),
    "hgd_check_bounded_wait": ([_p, _p], _i),
    "hgd_gemm_tc_weight_bytes": ([_i, _i, C.POINTER(_sz)], _i),
    "hgd_gemm_tc_pack_weight": ([_p, _p, _i, _i, _p], _i),
    "hgd_gemm_tc_workspace_bytes": ([_i, _i, _i, C.POINTER(_sz)], _i),
    "hgd_gemm_tc_plan": ([_i, _i, _i, C.POINTER(_i), C.POINTER(_i)], _i),
    "hgd_gemm_tc_bf16": ([_p, _p, _p, _i, _i, _i, _p, _sz, _p, _p], _i),
    "hgd_conv1d_tail_update": ([_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p], _i),
    "hgd_gdn_decode_step": ([_p, _p, _p, _i64, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p], _i),
    "hgd_gdn_decode_step_grouped": ([_p, _p, _p, _i64, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p],
                                    _i),
    "hgd_gdn_prefill": ([_p, _p, _p, _i64, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p], _i),
    "hgd_gdn_window_log": ([_p, _p, _p, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p], _i),
    "hgd_gdn_keep": ([_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p], _i),
    "hgd_conv1d_keep": ([_p, _p, _p, _p, _i, _i, _i, _i, _p], _i),
    "hgd_model_arena_bytes": ([C.POINTER(Config), C.POINTER(_sz)], _i),
    "hgd_model_tensor": ([C.POINTER(Config), _i, _i, C.POINTER(_sz), C.POINTER(_sz)], _i),
    "hgd_model_init": ([C.POINTER(_Model), C.POINTER(Config), _p, _sz], _i),
    "hgd_model_load_tensor": ([C.POINTER(Config), _p, _sz, _i, _i, _p, _p], _i),
    "hgd_state_arena_bytes": ([C.POINTER(Config), _i, _i, _i, C.POINTER(_sz)], _i),
    "hgd_state_tensor": ([C.POINTER(Config), _i, _i, _i, _i, C.POINTER(_sz), C.POINTER(_sz)], _i),
    "hgd_state_init": ([C.POINTER(_State), C.POINTER(_Model), _i, _i, _i, _p, _sz], _i),
    "hgd_decode_layer_stack": ([C.POINTER(_Model), C.POINTER(_State), _p, _i, _p, _p, _p, _p, _p, _p], _i),
    "hgd_decode_layer_stack_range": ([C.POINTER(_Model), C.POINTER(_State), _p, _i, _i, _i, _i, _p, _p, _p,
                                      _p, _p, _p], _i),
    "hgd_decode_layer_stack_launches": ([C.POINTER(_Model), _i, _i], _i),
    "hgd_verify_log_bytes": ([C.POINTER(Config), _i, _i, C.POINTER(_sz)], _i),
    "hgd_decode_layer_stack_verify": ([C.POINTER(_Model), C.POINTER(_State), _p, _i, _p, _p, _p, _sz, _p, _p], _i),
    "hgd_decode_layer_stack_keep": ([C.POINTER(_Model), C.POINTER(_State), _i, _p, _sz, _p, _p, _p], _i),
    "hgd_model_tc_bytes": ([C.POINTER(Config), C.POINTER(_sz)], _i),
    "hgd_model_tc_load": ([C.POINTER(Config), _p, _sz, _i, _i, _p, _p], _i),
    "hgd_model_attach_tc": ([C.POINTER(_Model), _p, _sz], _i),
    "hgd_decode_layer_stack_tc": ([C.POINTER(_Model), C.POINTER(_State), _p, _i, _p, _p, _p, _p, _p, _p], _i),
    "hgd_check_stack_timeout": ([C.POINTER(_Model), C.POINTER(_State), _p, _i, _p, _i, _i, _i, _p, _p, _p], _i),
    "hgd_check_not_coresident": ([C.POINTER(_Model), C.POINTER(_State), _i], _i),
}
for _name, (_args, _ret) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _ret

EXPORTED = tuple(_SIGS)


def _check(fn: str, rc: int) -> None:
    if rc != HGD_OK:
        raise HgdError(fn, rc)


def version() -> int:
    return _lib.hgd_version()


def status_string(code: int) -> str:
    return _lib.hgd_status_string(code).decode()


# --------------------------------------------------------------- helpers ----

def _torch():
    import torch
    return torch


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libhgd must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t, dtype, name):
    torch = _torch()
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")


# -------------------------------------------------------------- entry points

def gemv_workspace_bytes(M: int, N: int, K: int, swiglu: bool = False) -> int:
    n = C.c_size_t()
    _check("hgd_gemv_workspace_bytes", _lib.hgd_gemv_workspace_bytes(M, N, K, int(swiglu), C.byref(n)))
    return n.value


def make_workspace(M: int, N: int, K: int, swiglu: bool = False, device="cuda"):
    """A zero-filled split-K workspace for GEMVs of this shape (None if unused)."""
    torch = _torch()
    n = gemv_workspace_bytes(M, N, K, swiglu)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device) if n else None


def gemv_bf16(W, x, y=None, y_is_fp32=True, workspace=None, stream=None):
    """y[M,N] = x[M,K] . W[N,K]^T (bf16 in, fp32 accumulate)."""
    torch = _torch()
    _need(W, torch.bfloat16, "W")
    _need(x, torch.bfloat16, "x")
    N, K = W.shape
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32 if y_is_fp32 else torch.bfloat16, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("hgd_gemv_bf16", _lib.hgd_gemv_bf16(_ptr(W), _ptr(x), _ptr(y), int(y.dtype == torch.float32),
                                                M, N, K, _ptr(workspace), ws_bytes, _stream(stream)))
    return y


def check_bounded_wait(status, stream=None):
    """Run a bounded in-kernel wait that nothing completes; HGD_ERR_TIMEOUT lands in status."""
    _check("hgd_check_bounded_wait", _lib.hgd_check_bounded_wait(_ptr(status), _stream(stream)))


def gemm_tc_pack_weight(W, stream=None):
    """W [N,K] bf16 -> the tensor-core GEMM's packed weight (uint8 device tensor)."""
    torch = _torch()
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    n = C.c_size_t()
    _check("hgd_gemm_tc_weight_bytes", _lib.hgd_gemm_tc_weight_bytes(N, K, C.byref(n)))
    Wp = torch.empty(n.value, dtype=torch.uint8, device=W.device)
    _check("hgd_gemm_tc_pack_weight", _lib.hgd_gemm_tc_pack_weight(_ptr(W), _ptr(Wp), N, K, _stream(stream)))
    return Wp


def gemm_tc_workspace_bytes(M: int, N: int, K: int) -> int:
    n = C.c_size_t()
    _check("hgd_gemm_tc_workspace_bytes", _lib.hgd_gemm_tc_workspace_bytes(M, N, K, C.byref(n)))
    return n.value


def gemm_tc_bf16(Wp, x, N, y=None, workspace=None, status=None, stream=None):
    """y[M,N] fp32 = x[M,K] . W[N,K]^T on the tensor cores; Wp from gemm_tc_pack_weight."""
    torch = _torch()
    _need(x, torch.bfloat16, "x")
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(gemm_tc_workspace_bytes(M, N, K), dtype=torch.uint8, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("hgd_gemm_tc_bf16", _lib.hgd_gemm_tc_bf16(_ptr(Wp), _ptr(x), _ptr(y), M, N, K, _ptr(workspace),
                                                      ws_bytes, _ptr(status), _stream(stream)))
    return y


def gemv_swiglu_bf16(W_gate, W_up, x, h=None, workspace=None, stream=None):
    """h[M,I] = bf16(silu(x W_gate^T) * (x W_up^T))."""
    torch = _torch()
    for t, n in ((W_gate, "W_gate"), (W_up, "W_up"), (x, "x")):
        _need(t, torch.bfloat16, n)
    I, K = W_gate.shape
    M = x.shape[0]
    if h is None:
        h = torch.empty((M, I), dtype=torch.bfloat16, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("hgd_gemv_swiglu_bf16", _lib.hgd_gemv_swiglu_bf16(_ptr(W_gate), _ptr(W_up), _ptr(x), _ptr(h),
                                                              M, I, K, _ptr(workspace), ws_bytes,
                                                              _stream(stream)))
    return h


def conv1d_tail_update(x, tail, w, y=None, tail_rec=None, apply_silu=True, stream=None):
    """x [B,T,C] fp32, tail [B,kc-1,C] fp32 (in place), w [C,kc] bf16."""
    torch = _torch()
    _need(x, torch.float32, "x")
    _need(tail, torch.float32, "tail")
    _need(w, torch.bfloat16, "w")
    B, T, Cc = x.shape
    kc = w.shape[1]
    if y is None:
        y = torch.empty_like(x)
    _check("hgd_conv1d_tail_update", _lib.hgd_conv1d_tail_update(
        _ptr(x), _ptr(tail), _ptr(w), _ptr(y), _ptr(tail_rec), B, T, Cc, kc, int(apply_silu),
        _stream(stream)))
    return y


def gdn_decode_step(q, k, v, g, b, S, o=None, o_bf16=None, S_rec=None, l2norm_qk=True,
                    row_stride=None, B=None, T=None, stream=None):
    """Gated delta rule rows.  q,k [B,T,H,dk], v [B,T,H,dv] fp32 (or views into one
    packed [B*T, row_stride] buffer with row_stride given), g,b [B,T,H] fp32,
    S [B,H,dv,dk] fp32 in place.  Returns o [B,T,H,dv] fp32."""
    torch = _torch()
    _need(S, torch.float32, "S")
    Bs, H, dv, dk = S.shape
    Tn = g.shape[1] if T is None else T
    Bn = Bs if B is None else B
    if row_stride is None:
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _need(t, torch.float32, n)
            if not t.is_contiguous():
                raise ValueError(f"{n} must be contiguous")
        row_stride = H * dk
        qp, kp, vp = q.data_ptr(), k.data_ptr(), v.data_ptr()
    else:
        qp, kp, vp = q.data_ptr(), k.data_ptr(), v.data_ptr()
    if o is None:
        o = torch.empty((Bn, Tn, H, dv), dtype=torch.float32, device=S.device)
    _check("hgd_gdn_decode_step", _lib.hgd_gdn_decode_step(
        qp, kp, vp, int(row_stride), _ptr(g), _ptr(b), _ptr(S), _ptr(o), _ptr(o_bf16), _ptr(S_rec),
        Bn, Tn, H, dk, dv, int(l2norm_qk), _stream(stream)))
    return o


def gdn_decode_step_grouped(q, k, v, g, b, S, key_heads: int, row_stride: int, B: int, T: int, o=None,
                            o_bf16=None, S_rec=None, l2norm_qk=True, stream=None):
    """Gated delta rule rows with S's value heads over `key_heads` query/key heads
    (value head h reads key head h // (H // key_heads)); q, k, v are views into one
    packed [B*T, row_stride] buffer.  Returns o [B,T,H,dv]."""
    torch = _torch()
    _need(S, torch.float32, "S")
    _, H, dv, dk = S.shape
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=S.device)
    _check("hgd_gdn_decode_step_grouped", _lib.hgd_gdn_decode_step_grouped(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), int(row_stride), _ptr(g), _ptr(b), _ptr(S), _ptr(o), _ptr(o_bf16),
        _ptr(S_rec), B, T, key_heads, H, dk, dv, int(l2norm_qk), _stream(stream)))
    return o


def gdn_prefill(q, k, v, g, b, S, o=None, l2norm_qk=True, row_stride=None, B=None, T=None, stream=None):
    """The T rows of a prompt through the gated delta rule, a chunk at a time
    (same arguments and results as gdn_decode_step, to fp32 rounding).
    Returns o [B,T,H,dv]."""
    torch = _torch()
    _need(S, torch.float32, "S")
    Bs, H, dv, dk = S.shape
    Tn = g.shape[1] if T is None else T
    Bn = Bs if B is None else B
    if row_stride is None:
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _need(t, torch.float32, n)
            if not t.is_contiguous():
                raise ValueError(f"{n} must be contiguous")
        row_stride = H * dk
    if o is None:
        o = torch.empty((Bn, Tn, H, dv), dtype=torch.float32, device=S.device)
    _check("hgd_gdn_prefill", _lib.hgd_gdn_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), int(row_stride),
                                                   _ptr(g), _ptr(b), _ptr(S), _ptr(o), Bn, Tn, H, dk, dv,
                                                   int(l2norm_qk), _stream(stream)))
    return o


def gdn_window_log(q, k, v, g, b, S, o=None, o_bf16=None, l2norm_qk=True, row_stride=None, B=None, T=None,
                   stream=None):
    """The rows of gdn_decode_step with S only read; returns (o, log_alpha [B,T,H],
    log_delta [B,T,H,dv], log_k [B,T,H,dk])."""
    torch = _torch()
    _need(S, torch.float32, "S")
    Bs, H, dv, dk = S.shape
    Tn = g.shape[1] if T is None else T
    Bn = Bs if B is None else B
    if row_stride is None:
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _need(t, torch.float32, n)
            if not t.is_contiguous():
                raise ValueError(f"{n} must be contiguous")
        row_stride = H * dk
    dev = S.device
    if o is None:
        o = torch.empty((Bn, Tn, H, dv), dtype=torch.float32, device=dev)
    la = torch.empty((Bn, Tn, H), dtype=torch.float32, device=dev)
    ld = torch.empty((Bn, Tn, H, dv), dtype=torch.float32, device=dev)
    lk = torch.empty((Bn, Tn, H, dk), dtype=torch.float32, device=dev)
    _check("hgd_gdn_window_log", _lib.hgd_gdn_window_log(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), int(row_stride), _ptr(g), _ptr(b), _ptr(S), _ptr(o),
        _ptr(o_bf16), _ptr(la), _ptr(ld), _ptr(lk), Bn, Tn, H, dk, dv, int(l2norm_qk), _stream(stream)))
    return o, la, ld, lk


def gdn_keep(S, log_alpha, log_delta, log_k, keep, status=None, stream=None):
    """S [B,H,dv,dk] takes the first keep[b] logged rows of each stream (keep: int32 [B] device)."""
    torch = _torch()
    _need(S, torch.float32, "S")
    _need(keep, torch.int32, "keep")
    B, H, dv, dk = S.shape
    T = log_alpha.shape[1]
    _check("hgd_gdn_keep", _lib.hgd_gdn_keep(_ptr(S), _ptr(log_alpha), _ptr(log_delta), _ptr(log_k), _ptr(keep),
                                             _ptr(status), B, T, H, dk, dv, _stream(stream)))


def conv1d_keep(tail, x, keep, status=None, stream=None):
    """tail [B,kc-1,C] takes the first keep[b] rows of x [B,T,C]."""
    torch = _torch()
    _need(tail, torch.float32, "tail")
    _need(x, torch.float32, "x")
    _need(keep, torch.int32, "keep")
    B, nt, Cc = tail.shape
    _check("hgd_conv1d_keep", _lib.hgd_conv1d_keep(_ptr(tail), _ptr(x), _ptr(keep), _ptr(status), B, x.shape[1],
                                                   Cc, nt + 1, _stream(stream)))


# ------------------------------------------------------------------ stack

def make_config(cfg: dict) -> Config:
    c = Config()
    for name, _ in Config._fields_:
        setattr(c, name, cfg.get(name, 0) if name in ("gdn_v_heads", "untied_head") else cfg[name])
    return c


def gdn_heads(cfg: dict) -> tuple:
    """(query/key heads, value heads) of the GDN layers."""
    return cfg["gdn_heads"], (cfg.get("gdn_v_heads") or cfg["gdn_heads"])


class Model:
    """Weights in one device arena laid out by libhgd (hgd_model_tensor offsets).
    With tc=True the weights are also packed for the tensor-core decode chain
    (hgd_decode_layer_stack_tc) into a second arena."""

    def __init__(self, cfg: dict, weights: dict, device="cuda", tc: bool = False):
        torch = _torch()
        self.cfg_dict = dict(cfg)
        self.cfg = make_config(cfg)
        nbytes = C.c_size_t()
        _check("hgd_model_arena_bytes", _lib.hgd_model_arena_bytes(C.byref(self.cfg), C.byref(nbytes)))
        self.arena = torch.zeros(nbytes.value // 2 + 128, dtype=torch.int16, device=device)
        base = self.arena.data_ptr()
        pad = (-base) % 256
        self.arena_u8 = self.arena.view(torch.uint8)[pad:pad + nbytes.value]
        stream = torch.cuda.current_stream()
        for name, tid, layer in self._tensors(weights):
            off, n = self.tensor_offset(layer, tid)
            arr = weights[name] if layer < 0 else weights["layers"][layer][name]
            arr = np.ascontiguousarray(arr, dtype=np.uint16).reshape(-1)
            if arr.size != n:
                raise ValueError(f"layer {layer} {name}: {arr.size} elements, layout expects {n}")
            src = torch.from_numpy(arr.view(np.int16)).to(device)
            _check("hgd_model_load_tensor", _lib.hgd_model_load_tensor(
                C.byref(self.cfg), self.arena_u8.data_ptr(), nbytes.value, layer, tid, src.data_ptr(),
                stream.cuda_stream))
            stream.synchronize()
        self.m = _Model()
        _check("hgd_model_init", _lib.hgd_model_init(C.byref(self.m), C.byref(self.cfg),
                                                     self.arena_u8.data_ptr(), nbytes.value))
        self.tc_arena = None
        if tc:
            self._load_tc(weights, device)

    def _load_tc(self, weights, device):
        torch = _torch()
        nb = C.c_size_t()
        _check("hgd_model_tc_bytes", _lib.hgd_model_tc_bytes(C.byref(self.cfg), C.byref(nb)))
        self.tc_arena = torch.zeros(nb.value + 256, dtype=torch.uint8, device=device)
        pad = (-self.tc_arena.data_ptr()) % 256
        base = self.tc_arena.data_ptr() + pad
        stream = torch.cuda.current_stream()
        items = [(-1, W_LM_HEAD if self.cfg_dict.get("untied_head") else W_EMBED,
                  weights["lm_head"] if self.cfg_dict.get("untied_head") else weights["embed"])]
        for l, lw in enumerate(weights["layers"]):
            for name, tid in (("w_in", W_IN), ("w_out", W_OUT), ("w_gate", W_GATE), ("w_up", W_UP),
                              ("w_down", W_DOWN)):
                items.append((l, tid, lw[name]))
        for layer, tid, arr in items:
            src = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.uint16).view(np.int16)).to(device)
            _check("hgd_model_tc_load", _lib.hgd_model_tc_load(C.byref(self.cfg), base, nb.value, layer, tid,
                                                                src.data_ptr(), stream.cuda_stream))
            stream.synchronize()
        _check("hgd_model_attach_tc", _lib.hgd_model_attach_tc(C.byref(self.m), base, nb.value))

    def _tensors(self, weights):
        yield "embed", W_EMBED, -1
        yield "final_norm", W_FINAL_NORM, -1
        if self.cfg_dict.get("untied_head"):
            yield "lm_head", W_LM_HEAD, -1
        for l, lw in enumerate(weights["layers"]):
            for name in lw:
                yield name, LAYER_TENSORS[name], l

    def tensor_offset(self, layer: int, tid: int):
        off, n = C.c_size_t(), C.c_size_t()
        _check("hgd_model_tensor", _lib.hgd_model_tensor(C.byref(self.cfg), layer, tid, C.byref(off),
                                                         C.byref(n)))
        return off.value, n.value

    def launches(self, B: int, T: int) -> int:
        return _lib.hgd_decode_layer_stack_launches(C.byref(self.m), B, T)


class State:
    """Per-stream decode state (GDN S, conv tails, KV cache, positions) plus the
    call scratch, in one device arena laid out by libhgd."""

    def __init__(self, model: Model, B: int, Tmax: int, Lmax: int, init: dict | None = None,
                 device="cuda"):
        torch = _torch()
        self.model, self.B, self.Tmax, self.Lmax = model, B, Tmax, Lmax
        nbytes = C.c_size_t()
        _check("hgd_state_arena_bytes", _lib.hgd_state_arena_bytes(C.byref(model.cfg), B, Tmax, Lmax,
                                                                   C.byref(nbytes)))
        self.arena = torch.zeros(nbytes.value // 4 + 64, dtype=torch.int32, device=device)
        pad = (-self.arena.data_ptr()) % 256
        self.arena_u8 = self.arena.view(torch.uint8)[pad:pad + nbytes.value]
        self.st = _State()
        _check("hgd_state_init", _lib.hgd_state_init(C.byref(self.st), C.byref(model.m), B, Tmax, Lmax,
                                                     self.arena_u8.data_ptr(), nbytes.value))
        cfg = model.cfg_dict
        Hk, H = gdn_heads(cfg)
        dk, dv, kc = cfg["gdn_dk"], cfg["gdn_dv"], cfg["conv_k"]
        nkv, hd = cfg["attn_kv_heads"], cfg["attn_head_dim"]
        n_attn = sum(1 for l in range(cfg["n_layers"]) if l % cfg["attn_every"] == cfg["attn_every"] - 1)
        n_gdn = cfg["n_layers"] - n_attn
        Cc = 2 * Hk * dk + H * dv
        self.S = self._view(S_GDN, torch.float32, (n_gdn, B, H, dv, dk))
        self.conv = self._view(S_CONV, torch.float32, (n_gdn, B, kc - 1, Cc))
        self.kv = self._view(S_KV, torch.bfloat16, (n_attn, 2, B, nkv, Lmax, hd))
        self.pos = self._view(S_POS, torch.int32, (B,))
        self.resid = self._view(S_RESID, torch.bfloat16, (B * Tmax, cfg["hidden"]))
        if init is not None:
            self.load(init)

    def _view(self, tid, dtype, shape):
        torch = _torch()
        off, n = C.c_size_t(), C.c_size_t()
        _check("hgd_state_tensor", _lib.hgd_state_tensor(C.byref(self.model.cfg), self.B, self.Tmax,
                                                         self.Lmax, tid, C.byref(off), C.byref(n)))
        es = torch.empty((), dtype=dtype).element_size()
        assert int(np.prod(shape)) == n.value
        return self.arena_u8[off.value:off.value + n.value * es].view(dtype).view(shape)

    def load(self, init: dict) -> None:
        """Copy host arrays (from hgd_synth.stack_state) into the state tensors."""
        torch = _torch()
        self.S.copy_(torch.from_numpy(np.ascontiguousarray(init["S"], np.float32)))
        self.conv.copy_(torch.from_numpy(np.ascontiguousarray(init["tail"], np.float32)))
        kv = np.ascontiguousarray(init["kv"], np.uint16)
        if kv.shape[-2] != self.Lmax:
            full = np.zeros(kv.shape[:-2] + (self.Lmax, kv.shape[-1]), np.uint16)
            n = min(self.Lmax, kv.shape[-2])
            full[..., :n, :] = kv[..., :n, :]
            kv = full
        self.kv.view(torch.int16).copy_(torch.from_numpy(kv.view(np.int16)))
        self.pos.copy_(torch.from_numpy(np.ascontiguousarray(init["pos"], np.int32)))

    def snapshot(self) -> dict:
        return {"S": self.S.clone(), "conv": self.conv.clone(), "kv": self.kv.clone(), "pos": self.pos.clone()}

    def restore(self, snap: dict) -> None:
        self.S.copy_(snap["S"]); self.conv.copy_(snap["conv"]); self.kv.copy_(snap["kv"])
        self.pos.copy_(snap["pos"])


def decode_layer_stack(model: Model, state: State, tokens, T: int, logits=None, argmax=None, S_rec=None,
                       tail_rec=None, status=None, stream=None):
    """One decode call over T rows of each stream.  tokens [B,T] int32 (device).
    Returns argmax [B*T] int32 (device)."""
    torch = _torch()
    _need(tokens, torch.int32, "tokens")
    if argmax is None:
        argmax = torch.empty((state.B * T,), dtype=torch.int32, device=tokens.device)
    _check("hgd_decode_layer_stack", _lib.hgd_decode_layer_stack(
        C.byref(model.m), C.byref(state.st), _ptr(tokens), T, _ptr(logits), _ptr(argmax), _ptr(S_rec),
        _ptr(tail_rec), _ptr(status), _stream(stream)))
    return argmax


def decode_layer_stack_tc(model: Model, state: State, tokens, T: int, logits=None, argmax=None, S_rec=None,
                          tail_rec=None, status=None, stream=None):
    """One decode call through the tensor-core chain (the model must be built with
    tc=True).  Returns argmax [B*T] int32 (device)."""
    torch = _torch()
    _need(tokens, torch.int32, "tokens")
    if argmax is None:
        argmax = torch.empty((state.B * T,), dtype=torch.int32, device=tokens.device)
    _check("hgd_decode_layer_stack_tc", _lib.hgd_decode_layer_stack_tc(
        C.byref(model.m), C.byref(state.st), _ptr(tokens), T, _ptr(logits), _ptr(argmax), _ptr(S_rec),
        _ptr(tail_rec), _ptr(status), _stream(stream)))
    return argmax


def decode_layer_stack_range(model: Model, state: State, tokens, T: int, layer_begin: int, layer_end: int,
                             run_head: bool, logits=None, argmax=None, S_rec=None, tail_rec=None, status=None,
                             stream=None):
    """Layers [layer_begin, layer_end) (and the head if run_head) of one decode call;
    the residual rows live in state.resid between ranges."""
    _check("hgd_decode_layer_stack_range", _lib.hgd_decode_layer_stack_range(
        C.byref(model.m), C.byref(state.st), _ptr(tokens), T, layer_begin, layer_end, int(run_head),
        _ptr(logits), _ptr(argmax), _ptr(S_rec), _ptr(tail_rec), _ptr(status), _stream(stream)))
    return argmax


class VerifyLog:
    """Device memory for the logs of one verify call of T rows per stream."""

    def __init__(self, model: Model, B: int, T: int, device="cuda"):
        torch = _torch()
        n = C.c_size_t()
        _check("hgd_verify_log_bytes", _lib.hgd_verify_log_bytes(C.byref(model.cfg), B, T, C.byref(n)))
        self.B, self.T, self.nbytes = B, T, n.value
        self.buf = torch.empty(n.value + 256, dtype=torch.uint8, device=device)
        pad = (-self.buf.data_ptr()) % 256
        self.ptr = self.buf.data_ptr() + pad


def decode_layer_stack_verify(model: Model, state: State, tokens, T: int, log: VerifyLog, logits=None,
                              argmax=None, status=None, stream=None):
    """A verify window: logits/argmax as decode_layer_stack; the state is left as it
    was and the rows are logged in `log`.  Returns argmax [B*T]."""
    torch = _torch()
    _need(tokens, torch.int32, "tokens")
    if argmax is None:
        argmax = torch.empty((state.B * T,), dtype=torch.int32, device=tokens.device)
    _check("hgd_decode_layer_stack_verify", _lib.hgd_decode_layer_stack_verify(
        C.byref(model.m), C.byref(state.st), _ptr(tokens), T, _ptr(logits), _ptr(argmax), log.ptr, log.nbytes,
        _ptr(status), _stream(stream)))
    return argmax


def decode_layer_stack_keep(model: Model, state: State, T: int, log: VerifyLog, keep, status=None, stream=None):
    """Stream b keeps the first keep[b] rows of the verify call logged in `log`."""
    torch = _torch()
    _need(keep, torch.int32, "keep")
    _check("hgd_decode_layer_stack_keep", _lib.hgd_decode_layer_stack_keep(
        C.byref(model.m), C.byref(state.st), T, log.ptr, log.nbytes, _ptr(keep), _ptr(status), _stream(stream)))


def check_stack_timeout(model: Model, state: State, tokens, T: int, skip_cta: int, skip_phase: int,
                        wait_ms: int, status, report=None, argmax=None, stream=None):
    """One persistent decode call in which CTA skip_cta leaves out its arrival at
    phase skip_phase and phase waits are limited to wait_ms: HGD_ERR_TIMEOUT lands
    in status, what ran out first in report (uint32 [4] device, or None)."""
    torch = _torch()
    if argmax is None:
        argmax = torch.empty((state.B * T,), dtype=torch.int32, device=tokens.device)
    _check("hgd_check_stack_timeout", _lib.hgd_check_stack_timeout(
        C.byref(model.m), C.byref(state.st), _ptr(tokens), T, _ptr(argmax), skip_cta, skip_phase, wait_ms,
        _ptr(status), _ptr(report), _stream(stream)))


def check_not_coresident(model: Model, state: State, T: int) -> int:
    """The status the persistent launch's co-residency check returns when the
    device can hold none of its CTAs (HGD_ERR_NOT_CORESIDENT); nothing is run."""
    return _lib.hgd_check_not_coresident(C.byref(model.m), C.byref(state.st), T)


class DecodeGraph:
    """A greedy decode step (T = 1) captured as a CUDA graph and replayed on
    `stream`: one hgd_decode_layer_stack call, which is a single cooperative
    launch when the call fits it.  `tokens` [B,1] is read at the start of a step
    and `argmax` [B] written at its end, so tokens = argmax.view(B, 1) feeds each
    step's argmax to the next on the device.  With split=True the step is
    captured as two graphs (all layers; then the head) through the layer-range
    entry point instead.  Capturing runs the step once eagerly first (to load the
    kernels) on a copy of the state, which is then restored."""

    def __init__(self, model: Model, state: State, tokens, argmax, status=None, stream=None, split=False):
        torch = _torch()
        self.model, self.state, self.tokens, self.argmax, self.status = model, state, tokens, argmax, status
        self.stream = stream or torch.cuda.Stream()
        self.split = split
        L = model.cfg_dict["n_layers"]
        snap = state.snapshot()
        tok0 = tokens.clone()
        with torch.cuda.stream(self.stream):
            if split:
                decode_layer_stack_range(model, state, tokens, 1, 0, L, False, status=status, stream=self.stream)
                decode_layer_stack_range(model, state, None, 1, L, L, True, argmax=argmax, status=status,
                                         stream=self.stream)
            else:
                decode_layer_stack(model, state, tokens, 1, argmax=argmax, status=status, stream=self.stream)
        self.stream.synchronize()
        state.restore(snap)
        tokens.copy_(tok0)
        torch.cuda.synchronize()
        self.g_layers = torch.cuda.CUDAGraph()
        self.g_head = torch.cuda.CUDAGraph() if split else None
        if split:
            with torch.cuda.graph(self.g_layers, stream=self.stream):
                decode_layer_stack_range(model, state, tokens, 1, 0, L, False, status=status)
            with torch.cuda.graph(self.g_head, stream=self.stream):
                decode_layer_stack_range(model, state, None, 1, L, L, True, argmax=argmax, status=status)
        else:
            with torch.cuda.graph(self.g_layers, stream=self.stream):
                decode_layer_stack(model, state, tokens, 1, argmax=argmax, status=status)
        torch.cuda.synchronize()

    def replay_layers(self):
        self.g_layers.replay()

    def replay_head(self):
        if self.g_head is not None:
            self.g_head.replay()

    def replay(self):
        self.g_layers.replay()
        if self.g_head is not None:
            self.g_head.replay()

    def step_host(self, h_tok, h_out):
        """One step from a pinned host token tensor to a pinned host argmax tensor."""
        torch = _torch()
        with torch.cuda.stream(self.stream):
            self.tokens.copy_(h_tok, non_blocking=True)
            self.replay()
            h_out.copy_(self.argmax, non_blocking=True)
        self.stream.synchronize()

    def close(self):
        self.g_layers.reset()
        if self.g_head is not None:
            self.g_head.reset()
