"""Python access to the CPU oracle (ctypes over libhgd_oracle*.so).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product package never imports this.
All arrays are host numpy arrays; bf16 tensors are carried as uint16 bit
patterns.  `real` arrays are float64 for the default build (`Oracle()`) and
float32 for `Oracle(fp32=True)`.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
MAX_LAYERS = 64

_p = C.c_void_p


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("hidden", C.c_int32), ("vocab", C.c_int32),
                ("gdn_heads", C.c_int32), ("gdn_dk", C.c_int32), ("gdn_dv", C.c_int32),
                ("conv_k", C.c_int32), ("attn_q_heads", C.c_int32),
                ("attn_kv_heads", C.c_int32), ("attn_head_dim", C.c_int32),
                ("mlp_inter", C.c_int32), ("attn_every", C.c_int32),
                ("norm_eps", C.c_double), ("rope_base", C.c_double), ("gdn_v_heads", C.c_int32)]


class Layer(C.Structure):
    _fields_ = [(n, _p) for n in ("in_norm", "w_in", "conv_w", "A_log", "dt_bias", "gnorm_w",
                                  "w_out", "post_norm", "w_gate", "w_up", "w_down")]


class Model(C.Structure):
    _fields_ = [("cfg", Config), ("embed", _p), ("final_norm", _p),
                ("layers", Layer * MAX_LAYERS), ("lm_head", _p)]


class State(C.Structure):
    _fields_ = [("S", _p), ("tail", _p), ("kv", _p), ("pos", _p), ("B", C.c_int32),
                ("Lmax", C.c_int32)]


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    if not a.flags["C_CONTIGUOUS"]:
        raise ValueError("oracle arrays must be C-contiguous")
    return a.ctypes.data_as(C.c_void_p)


def build_lib() -> None:
    from . import build as _b  # noqa: WPS433
    _b.build()


class Oracle:
    """One loaded oracle library (double by default, float with fp32=True)."""

    def __init__(self, fp32: bool = False, all_cores: bool = False):
        # all_cores: the double build whose GEMV and dense state product run over
        # every host core (OpenMP); same results as the default build
        name = "libhgd_oracle_f32.so" if fp32 else ("libhgd_oracle_omp.so" if all_cores else "libhgd_oracle.so")
        path = os.path.join(_HERE, name)
        if not os.path.exists(path):
            build_lib()
        self.lib = C.CDLL(path)
        nb = self.lib.hgdo_real_bytes()
        self.real = np.float32 if nb == 4 else np.float64
        assert (nb == 4) == fp32
        L = self.lib
        L.hgdo_bf16_value.restype = C.c_double if nb == 8 else C.c_float
        L.hgdo_bf16_value.argtypes = [C.c_uint16]
        L.hgdo_round_bf16.restype = C.c_uint16
        L.hgdo_round_bf16.argtypes = [C.c_double if nb == 8 else C.c_float]
        L.hgdo_round_bf16_array.argtypes = [_p, _p, C.c_int64]
        L.hgdo_gemv.argtypes = [_p, _p, _p, C.c_int, C.c_int, C.c_int]
        L.hgdo_swiglu.argtypes = [_p, _p, _p, _p, C.c_int, C.c_int, C.c_int]
        L.hgdo_conv1d_tail_update.argtypes = [_p, _p, _p, _p, _p] + [C.c_int] * 5
        L.hgdo_gdn_step.argtypes = [_p, _p, _p, C.c_int64, _p, _p, _p, _p, _p] + [C.c_int] * 6
        L.hgdo_gdn_step_grouped.argtypes = [_p, _p, _p, C.c_int64, _p, _p, _p, _p, _p] + [C.c_int] * 7
        L.hgdo_gdn_window_log.argtypes = [_p, _p, _p, C.c_int64, _p, _p, _p, _p, _p, _p, _p] + [C.c_int] * 6
        L.hgdo_gdn_keep.restype = C.c_int
        L.hgdo_gdn_keep.argtypes = [_p, _p, _p, _p, _p] + [C.c_int] * 5
        L.hgdo_conv1d_keep.restype = C.c_int
        L.hgdo_conv1d_keep.argtypes = [_p, _p, _p] + [C.c_int] * 4
        L.hgdo_softplus.restype = C.c_double if nb == 8 else C.c_float
        L.hgdo_softplus.argtypes = [C.c_double if nb == 8 else C.c_float]
        L.hgdo_gdn_gates.argtypes = [_p, _p, _p, _p, C.c_int]
        L.hgdo_rmsnorm.argtypes = [_p, _p, _p, C.c_int, C.c_int, C.c_double]
        L.hgdo_gated_rmsnorm.argtypes = [_p, _p, _p, _p, C.c_int, C.c_int, C.c_int, C.c_double]
        L.hgdo_rope.argtypes = [_p, C.c_int, C.c_int, C.c_double]
        L.hgdo_attention_row.argtypes = [_p, _p, _p, _p] + [C.c_int] * 5 + [_p]
        L.hgdo_decode_stack.restype = C.c_int
        L.hgdo_decode_stack.argtypes = [C.POINTER(Model), C.POINTER(State), _p, C.c_int,
                                        _p, _p, _p, _p, _p]

    # -- helpers -----------------------------------------------------------
    def _r(self, a) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=self.real)

    @staticmethod
    def _u16(a) -> np.ndarray:
        a = np.ascontiguousarray(a)
        if a.dtype != np.uint16:
            raise TypeError("bf16 arrays are passed as uint16 bit patterns")
        return a

    # -- elementwise -------------------------------------------------------
    def round_bf16(self, v) -> np.ndarray:
        v = self._r(v)
        out = np.empty(v.shape, np.uint16)
        self.lib.hgdo_round_bf16_array(_ptr(v), _ptr(out), v.size)
        return out

    def bf16_value(self, h) -> np.ndarray:
        h = self._u16(h)
        return (h.astype(np.uint32) << 16).view(np.float32).astype(self.real)

    # -- ops ---------------------------------------------------------------
    def gemv(self, W, x) -> np.ndarray:
        W, x = self._u16(W), self._u16(x)
        N, K = W.shape
        M = x.shape[0]
        assert x.shape == (M, K)
        y = np.empty((M, N), self.real)
        self.lib.hgdo_gemv(_ptr(W), _ptr(x), _ptr(y), M, N, K)
        return y

    def swiglu(self, Wg, Wu, x) -> np.ndarray:
        Wg, Wu, x = self._u16(Wg), self._u16(Wu), self._u16(x)
        I, K = Wg.shape
        M = x.shape[0]
        h = np.empty((M, I), np.uint16)
        self.lib.hgdo_swiglu(_ptr(Wg), _ptr(Wu), _ptr(x), _ptr(h), M, I, K)
        return h

    def conv1d_tail_update(self, x, tail, w, apply_silu=True, record=False):
        """x [B,T,C] real; tail [B,kc-1,C] real (updated in place); w [C,kc] bf16."""
        assert tail.dtype == self.real and tail.flags["C_CONTIGUOUS"]
        x = self._r(x)
        w = self._u16(w)
        B, T, C_ = x.shape
        kc = w.shape[1]
        y = np.empty_like(x)
        rec = np.empty((B, T, kc - 1, C_), self.real) if record else None
        self.lib.hgdo_conv1d_tail_update(_ptr(x), _ptr(tail), _ptr(w), _ptr(y), _ptr(rec),
                                         B, T, C_, kc, int(apply_silu))
        return (y, rec) if record else y

    def gdn_step(self, q, k, v, g, b, S, l2norm=True, record=False, row_stride=None):
        """q,k [B,T,H,dk], v [B,T,H,dv] (or flat rows with row_stride), g,b [B,T,H];
        S [B,H,dv,dk] updated in place.  Returns o [B,T,H,dv] (and S_rec)."""
        assert S.dtype == self.real and S.flags["C_CONTIGUOUS"]
        B, H, dv, dk = S.shape
        g, b = self._r(g), self._r(b)
        T = g.shape[1]
        if row_stride is None:
            q, k, v = self._r(q), self._r(k), self._r(v)
            assert q.shape == (B, T, H, dk) and v.shape == (B, T, H, dv)
            assert H * dk == H * dv, "separate q/k/v arrays share one row stride"
            row_stride = H * dk
        o = np.empty((B, T, H, dv), self.real)
        rec = np.empty((B, T, H, dv, dk), self.real) if record else None
        self.lib.hgdo_gdn_step(_ptr(q), _ptr(k), _ptr(v), row_stride, _ptr(g), _ptr(b),
                               _ptr(S), _ptr(o), _ptr(rec), B, T, H, dk, dv, int(l2norm))
        return (o, rec) if record else o

    def gdn_window_log(self, q, k, v, g, b, S, l2norm=True):
        """As gdn_step (separate q,k,v [B,T,H,d]) but S is left unchanged; returns
        (o [B,T,H,dv], log_alpha [B,T,H], log_delta [B,T,H,dv], log_k [B,T,H,dk])."""
        assert S.dtype == self.real and S.flags["C_CONTIGUOUS"]
        B, H, dv, dk = S.shape
        g, b = self._r(g), self._r(b)
        T = g.shape[1]
        q, k, v = self._r(q), self._r(k), self._r(v)
        assert q.shape == (B, T, H, dk) and k.shape == (B, T, H, dk) and v.shape == (B, T, H, dv) and dk == dv
        o = np.empty((B, T, H, dv), self.real)
        la = np.empty((B, T, H), self.real)
        ld = np.empty((B, T, H, dv), self.real)
        lk = np.empty((B, T, H, dk), self.real)
        self.lib.hgdo_gdn_window_log(_ptr(q), _ptr(k), _ptr(v), H * dk, _ptr(g), _ptr(b), _ptr(S), _ptr(o),
                                     _ptr(la), _ptr(ld), _ptr(lk), B, T, H, dk, dv, int(l2norm))
        return o, la, ld, lk

    def gdn_keep(self, S, log_alpha, log_delta, log_k, keep):
        """S [B,H,dv,dk] updated in place by the first keep[b] logged rows of stream b."""
        assert S.dtype == self.real and S.flags["C_CONTIGUOUS"]
        B, H, dv, dk = S.shape
        T = log_alpha.shape[1]
        keep = np.ascontiguousarray(keep, np.int32)
        la, ld, lk = self._r(log_alpha), self._r(log_delta), self._r(log_k)
        rc = self.lib.hgdo_gdn_keep(_ptr(S), _ptr(la), _ptr(ld), _ptr(lk), _ptr(keep), B, T, H, dk, dv)
        if rc:
            raise ValueError("oracle gdn_keep: a keep count outside [0, T]")

    def conv1d_keep(self, tail, x, keep):
        """tail [B,kc-1,C] (in place) after the first keep[b] rows of x [B,T,C]."""
        assert tail.dtype == self.real and tail.flags["C_CONTIGUOUS"]
        B, nt, C_ = tail.shape
        x = self._r(x)
        keep = np.ascontiguousarray(keep, np.int32)
        rc = self.lib.hgdo_conv1d_keep(_ptr(tail), _ptr(x), _ptr(keep), B, x.shape[1], C_, nt + 1)
        if rc:
            raise ValueError("oracle conv1d_keep: a keep count outside [0, T]")

    def gdn_step_grouped(self, q, k, v, g, b, S, l2norm=True):
        """q,k [B,T,Hk,dk] (key heads), v [B,T,H,dv], g,b [B,T,H]; S [B,H,dv,dk] in place;
        value head h reads key head h // (H // Hk).  Returns o [B,T,H,dv]."""
        assert S.dtype == self.real and S.flags["C_CONTIGUOUS"]
        B, H, dv, dk = S.shape
        g, b = self._r(g), self._r(b)
        T = g.shape[1]
        Hk = q.shape[2]
        # one packed row per (b, t): q | k | v, so that one stride serves all three
        rows = np.concatenate([self._r(q).reshape(B * T, -1), self._r(k).reshape(B * T, -1),
                               self._r(v).reshape(B * T, -1)], axis=1)
        rows = np.ascontiguousarray(rows)
        stride = rows.shape[1]
        base = rows.reshape(-1)
        o = np.empty((B, T, H, dv), self.real)
        self.lib.hgdo_gdn_step_grouped(_ptr(base), base[Hk * dk:].ctypes.data_as(C.c_void_p),
                                       base[2 * Hk * dk:].ctypes.data_as(C.c_void_p), stride, _ptr(g), _ptr(b),
                                       _ptr(S), _ptr(o), None, B, T, Hk, H, dk, dv, int(l2norm))
        return o

    def gdn_step_packed(self, qkv, g, b, S, l2norm=True, record=False):
        """qkv [B,T,2*H*dk + H*dv] real with channels q|k|v."""
        qkv = self._r(qkv)
        B, H, dv, dk = S.shape
        stride = qkv.shape[-1]
        base = qkv.reshape(-1)
        q = base
        k = base[H * dk:]
        v = base[2 * H * dk:]
        assert S.dtype == self.real and S.flags["C_CONTIGUOUS"]
        g, b = self._r(g), self._r(b)
        T = g.shape[1]
        o = np.empty((B, T, H, dv), self.real)
        rec = np.empty((B, T, H, dv, dk), self.real) if record else None
        self.lib.hgdo_gdn_step(_ptr(q), k.ctypes.data_as(C.c_void_p), v.ctypes.data_as(C.c_void_p),
                               stride, _ptr(g), _ptr(b), _ptr(S), _ptr(o), _ptr(rec),
                               B, T, H, dk, dv, int(l2norm))
        return (o, rec) if record else o

    def softplus(self, t) -> float:
        return float(self.lib.hgdo_softplus(float(t)))

    def gdn_gates(self, a, A_log, dt_bias) -> np.ndarray:
        """a [H] real; A_log, dt_bias [H] bf16.  Returns g [H] (log-decay)."""
        a = self._r(a)
        A_log, dt_bias = self._u16(A_log), self._u16(dt_bias)
        H = a.shape[0]
        assert A_log.shape == (H,) and dt_bias.shape == (H,)
        g = np.empty(H, self.real)
        self.lib.hgdo_gdn_gates(_ptr(a), _ptr(A_log), _ptr(dt_bias), _ptr(g), H)
        return g

    def rmsnorm(self, x, w, eps=1e-6) -> np.ndarray:
        x, w = self._u16(x), self._u16(w)
        M, D = x.shape
        y = np.empty_like(x)
        self.lib.hgdo_rmsnorm(_ptr(x), _ptr(w), _ptr(y), M, D, eps)
        return y

    def gated_rmsnorm(self, o, z, w, nh, eps=1e-6) -> np.ndarray:
        o = self._r(o)
        z, w = self._u16(z), self._u16(w)
        M = o.shape[0]
        d = w.shape[0]
        u = np.empty((M, nh * d), np.uint16)
        self.lib.hgdo_gated_rmsnorm(_ptr(o), _ptr(z), _ptr(w), _ptr(u), M, nh, d, eps)
        return u

    def rope(self, x, pos, base=10000.0) -> np.ndarray:
        x = self._r(x).copy()
        self.lib.hgdo_rope(_ptr(x), x.shape[-1], int(pos), float(base))
        return x

    def attention_row(self, q, gate, Kc, Vc, nkeys) -> np.ndarray:
        """q, gate [nq,hd] real; Kc, Vc [nkv,Lmax,hd] bf16."""
        q, gate = self._r(q), self._r(gate)
        Kc, Vc = self._u16(Kc), self._u16(Vc)
        nq, hd = q.shape
        nkv, Lmax, _ = Kc.shape
        out = np.empty((nq, hd), np.uint16)
        self.lib.hgdo_attention_row(_ptr(q), _ptr(gate), _ptr(Kc), _ptr(Vc), int(nkeys), Lmax,
                                    nq, nkv, hd, _ptr(out))
        return out

    # -- stack -------------------------------------------------------------
    def make_model(self, cfg: dict, weights: dict) -> Model:
        """cfg: dict of Config fields; weights: dict from hgd_synth.stack_weights()."""
        m = Model()
        for k, v in cfg.items():
            if hasattr(m.cfg, k):
                setattr(m.cfg, k, v)
        keep = []
        def P(a):
            a = self._u16(a)
            keep.append(a)
            return _ptr(a)
        m.embed = P(weights["embed"])
        m.final_norm = P(weights["final_norm"])
        m.lm_head = P(weights["lm_head"]) if weights.get("lm_head") is not None else None
        for l, lw in enumerate(weights["layers"]):
            for name, arr in lw.items():
                setattr(m.layers[l], name, P(arr))
        m._keep = keep  # keep the arrays alive with the struct
        return m

    def decode_stack(self, model: Model, state: dict, tokens, logits=True, record=False):
        """state: dict with S, tail (real, in place), kv (uint16, in place), pos (int32, in place).
        tokens [B,T] int32.  Returns dict(argmax, logits?, S_rec?, tail_rec?, status)."""
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        B, T = tokens.shape
        S, tail, kv, pos = state["S"], state["tail"], state["kv"], state["pos"]
        for a, dt in ((S, self.real), (tail, self.real), (kv, np.uint16), (pos, np.int32)):
            assert a.dtype == dt and a.flags["C_CONTIGUOUS"]
        st = State()
        st.S, st.tail, st.kv, st.pos = _ptr(S), _ptr(tail), _ptr(kv), _ptr(pos)
        st.B = B
        st.Lmax = kv.shape[-2]
        cfg = model.cfg
        V = cfg.vocab
        out = {"argmax": np.empty((B, T), np.int32)}
        lg = np.empty((B, T, V), self.real) if logits else None
        srec = trec = xrec = None
        if record:
            n_gdn = S.shape[0]
            srec = np.empty((n_gdn, B, T) + S.shape[2:], self.real)
            trec = np.empty((n_gdn, B, T) + tail.shape[2:], self.real)
            xrec = np.empty((cfg.n_layers, B, T, cfg.hidden), np.uint16)
        rc = self.lib.hgdo_decode_stack(C.byref(model), C.byref(st), _ptr(tokens), T, _ptr(lg),
                                        _ptr(out["argmax"]), _ptr(srec), _ptr(trec), _ptr(xrec))
        if rc == 2:
            raise ValueError("oracle decode_stack rejected its arguments")
        out["status"] = rc
        if logits:
            out["logits"] = lg
        if record:
            out["S_rec"], out["tail_rec"], out["x_rec"] = srec, trec, xrec
        return out
