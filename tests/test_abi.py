"""Host-side checks of the C ABI: the library loads, exports every function the
header declares, and validates arguments without touching a GPU (every rejected
call returns before any CUDA call)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hgd():
    import __graft_entry__ as g
    g.build()
    import hybrid_gated_delta_b200 as m
    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hgd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hgd_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function(hgd):
    names = declared_functions()
    assert len(names) >= 14
    lib = C.CDLL(hgd.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(hgd.EXPORTED)


def test_exports_nothing_else(hgd):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", hgd.LIB_PATH], capture_output=True, text=True).stdout
    syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {s for s in syms if s.startswith("hgd_")}
    assert ours == set(declared_functions())


def test_status_strings(hgd):
    assert hgd.status_string(0) == "ok"
    assert "unsupported shape" == hgd.status_string(2)
    assert hgd.status_string(999) == "unknown status"
    assert hgd.version() >= 100


def test_validation_before_any_cuda_call(hgd):
    L = hgd._lib
    # NULL buffers, bad sizes, misaligned pointers: rejected on the host
    assert L.hgd_gemv_bf16(None, None, None, 1, 1, 1, 32, None, 0, None) == 1
    assert L.hgd_gemv_bf16(16, 16, 16, 1, 1, 1, 48, None, 0, None) == 2      # K % 32
    assert L.hgd_gemv_bf16(16, 16, 16, 1, 1, 1, 0, None, 0, None) == 1
    assert L.hgd_gemv_bf16(18, 16, 16, 1, 1, 1, 64, None, 0, None) == 3      # misaligned W
    assert L.hgd_gemv_bf16(16, 16, 16, 1, 1, 1, 64, 24, 64, None) == 3       # misaligned workspace
    assert L.hgd_gemv_swiglu_bf16(16, 16, 16, 16, 1, 1, 33, None, 0, None) == 2
    n = C.c_size_t()
    assert L.hgd_gemv_workspace_bytes(1, 1024, 2048, 0, C.byref(n)) == 0 and n.value > 0
    assert L.hgd_gemv_workspace_bytes(1, 248320, 1024, 0, C.byref(n)) == 0 and n.value == 0
    assert L.hgd_conv1d_tail_update(16, 16, 16, 16, None, 1, 1, 1, 9, 1, None) == 2
    assert L.hgd_conv1d_tail_update(16, 16, 16, 20, None, 1, 1, 1, 4, 1, None) == 3
    assert L.hgd_gdn_decode_step(16, 16, 16, 512, 16, 16, 16, 16, None, None, 1, 1, 4, 96, 64, 1, None) == 2
    assert L.hgd_gdn_decode_step(16, 16, 16, 512, 16, 16, 16, 16, None, None, 1, 1, 4, 128, 24, 1, None) == 2
    assert L.hgd_gdn_decode_step(16, 16, 16, 100, 16, 16, 16, 16, None, None, 1, 1, 4, 64, 64, 1, None) == 1
    # tensor-core GEMM: shapes, alignment and workspace size checked on the host
    assert L.hgd_gemm_tc_weight_bytes(128, 96, C.byref(n)) == 2                    # K % 64
    assert L.hgd_gemm_tc_weight_bytes(0, 64, C.byref(n)) == 1
    assert L.hgd_gemm_tc_weight_bytes(129, 128, C.byref(n)) == 0 and n.value == 256 * 128 * 2
    assert L.hgd_gemm_tc_workspace_bytes(257, 128, 128, C.byref(n)) == 2           # M > 256
    assert L.hgd_gemm_tc_workspace_bytes(128, 8224, 1024, C.byref(n)) == 0 and n.value >= 128 * 1024 * 2
    assert L.hgd_gemm_tc_pack_weight(16, 16, 128, 96, None) == 2
    assert L.hgd_gemm_tc_pack_weight(18, 16, 128, 128, None) == 3
    assert L.hgd_gemm_tc_bf16(16, 16, 16, 1, 128, 96, 16, 1 << 20, None, None) == 2
    assert L.hgd_gemm_tc_bf16(16, 18, 16, 1, 128, 128, 16, 1 << 20, None, None) == 3   # misaligned x
    assert L.hgd_gemm_tc_bf16(16, 16, 16, 1, 128, 128, None, 1 << 20, None, None) == 1
    assert L.hgd_gemm_tc_bf16(16, 16, 16, 1, 128, 128, 16, 16, None, None) == 9        # workspace too small
    assert L.hgd_check_bounded_wait(None, None) == 1
    assert L.hgd_check_bounded_wait(20, None) == 3


def test_model_and_state_layout(hgd):
    import hgd_synth as syn
    cfg = hgd.make_config(syn.STACK_CFG)
    n = C.c_size_t()
    assert hgd._lib.hgd_model_arena_bytes(C.byref(cfg), C.byref(n)) == 0
    # every tensor fits, is 256-byte aligned and the tensors do not overlap
    spans = []
    w = syn.STACK_CFG
    for layer in range(-1, w["n_layers"]):
        tids = [hgd.W_EMBED, hgd.W_FINAL_NORM] if layer < 0 else range(hgd.W_LAYER_COUNT)
        gate_off = None
        for t in tids:
            off, num = C.c_size_t(), C.c_size_t()
            assert hgd._lib.hgd_model_tensor(C.byref(cfg), layer, t, C.byref(off), C.byref(num)) == 0
            if t == hgd.W_GATE:
                gate_off = off.value
            if t == hgd.W_UP:          # the up rows share the packed SwiGLU region of the gate rows
                assert off.value == gate_off
                continue
            if num.value:
                assert off.value % 256 == 0
                size = 2 * num.value * (2 if t == hgd.W_GATE else 1)
                spans.append((off.value, off.value + size))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= n.value
    total_params = sum((b - a) // 2 for a, b in spans)
    assert abs(total_params * 2 / 1e6 - 1504.8) < 1.0   # 1,504.8 MB of bf16 weights
    # embedding first: [V, D]
    off, num = C.c_size_t(), C.c_size_t()
    hgd._lib.hgd_model_tensor(C.byref(cfg), -1, hgd.W_EMBED, C.byref(off), C.byref(num))
    assert off.value == 0 and num.value == 248320 * 1024
    # attention layers have no conv weights
    hgd._lib.hgd_model_tensor(C.byref(cfg), 3, hgd.W_CONV, C.byref(off), C.byref(num))
    assert num.value == 0
    assert hgd._lib.hgd_model_tensor(C.byref(cfg), 24, 0, C.byref(off), C.byref(num)) == 1
    sb = C.c_size_t()
    assert hgd._lib.hgd_state_arena_bytes(C.byref(cfg), 1, 1, 640, C.byref(sb)) == 0
    assert hgd._lib.hgd_state_arena_bytes(C.byref(cfg), 64, 8, 640, C.byref(sb)) == 2
    for t, expect in ((hgd.S_GDN, 18 * 16 * 128 * 128), (hgd.S_CONV, 18 * 3 * 6144),
                      (hgd.S_KV, 6 * 2 * 2 * 640 * 256), (hgd.S_POS, 1)):
        assert hgd._lib.hgd_state_tensor(C.byref(cfg), 1, 1, 640, t, C.byref(off), C.byref(num)) == 0
        assert num.value == expect and off.value % 256 == 0


def test_model_init_rejects_unsupported(hgd):
    import hgd_synth as syn
    bad = dict(syn.STACK_CFG, conv_k=3)
    cfg = hgd.make_config(bad)
    m = hgd._Model()
    assert hgd._lib.hgd_model_init(C.byref(m), C.byref(cfg), 256, 1 << 40) == 2
    cfg = hgd.make_config(syn.STACK_CFG)
    assert hgd._lib.hgd_model_init(C.byref(m), C.byref(cfg), 256, 1024) == 9
    assert hgd._lib.hgd_model_init(C.byref(m), C.byref(cfg), 272, 1 << 40) == 3
    assert hgd._lib.hgd_model_init(C.byref(m), C.byref(cfg), 256, 1 << 40) == 0
    assert m.embed == 256


def test_tensor_core_split_depends_on_n_and_k_only(hgd):
    """The tensor-core GEMM splits K over the CTAs of one cluster by a fixed
    function of N and K (a split never depends on M or on the device): a power
    of two up to 8, the same at every M, one split once the row tiles alone fill
    the device (N = 248320); its workspace is the packed token rows only, and
    with splits its pipeline holds the NTp x 128 fp32 accumulator."""
    L = hgd._lib
    n = C.c_size_t()
    sp, st = C.c_int(), C.c_int()

    def ws(M, N, K):
        assert L.hgd_gemm_tc_workspace_bytes(M, N, K, C.byref(n)) == 0
        return n.value

    def plan(M, N, K):
        assert L.hgd_gemm_tc_plan(M, N, K, C.byref(sp), C.byref(st)) == 0
        return sp.value, st.value

    def ntp(M):
        return 16 if M <= 16 else (M + 15) // 16 * 16

    for N, K in ((1024, 3584), (1024, 2048), (8224, 1024), (7168, 1024), (300, 640), (128, 64)):
        splits = {plan(M, N, K)[0] for M in (1, 16, 33, 128, 256)}
        assert len(splits) == 1, (N, K, splits)
        s = splits.pop()
        assert s in (1, 2, 4, 8) and s <= max(1, K // 64)
        for M in (1, 16, 33, 128, 256):
            assert ws(M, N, K) == (ntp(M) * K * 2 + 255) // 256 * 256
            if s > 1:
                stages = plan(M, N, K)[1]
                assert stages * (128 * 64 * 2 + ntp(M) * 64 * 2) >= ntp(M) * 128 * 4
    assert plan(128, 1024, 2048)[0] == 8 and plan(128, 1024, 3584)[0] == 8 and plan(128, 8224, 1024)[0] == 2
    assert plan(128, 248320, 1024)[0] == 1
    assert L.hgd_gemm_tc_plan(0, 1024, 1024, C.byref(sp), C.byref(st)) != 0
    assert L.hgd_gemm_tc_plan(16, 1024, 100, C.byref(sp), C.byref(st)) != 0
