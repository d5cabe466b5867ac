#!/usr/bin/env python3
"""Decode throughput of the 24-layer hybrid gated-delta stack at batch 1.

Workload: hidden 1024, 24 layers (3 gated-delta-rule layers : 1 gated
full-attention layer, x6), GDN 16 heads d=128, conv k=4, attention 8 q / 2 kv
heads of 256, SwiGLU MLP 3584, vocab 248320 (tied head), random-init bf16
weights N(0, 0.02), KV context 512 prefilled, greedy decoding: one step = one
token through the whole stack (every weight byte streamed from HBM: 1.5 GB per
step, far larger than the 126 MB L2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  Under torchrun (N > 1) every rank decodes its own
stream (replicas, no collective on the data path); value = all ranks' tokens /
the slowest rank's device time.  `--impl reference` times the CPU oracle on this
host's cores instead (a bounded sample of the same workload).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s at B=1 (24-layer stack) and achieved HBM GB/s vs 8 TB/s"
UNIT = "tokens/s"
PREFILL = 512
WORKLOAD = ("24-layer hybrid stack (3 GDN : 1 gated attention), hidden 1024, vocab 248320, "
            "GDN 16x128, attn 8q/2kv x256, MLP 3584, batch 1, KV context 512, greedy decode")


def chain_launches(cfg: dict) -> int:
    """Kernels one B=1, T=1 step launches on the kernel-chain path: per GDN layer
    in-projection (with the conv tail), mixer, out-projection, SwiGLU, down; per
    attention layer the same with partials and merge as the mixer (RoPE and the
    KV append run in the in-projection); then the LM head and the argmax
    finalisation."""
    import hgd_synth as syn

    n_gdn, n_att = syn.layer_counts(cfg)
    return n_gdn * 5 + n_att * 6 + 2


def algorithmic_bytes(cfg: dict, L_keys: float) -> dict:
    """Bytes one decode token must move, by component (the HBM roofline numerator)."""
    D, V, H, dk, dv, kc = (cfg[k] for k in ("hidden", "vocab", "gdn_heads", "gdn_dk", "gdn_dv", "conv_k"))
    nq, nkv, hd, I = (cfg[k] for k in ("attn_q_heads", "attn_kv_heads", "attn_head_dim", "mlp_inter"))
    import hgd_synth as syn
    n_gdn, n_attn = syn.layer_counts(cfg)
    Cc = 2 * H * dk + H * dv
    w_gdn = (Cc + H * dv + 2 * H) * D + D * H * dv + 3 * I * D + 2 * D + Cc * kc + 2 * H + dv
    w_att = (2 * nq * hd + 2 * nkv * hd) * D + D * nq * hd + 3 * I * D + 2 * D
    weights = 2 * (n_gdn * w_gdn + n_attn * w_att + V * D + D)
    state = n_gdn * H * dv * dk * 4 * 2
    tails = n_gdn * (kc - 1) * Cc * 4 * 2
    kv = n_attn * 2 * nkv * hd * 2 * L_keys + n_attn * 2 * nkv * hd * 2  # read L keys, write 1
    head = 2 * V * D
    return {"weights": weights, "state": state, "tails": tails, "kv": kv, "head": head,
            "total": weights + state + tails + kv}


def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "_fallback": True}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ host cores --

def host_info() -> dict:
    """The host the oracle is timed on: online cores and the CPU model."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


class one_core:
    """Pin this process to one of its allowed cores while timing the oracle
    (single-threaded), and restore the previous set afterwards."""

    def __enter__(self):
        self.prev = None
        if hasattr(os, "sched_getaffinity"):
            self.prev = os.sched_getaffinity(0)
            os.sched_setaffinity(0, {min(self.prev)})
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            os.sched_setaffinity(0, self.prev)
        return False


# ---------------------------------------------------------------- reference --

def run_reference(args) -> None:
    """The CPU oracle on this host: greedy decode of the same workload, one token
    per step, single-threaded; a bounded number of steps."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import hgd_synth as syn
    from oracle import Oracle
    orc = Oracle()
    cfg = syn.STACK_CFG
    w = syn.stack_weights(cfg, seed=4)
    m = orc.make_model(cfg, w)
    init = syn.stack_state(cfg, 1, PREFILL + 64, prefill=PREFILL, seed=4)
    st = {"S": init["S"].astype(np.float64), "tail": init["tail"].astype(np.float64), "kv": init["kv"],
          "pos": init["pos"]}
    tok = syn.stack_tokens(cfg, 1, 1, seed=4)
    budget_s = float(os.environ.get("HGD_REF_BUDGET_S", "60"))
    warm = min(args.warmup, 1)
    with one_core():
        for _ in range(warm):
            tok = orc.decode_stack(m, st, tok, logits=False)["argmax"]
        t0 = time.perf_counter()
        n = 0
        while n < args.steps:
            tok = orc.decode_stack(m, st, tok, logits=False)["argmax"]
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
    v = n / dt
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
           "steps": n, "warmup": warm, "ms_per_step": 1000 * dt / n, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": WORKLOAD, "batch": 1, "kv_context": PREFILL},
           "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                            "sample": f"{n} greedy tokens of the full stack (of {args.steps} asked; "
                                      f"{budget_s:.0f} s budget), single-threaded C oracle, fp64, pinned "
                                      f"to one core", **host_info()},
           "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def cpu_baseline_sample(tokens: int = 4) -> dict:
    import hgd_synth as syn
    from oracle import Oracle
    orc = Oracle()
    cfg = syn.STACK_CFG
    m = orc.make_model(cfg, syn.stack_weights(cfg, seed=4))
    init = syn.stack_state(cfg, 1, PREFILL + 64, prefill=PREFILL, seed=4)
    st = {"S": init["S"].astype(np.float64), "tail": init["tail"].astype(np.float64), "kv": init["kv"],
          "pos": init["pos"]}
    tok = syn.stack_tokens(cfg, 1, 1, seed=4)
    with one_core():
        t0 = time.perf_counter()
        for _ in range(tokens):
            tok = orc.decode_stack(m, st, tok, logits=False)["argmax"]
        dt = time.perf_counter() - t0
    out = {"value": tokens / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{tokens} greedy tokens of the full stack, single-threaded C oracle (fp64), pinned to one core",
           **host_info()}
    # the same oracle loops with their output elements over every host core
    # (OpenMP build; same results), on the next tokens of the same stream
    omp = Oracle(all_cores=True)
    mo = omp.make_model(cfg, syn.stack_weights(cfg, seed=4))
    ncores = os.cpu_count() or 1
    t0 = time.perf_counter()
    for _ in range(tokens):
        tok = omp.decode_stack(mo, st, tok, logits=False)["argmax"]
    dt = time.perf_counter() - t0
    out["all_cores"] = {"value": tokens / dt, "unit": UNIT, "cores": ncores, "kind": "oracle (OpenMP build)",
                        "sample": f"{tokens} further greedy tokens of the same stream"}
    return out


# ---------------------------------------------------------------- replicas --

def replica_reduce(vals: list, device: str) -> list:
    """Max over the ranks of each value (device-timed milliseconds, end-to-end
    seconds, status word): the job takes as long as its slowest replica, and an
    error on any rank is the job's.  One all-reduce, which every rank issues at
    the same point."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def aggregate_rate(world: int, units_per_rank: float, seconds: float) -> float:
    """Whole-job throughput of `world` replicas that each processed
    `units_per_rank` units in at most `seconds`."""
    return world * units_per_rank / seconds


# --------------------------------------------------------------------- GPU --

def run_gpu(args) -> None:
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    import hgd_synth as syn
    import hybrid_gated_delta_b200 as hgd

    cfg = syn.STACK_CFG
    if args.layers and args.layers != cfg["n_layers"]:
        cfg = dict(cfg, n_layers=args.layers)
    B = 1
    e2e_steps = max(8, min(args.steps, 64))
    # cache positions for every token this run decodes: warm-up, timed and end-to-end steps
    Lmax = ((PREFILL + args.warmup + args.steps + e2e_steps + 2 + 63) // 64) * 64
    model = hgd.Model(cfg, syn.stack_weights(cfg, seed=4))
    init = syn.stack_state(cfg, B, Lmax, prefill=PREFILL, seed=4 + rank)
    state = hgd.State(model, B, 1, Lmax, init)
    stream = torch.cuda.Stream()
    tok = torch.from_numpy(syn.stack_tokens(cfg, B, 1, seed=4 + rank)).cuda()
    argmax = torch.zeros(B, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok_buf = argmax.view(B, 1)  # greedy: each step reads the previous step's argmax
    tok_buf.copy_(tok)
    split = args.path == "chain"
    launches = chain_launches(cfg) if split else model.launches(B, 1)

    dec = hgd.DecodeGraph(model, state, tok_buf, argmax, status, stream=stream, split=split)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        dec.replay()
    stream.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            dec.replay()
            ev[i][1].record(stream)
        t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    step_ms = [a.elapsed_time(b) for a, b in ev]

    # end to end through the public API: host token in (pinned H2D), host argmax out
    h_tok = torch.empty((B, 1), dtype=torch.int32).pin_memory()
    h_out = torch.empty((B,), dtype=torch.int32).pin_memory()
    h_tok.copy_(argmax.view(B, 1).cpu())
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        dec.step_host(h_tok, h_out)
        h_tok.view(-1).copy_(h_out)
    e2e_s = time.perf_counter() - t0
    dec.close()
    st = int(status.item())

    if world > 1:
        elapsed_ms, e2e_s, st_max = replica_reduce([elapsed_ms, e2e_s, st], "cuda")
        st = int(st_max)
        dist.barrier()
        dist.destroy_process_group()
    assert st == 0, hgd.status_string(st)
    if rank != 0:
        return

    ms_step = elapsed_ms / args.steps
    value = aggregate_rate(world, B * args.steps, elapsed_ms / 1000.0)
    e2e_val = aggregate_rate(world, B * e2e_steps, e2e_s)  # every rank runs the same loop
    L_avg = PREFILL + args.warmup + (args.steps + 1) / 2.0
    ab = algorithmic_bytes(cfg, L_avg)
    peaks = measured_peaks()
    peak = float(peaks.get("hbm_gbs", 6650.0))
    launch_ms = statistics.mean(step_ms)
    kern_gbs = ab["total"] / (launch_ms * 1e-3) / 1e9
    step_gbs = ab["total"] / (ms_step * 1e-3) / 1e9
    prof = {}
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            prof = json.load(f)
    except OSError:
        pass
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD if cfg is syn.STACK_CFG else
                   f"PROFILING ONLY, not a bench line: {cfg['n_layers']}-layer stack of the same width",
                   "batch": 1, "kv_context": PREFILL, "decode_tokens": args.steps,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: 1.5 GB of weights streamed per step (L2 126 MB)"},
        "hbm_gbs": step_gbs,
        "frac_of_8tbs": step_gbs / 8000.0,
        "roofline": {"kernel": ("k_stack: the whole decode step in one cooperative launch" if not split else
                                "the kernel chain of one decode step (GEMV, GDN, attention, argmax kernels)"),
                     "bound": "hbm", "achieved": kern_gbs, "peak": peak, "unit": "GB/s",
                     "frac": kern_gbs / peak, "frac_of_8tbs": kern_gbs / 8000.0,
                     "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if "_fallback" not in peaks
                     else "fallback",
                     "traffic": prof.get("k_stack_bytes_per_launch" if not split else "chain_bytes_per_step"),
                     "algorithmic_bytes": ab["total"], "avg_launch_ms": launch_ms},
        "step_ms": {"median": float(np.median(step_ms)), "p90": float(np.percentile(step_ms, 90)),
                    "p99": float(np.percentile(step_ms, 99)), "how": "CUDA events around each step's graph replay"},
        "gpu_launches": launches * args.steps,
        "path": "kernel chain" if split else "persistent",
        "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": 4 * B, "d2h_bytes_per_step": 4 * B,
                "steps": e2e_steps, "how": "per token: pinned H2D of the token, graph replay of the step, "
                                          "D2H of the argmax, host synchronisation"},
    }
    if clk:
        out["clocks"] = clk
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_sample(tokens=args.cpu_tokens)
    print(json.dumps(out), flush=True)


# ------------------------------------------------------- standalone kernels --

def run_kernels(args) -> None:
    """Per-kernel rooflines of the standalone entry points at the GEMV sweep's
    shapes (K = 1536 projections, fused up/gate, down, a 100000-row head; M = 1,
    8, 32) and the GDN sweep's batches (B = 1, 4, 16, 64; 16 heads of 128).
    Each call streams a different copy of its weights or state (copies totalling
    more than twice the L2), timed with CUDA events; GB/s counts algorithmic
    bytes.  One JSON line per kernel shape; these are not the benchmark line."""
    import torch
    import hybrid_gated_delta_b200 as hgd

    peak = float(measured_peaks().get("hbm_gbs", 6650.0))
    rot_bytes = 256 << 20  # > 2 x the 126 MB L2
    gen = torch.Generator(device="cuda").manual_seed(2)
    stream = torch.cuda.current_stream()

    def timed(fn, ncopies, iters):
        """us per call: `iters` calls (rotating over the copies) captured in one CUDA
        graph and replayed between two events, so the time is the kernels' and not
        the host binding's."""
        for i in range(3 * ncopies if ncopies < 8 else ncopies):
            fn(i % ncopies)
        torch.cuda.synchronize()
        cap = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            for i in range(iters):
                fn(i % ncopies)
        graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        graph.reset()
        return a.elapsed_time(b) * 1e3 / iters  # us per call

    def line(kernel, shape, us, nbytes):
        gbs = nbytes / (us * 1e-6) / 1e9
        print(json.dumps({"kernel": kernel, "shape": shape, "us": us, "algorithmic_bytes": nbytes, "gb_s": gbs,
                          "frac_of_measured_peak": gbs / peak, "frac_of_8tbs": gbs / 8000.0,
                          "note": "standalone kernel roofline, not the benchmark line"}), flush=True)

    K = 1536
    shapes = [("q/k/v/o", 1536, 1536, False), ("up+gate SwiGLU", 4096, 1536, True), ("down", 1536, 4096, False),
              ("LM head", 100000, 1536, False)]
    for name, N, KK, swi in shapes:
        wbytes = (2 if swi else 1) * 2 * N * KK
        ncopies = max(1, min(64, rot_bytes // wbytes))
        Ws = [torch.randn(N, KK, device="cuda", generator=gen).mul_(KK ** -0.5).to(torch.bfloat16)
              for _ in range(ncopies)]
        Us = [torch.randn(N, KK, device="cuda", generator=gen).mul_(KK ** -0.5).to(torch.bfloat16)
              for _ in range(ncopies)] if swi else None
        for M in (1, 8, 32):
            x = torch.randn(M, KK, device="cuda", generator=gen).to(torch.bfloat16)
            ws = hgd.make_workspace(M, N, KK, swiglu=swi)
            if swi:
                h = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
                us = timed(lambda i: hgd.gemv_swiglu_bf16(Ws[i], Us[i], x, h=h, workspace=ws), ncopies, 200)
                nbytes = 2 * 2 * N * KK + 2 * M * KK + 2 * M * N
                line("hgd_gemv_swiglu_bf16 (k_gemv, SwiGLU epilogue)", {"M": M, "I": N, "K": KK}, us, nbytes)
            else:
                y = torch.empty(M, N, dtype=torch.float32, device="cuda")
                us = timed(lambda i: hgd.gemv_bf16(Ws[i], x, y=y, y_is_fp32=True, workspace=ws), ncopies,
                           200 if N < 50000 else 50)
                nbytes = 2 * N * KK + 2 * M * KK + 4 * M * N
                line(f"hgd_gemv_bf16 (k_gemv) {name}", {"M": M, "N": N, "K": KK}, us, nbytes)
        del Ws, Us
        torch.cuda.empty_cache()

    # the tensor-core GEMM at 128 token rows (an 8 x 16 window) on the stack's
    # projection shapes: bytes and flops per call, against the copy and bf16 peaks
    tflops_peak = float(measured_peaks().get("bf16_tflops", 1590.0))
    for name, N, KK in (("GDN in-projection", 8224, 1024), ("up+gate", 7168, 1024), ("down", 1024, 3584),
                        ("LM head", 248320, 1024)):
        M = 128
        wbytes = 2 * N * KK
        ncopies = max(1, min(64, rot_bytes // wbytes))
        Wps = []
        for _ in range(ncopies):
            W = torch.randn(N, KK, device="cuda", generator=gen).mul_(KK ** -0.5).to(torch.bfloat16)
            Wps.append(hgd.gemm_tc_pack_weight(W))
            del W
        torch.cuda.synchronize()
        x = torch.randn(M, KK, device="cuda", generator=gen).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        ws = torch.empty(hgd.gemm_tc_workspace_bytes(M, N, KK), dtype=torch.uint8, device="cuda")
        us = timed(lambda i: hgd.gemm_tc_bf16(Wps[i], x, N, y=y, workspace=ws), ncopies, 50 if N > 50000 else 200)
        nbytes = wbytes + 2 * M * KK + 4 * M * N
        line(f"hgd_gemm_tc_bf16 (k_tc_pack_x + k_gemm_tc) {name}", {"M": M, "N": N, "K": KK}, us,
             nbytes)
        tf = 2.0 * M * N * KK / (us * 1e-6) / 1e12
        print(json.dumps({"kernel": f"hgd_gemm_tc_bf16 {name}", "shape": {"M": M, "N": N, "K": KK}, "tflops": tf,
                          "frac_of_measured_bf16_peak": tf / tflops_peak,
                          "note": "standalone kernel, tensor-core throughput"}), flush=True)
        del Wps
        torch.cuda.empty_cache()

    H, d = 16, 128
    for B in (1, 4, 16, 64):
        sbytes = B * H * d * d * 4
        ncopies = max(4, min(256, rot_bytes // sbytes))
        Ss = [torch.randn(B, H, d, d, device="cuda", generator=gen).mul_(0.1) for _ in range(ncopies)]
        q = torch.randn(B, 1, H, d, device="cuda", generator=gen)
        k = torch.randn(B, 1, H, d, device="cuda", generator=gen)
        v = torch.randn(B, 1, H, d, device="cuda", generator=gen)
        g = -torch.nn.functional.softplus(torch.randn(B, 1, H, device="cuda", generator=gen))
        bb = torch.randn(B, 1, H, device="cuda", generator=gen)
        o = torch.empty(B, 1, H, d, device="cuda")
        us = timed(lambda i: hgd.gdn_decode_step(q, k, v, g, bb, Ss[i], o=o), ncopies, 400)
        nbytes = 2 * sbytes + 4 * B * H * d * 4 + 2 * B * H * 4
        line("hgd_gdn_decode_step (k_gdn_step)", {"B": B, "H": H, "dk": d, "dv": d, "T": 1}, us, nbytes)
        # a 16-row verify window that logs instead of writing the state, then keep(16)
        T = 16
        qw = torch.randn(B, T, H, d, device="cuda", generator=gen)
        kw = torch.randn(B, T, H, d, device="cuda", generator=gen)
        vw = torch.randn(B, T, H, d, device="cuda", generator=gen)
        gw = -torch.nn.functional.softplus(torch.randn(B, T, H, device="cuda", generator=gen))
        bw = torch.randn(B, T, H, device="cuda", generator=gen)
        ow = torch.empty(B, T, H, d, device="cuda")
        _, la, ld, lk = hgd.gdn_window_log(qw, kw, vw, gw, bw, Ss[0], o=ow)
        us = timed(lambda i: hgd.gdn_window_log(qw, kw, vw, gw, bw, Ss[i], o=ow), ncopies, 200)
        nbytes = sbytes + 4 * B * T * H * (3 * d + 2) + 4 * B * T * H * (d + 1 + d + d)
        line("hgd_gdn_window_log (k_gdn_window_log)", {"B": B, "H": H, "dk": d, "dv": d, "T": T}, us, nbytes)
        keep = torch.full((B,), T, dtype=torch.int32, device="cuda")
        us = timed(lambda i: hgd.gdn_keep(Ss[i], la, ld, lk, keep), ncopies, 200)
        nbytes = 2 * sbytes + 4 * B * T * H * (1 + 2 * d) + 4 * B
        line("hgd_gdn_keep (k_gdn_keep)", {"B": B, "H": H, "dk": d, "dv": d, "T": T}, us, nbytes)
        del Ss
        torch.cuda.empty_cache()

    # prefill: a 512-row prompt through one GDN layer's recurrence (16 heads of 128),
    # the chunked form against the one-row-at-a-time kernel over the same rows
    H, d, T = 16, 128, 512
    for B in (1, 8):
        qp = torch.randn(B, T, H, d, device="cuda", generator=gen)
        kp = torch.randn(B, T, H, d, device="cuda", generator=gen)
        vp = torch.randn(B, T, H, d, device="cuda", generator=gen)
        gp = -torch.nn.functional.softplus(torch.randn(B, T, H, device="cuda", generator=gen))
        bp = torch.randn(B, T, H, device="cuda", generator=gen)
        Sp = [torch.randn(B, H, d, d, device="cuda", generator=gen).mul_(0.1) for _ in range(4)]
        op = torch.empty(B, T, H, d, device="cuda")
        for name, fn in (("hgd_gdn_prefill (k_gdn_chunked, 32-row chunks)",
                          lambda i: hgd.gdn_prefill(qp, kp, vp, gp, bp, Sp[i], o=op)),
                         ("hgd_gdn_decode_step over the prompt (k_gdn_step, row by row)",
                          lambda i: hgd.gdn_decode_step(qp, kp, vp, gp, bp, Sp[i], o=op))):
            us = timed(fn, 4, 20)
            print(json.dumps({"kernel": name, "shape": {"B": B, "T": T, "H": H, "dk": d, "dv": d}, "us": us,
                              "tokens_per_s": B * T / (us * 1e-6),
                              "note": "prefill of one GDN layer's recurrence, not the benchmark line"}), flush=True)
        del Sp
        torch.cuda.empty_cache()

    # the causal conv tail update of one GDN layer's q|k|v channels (6144), one row
    Cc, kc = 6144, 4
    for B in (1, 8, 64):
        tbytes = B * (kc - 1) * Cc * 4
        ncopies = max(4, min(256, rot_bytes // (2 * tbytes)))
        xs = [torch.randn(B, 1, Cc, device="cuda", generator=gen) for _ in range(ncopies)]
        tails = [torch.randn(B, kc - 1, Cc, device="cuda", generator=gen) for _ in range(ncopies)]
        wc = torch.randn(Cc, kc, device="cuda", generator=gen).to(torch.bfloat16)
        yc = torch.empty(B, 1, Cc, device="cuda")
        us = timed(lambda i: hgd.conv1d_tail_update(xs[i], tails[i], wc, y=yc), ncopies, 400)
        nbytes = 2 * tbytes + 2 * B * Cc * 4 + Cc * kc * 2
        line("hgd_conv1d_tail_update (k_conv_tail)", {"B": B, "T": 1, "C": Cc, "kc": kc}, us, nbytes)
        del xs, tails
        torch.cuda.empty_cache()


def run_windows(args) -> None:
    """Throughput of the window workload: 8 streams x 16 rows per decode call
    (128 token rows through the 24-layer stack, the kernel chain's path for more
    than 8 rows), replayed from a CUDA graph; 16 windows per stream after the
    512-key prefill.  Not the benchmark line."""
    import torch
    import hgd_synth as syn
    import hybrid_gated_delta_b200 as hgd

    cfg = syn.STACK_CFG
    B, T, n_win, warm = 8, 16, 16, 2
    Lmax = ((PREFILL + (n_win + warm + 1) * T + 63) // 64) * 64
    model = hgd.Model(cfg, syn.stack_weights(cfg, seed=5), tc=args.tc)
    state = hgd.State(model, B, T, Lmax, syn.stack_state(cfg, B, Lmax, prefill=PREFILL, seed=5))
    decode = hgd.decode_layer_stack_tc if args.tc else hgd.decode_layer_stack
    toks = torch.from_numpy(syn.stack_tokens(cfg, B, T, seed=5)).cuda()
    am = torch.zeros(B * T, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        decode(model, state, toks, T, argmax=am, status=status, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        decode(model, state, toks, T, argmax=am, status=status)
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(n_win - warm - 1):
            g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, hgd.status_string(int(status.item()))
    n = n_win - warm - 1
    ms = a.elapsed_time(b) / n
    ab = algorithmic_bytes(cfg, PREFILL + (warm + 1 + n / 2.0) * T)
    nbytes = ab["weights"] + B * (ab["total"] - ab["weights"])  # weights once, state and cache per stream
    print(json.dumps({"workload": "8 streams x 16-row windows (128 token rows per call), 24-layer stack",
                      "path": "tensor-core chain (tcgen05 GEMMs)" if args.tc else "mma.sync kernel chain",
                      "calls": n, "ms_per_call": ms, "tokens_per_s": B * T / (ms * 1e-3),
                      "algorithmic_bytes_per_call": nbytes, "gb_s": nbytes / (ms * 1e-3) / 1e9,
                      "launches_per_call": None if args.tc else model.launches(B, T),
                      "note": "window throughput, not the benchmark line"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling aid: a stack of this many layers of the same width (the line it prints "
                         "is marked as not a bench line); 0 = the benchmark's 24")
    ap.add_argument("--path", default="persistent", choices=["chain", "persistent"],
                    help="chain: one kernel per op, PDL-overlapped, in CUDA graphs; "
                         "persistent: the whole step in one cooperative launch")
    ap.add_argument("--cpu-tokens", type=int, default=12)  # about 13 s of oracle work at ~1 token/s
    ap.add_argument("--windows", action="store_true",
                    help="instead of the benchmark line: throughput of 8 streams x 16-row windows")
    ap.add_argument("--tc", action="store_true",
                    help="with --windows: the tensor-core decode chain (hgd_decode_layer_stack_tc)")
    ap.add_argument("--kernels", action="store_true",
                    help="instead of the benchmark line: per-kernel rooflines of the standalone GEMV and GDN "
                         "entry points at the sweep shapes")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.kernels:
        run_kernels(args)
    elif args.windows:
        run_windows(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
