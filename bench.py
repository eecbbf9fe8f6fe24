#!/usr/bin/env python3
"""Benchmark of the TTT-E2E inner loop with the E2-TTT chunk update on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one full prefill call (every chunk of every sequence of the
workload: gather, MLP forward, fused LM-head cross-entropy, backward and the
closed-form weight/momentum update) on inputs already resident in HBM.
Metric: inner-loop tokens per second over the whole job (all GPUs), and the
algorithmic FLOP rate against the measured bf16 tensor-core peak.

Multi-GPU (launched by torch.distributed.run): every rank processes its own
independent sequences (the workload with seed = rank); there is no
data-path collective, only a barrier around the timed region and a max of the
elapsed time over ranks (weak scaling).

--impl reference times the CPU oracle (numpy, float32 BLAS on the host cores)
on a bounded sample of the same workload: it is a baseline, not the target.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_long_context_b200 import inputs as I  # noqa: E402

METRIC = "TTT inner-loop tokens/sec at 1 B200; % of bf16 tensor-core peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "stack_128k"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# Workload arithmetic (algorithmic work per token; a restatement of the
# method's FLOP count, not a measurement)
# ---------------------------------------------------------------------------

def flops_per_token(w: I.Workload) -> float:
    """Algorithmic FLOPs per token of one inner-loop pass.

    Each MLP forward 2 m d h; LM head 4 d V (logits + dz, the head is frozen);
    backward to every dynamic MLP's activation 2 d h, plus 2 (m-1) d h for dX
    when a dynamic MLP lies below, plus 2 m d h per static MLP above the lowest
    dynamic one; aggregation 2 m d h per dynamic MLP per kernel (x2 for K_W and
    K_M, x1 for plain SGD where M_C = eta_C G_C is a rank-1 write).  The
    logits recompute of the cross-entropy backward is not counted.
    """
    d, h, V, L, m = w.d, w.hidden, w.vocab, w.n_blocks, w.n_mats
    if w.head == "recon":
        # E2-TTT's layer: MLP forward on keys and on queries, backward to the
        # activation only (one block), both aggregations
        return float(2 * (2 * m * d * h) + 2 * d * h + 2 * m * d * h * (1 if w.scalars == "sgd" else 2))
    n_static = L if w.has_static else 0
    fwd = (L + n_static) * 2 * m * d * h
    head = 4 * d * V
    bwd = L * 2 * d * h + (L - 1) * 2 * (m - 1) * d * h + (max(n_static - 1, 0)) * 2 * m * d * h
    agg = L * 2 * m * d * h * (1 if w.scalars == "sgd" else 2)
    return float(fwd + head + bwd + agg) + attention_flops_per_token(w)


def attention_flops_per_token(w: I.Workload) -> float:
    """Algorithmic FLOPs per token added by frozen sliding-window attention.

    Forward, every block: the q|k|v and o projections 8 d^2 and the scores and
    P V over the keys a query sees, 4 d k_bar (k_bar = mean over positions of
    min(window, t + 1)).  Backward, every block above the lowest, once per
    weighted stream (two): the projections 8 d^2, dP and dQ 4 d k_bar, dK and
    dV over the query's own chunk 4 d b_bar (b_bar = mean of min(window, i + 1)
    over in-chunk positions i); plus the second stream through the MLPs of the
    blocks below the top one (B1 2 d h, B2 2 (m - 1) d h where a gradient
    continues below).
    """
    if not w.attn_heads:
        return 0.0
    d, h, L, m = w.d, w.hidden, w.n_blocks, w.n_mats
    t = np.arange(w.T)
    kbar = float(np.minimum(w.attn_window, t + 1).mean())
    bbar = float(np.minimum(w.attn_window, np.arange(w.b) + 1).mean())
    fwd = L * (8 * d * d + 4 * d * kbar)
    bwd = (L - 1) * 2 * (8 * d * d + 4 * d * kbar + 4 * d * bbar)
    mlp2 = 0.0
    for l in range(L - 1):
        mlp2 += 2 * d * h + (2 * (m - 1) * d * h if l > 0 else 0)
        if w.has_static and l > 0:
            mlp2 += 2 * d * h + 2 * (m - 1) * d * h
    return float(fwd + bwd + mlp2)


def predict_flops_per_token(w: I.Workload) -> float:
    """Algorithmic FLOPs per token of the forward-only final prediction: every
    MLP forward 2 m d h and the logits 2 d V."""
    n_static = w.n_blocks if w.has_static else 0
    return float((w.n_blocks + n_static) * 2 * w.n_mats * w.d * w.hidden + 2 * w.d * w.vocab)


def state_bytes(w: I.Workload) -> int:
    return w.batch * w.n_blocks * w.block_params * 4 * 2


def input_bytes(w: I.Workload) -> int:
    return w.batch * w.T * (w.d * 4 + 4 + 12)


def min_bytes_per_step(w: I.Workload) -> float:
    """Algorithmic HBM bytes of one inner-loop pass: per chunk, every dynamic
    parameter's fp32 W and M read and written once plus its bf16 (fp32 in fp32
    mode) operand shadow written; the frozen LM head and static MLPs read once
    per chunk (they are shared by the sequences of a batch); the inputs (hidden
    rows, tokens, three scalars) read once."""
    e = 4 if w.precision == "fp32" else 2
    dyn = w.batch * w.n_blocks * w.block_params
    frozen = (w.vocab * w.d + (w.n_blocks * w.block_params if w.has_static else 0)) * e
    per_chunk = dyn * (16 + e) + frozen
    return float(w.n_chunks * per_chunk + input_bytes(w))


def hbm_line(w: I.Workload, ms: float, pk: dict) -> dict:
    by = min_bytes_per_step(w)
    gbs = by / (ms / 1e3) / 1e9
    return {"algorithmic_bytes_per_step": by, "achieved_GBs": gbs, "frac": gbs / pk["hbm"],
            "peak_GBs": pk["hbm"], "what": "state read+write and operand shadow per chunk, frozen head and "
                                         "static MLPs once per chunk, inputs once"}


def measured_peaks() -> dict:
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return {}


def peaks():
    m = measured_peaks()
    if m.get("bf16_tflops") and m.get("hbm_gbs"):
        return dict(tflops=float(m["bf16_tflops"]), tflops_sustained=float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                    hbm=float(m["hbm_gbs"]), source="measured")
    return dict(tflops=1590.0, tflops_sustained=1400.0, hbm=6650.0, source="fallback")


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    def __init__(self):
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="ttt_clocks_", suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             + ",".join("clocks_event_reasons." + r for r in REASONS))
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvidia-smi unavailable"}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons, power = [], [], set(), []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 5 + len(REASONS):
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for r, v in zip(REASONS, f[5:5 + len(REASONS)]):
                if v.lower() == "active":
                    reasons.add(r)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": sorted(reasons), "samples": 0}
        # samples under load: power above the midpoint of the observed range
        pmin, pmax = min(power), max(power)
        load = [s for s, p in zip(sm, power) if p >= pmin + 0.5 * (pmax - pmin)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": pmax}


# ---------------------------------------------------------------------------
# Multi-rank helpers (tested on CPU with gloo)
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(backend: str, timeout_s: int = 180):
    import datetime
    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    return units_per_rank * world / max_seconds if max_seconds > 0 else 0.0


# The sources that define the profiled GEMM kernels (engine, epilogues and the
# helpers they include): a committed ncu summary is used only while these match.
KERNEL_SOURCES = ("common.cuh", "gemm_types.cuh", "gemm_tc.cuh", "epilogue.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "weight_long_context_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m_h = re.search(r"kernel_source_hash:\s*(\w+)", txt)
    m_t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not (m_h and m_t) or m_h.group(1) != kernel_source_hash():
        return None
    return float(m_t.group(1))


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline of our arm; the whole reference arm)
# ---------------------------------------------------------------------------

def oracle_chunks(w: I.Workload, n_chunks: int, seed: int = 0):
    """Run the oracle on the first n_chunks chunks of one sequence; returns seconds."""
    import oracle  # test infrastructure: the CPU baseline only
    ws = w.with_(T=n_chunks * w.b, batch=1)
    dtype = np.float64 if w.precision == "fp32" else np.float32
    if w.head == "recon":
        x = I.make_recon_inputs(ws, seed=seed)
        t0 = time.perf_counter()
        oracle.prefill_recon(w.mlp, w.d, w.hidden, x["W0"], x["M0"], x["K"], x["V"], x["Q"], x["eta"], x["beta"],
                             x["gamma"], w.b, w.rms_eps, dtype=dtype, reduction=w.reduction,
                             update="lact" if w.update_rule == "lact" else "closed")
        return time.perf_counter() - t0
    x = I.make_inputs(ws, seed=seed)
    model = oracle.make_model(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.rms_eps, x["lm_head"], x["rms_gain"],
                              x["static_w"], dtype=dtype)
    if w.attn_heads:
        a = I.make_swa_inputs(ws, seed=seed)
        sw = oracle.swa_oracle.make_swa(w.d, w.n_blocks, w.attn_heads, w.attn_window, a["attn_w"], a["ln_gain"],
                                        a["ln_bias"])
        t0 = time.perf_counter()
        oracle.swa_oracle.prefill(model, sw, x["W0"], x["M0"], x["hidden"], x["tokens"], x["eta"], x["beta"],
                                  x["gamma"], w.b, dtype=dtype, rule=w.update_rule, reduction=w.reduction)
        return time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.prefill(model, x["W0"], x["M0"], x["hidden"], x["tokens"], x["eta"], x["beta"], x["gamma"], w.b,
                   dtype=dtype, reduction=w.reduction, update="lact" if w.update_rule == "lact" else "closed")
    return time.perf_counter() - t0


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(w: I.Workload, budget_s: float = 12.0) -> dict:
    """Oracle tokens/s on a bounded sample: whole chunks of one sequence until
    about budget_s of CPU work (at least one chunk)."""
    t1 = oracle_chunks(w, 1)
    k = max(1, min(w.n_chunks, int(budget_s / max(t1, 1e-3))))
    tk = oracle_chunks(w, k) if k > 1 else t1
    prec = "float64" if w.precision == "fp32" else "float32"
    return {"value": k * w.b / tk, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"first {k} chunk(s) ({k * w.b} tokens) of one sequence of {w.name}, numpy {prec} "
                      f"BLAS, {tk:.1f} s"}


def cpu_baseline_predict(w: I.Workload, rows: int = 512) -> dict:
    """Oracle tokens/s of the final prediction on a bounded sample: the first
    `rows` tokens of one sequence."""
    import oracle  # test infrastructure: the CPU baseline only
    ws = w.with_(T=rows, b=rows, batch=1)
    x = I.make_inputs(ws, seed=0)
    dtype = np.float64 if w.precision == "fp32" else np.float32
    model = oracle.make_model(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.rms_eps, x["lm_head"], x["rms_gain"],
                              x["static_w"], dtype=dtype)
    t0 = time.perf_counter()
    oracle.final_prediction(model, x["W0"], x["hidden"], x["tokens"], rows, dtype=dtype)
    dt = time.perf_counter() - t0
    prec = "float64" if w.precision == "fp32" else "float32"
    return {"value": rows / dt, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"final prediction of the first {rows} tokens of one sequence of {w.name}, numpy {prec} "
                      f"BLAS, {dt:.1f} s"}


def run_reference(args, w: I.Workload):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    per = oracle_chunks(w, 1)
    k_chunks = max(1, min(w.n_chunks, int(15.0 / max(per * (args.steps + args.warmup), 1e-3))))
    for _ in range(args.warmup):
        oracle_chunks(w, k_chunks)
    times = [oracle_chunks(w, k_chunks) for _ in range(args.steps)]
    tok = k_chunks * w.b
    value = tok * args.steps / sum(times)
    cb = {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
          "sample": f"each step: first {k_chunks} chunk(s) ({tok} tokens) of one sequence of {w.name}, "
                    f"numpy float32 BLAS"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32" if w.precision != "fp32" else "f64",
            "data": "synthetic", "impl": "reference", "config": workload_config(w),
            "cpu_baseline": cb, "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: I.Workload) -> dict:
    big = input_bytes(w) + state_bytes(w) > 2 * L2_BYTES
    return {"workload": w.name, "d": w.d, "hidden": w.hidden, "vocab": w.vocab, "blocks": w.n_blocks,
            "mlp": w.mlp, "static_mlp": w.has_static, "T": w.T, "chunk_b": w.b, "sequences_per_gpu": w.batch,
            "scalars": w.scalars, "loss_reduction": w.reduction, "update_rule": w.update_rule,
            "head": "next-token cross-entropy" if w.head == "lm" else "key/value reconstruction (E2-TTT layer)",
            "precision": "fp32" if w.precision == "fp32" else "bf16 GEMM operands, fp32 accumulate/state",
            **({"attention": {"heads": w.attn_heads, "window": w.attn_window,
                              "kind": "frozen causal sliding-window, rotary, LayerNorm in front"}}
               if w.attn_heads else {}),
            "l2": ("inputs larger than L2 (hidden + fast-weight state %.2f GiB per step)" % ((input_bytes(w) + state_bytes(w)) / 2 ** 30))
                  if big else "L2 flushed between timed steps (write of a 256 MiB buffer)"}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def run_ours(args, w: I.Workload):
    if w.head == "recon":
        return run_ours_recon(args, w)
    import torch
    from weight_long_context_b200 import ttt

    rank, world, local = dist_env()
    if world > 1:
        init_dist("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    st = torch.cuda.current_stream(dev)

    x = I.make_inputs(w, seed=rank)
    T = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    h = ttt.Handle(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.has_static, w.precision, T(x["lm_head"]),
                   T(x["rms_gain"]), T(x["static_w"]) if x["static_w"] is not None else None, w.rms_eps,
                   w.reduction, w.update_rule)
    if w.attn_heads:
        a = I.make_swa_inputs(w, seed=rank)
        h.set_attention(w.attn_heads, w.attn_window, T(a["attn_w"]), T(a["ln_gain"]), T(a["ln_bias"]))
    hidden, tokens = T(x["hidden"]), T(x["tokens"], torch.int32)
    W, M = T(x["W0"]), T(x["M0"])
    eta, beta, gamma = T(x["eta"]), T(x["beta"]), T(x["gamma"])
    flush = None
    if input_bytes(w) + state_bytes(w) <= 2 * L2_BYTES:
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)

    heads = None
    if args.scalar_heads:
        rng = np.random.default_rng(100 + rank)
        heads = (T(rng.normal(0.0, 1.0 / np.sqrt(w.d), (3, w.d))), (0.0, 0.0, 0.0), 0.01, 1.0, 16.0)

    # Every step is one prefill from the initial state: W and M are restored
    # from W0 / M0 before each step, outside the timed events.
    W0d, M0d = W.clone(), M.clone()

    def step(g=None):
        if heads is not None:
            e_, b_, g_ = ttt.ttt_scalar_heads(hidden, *heads, stream=st)
            return h.prefill(hidden, tokens, W, M, e_, b_, g_, w.b, stream=st)
        return h.prefill(hidden, tokens, W, M, eta, beta, gamma if g is None else g, w.b, stream=st)

    def timed_steps(n_steps, g=None):
        """args.warmup untimed steps, then n_steps steps each bracketed by CUDA
        events on the launching stream (the state restore and the L2 flush sit
        outside the events); returns per-step ms and the sampled clocks."""
        for _ in range(args.warmup):
            W.copy_(W0d)
            M.copy_(M0d)
            step(g)
        torch.cuda.synchronize()
        assert h.device_status() == 0, "device status after warm-up"
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
        clocks = ClockSampler()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        if rank == 0:
            clocks.start()
        for i in range(n_steps):
            W.copy_(W0d)
            M.copy_(M0d)
            if flush is not None:
                flush.fill_(i & 0xff)
            ev[i][0].record(st)
            step(g)
            ev[i][1].record(st)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        clk = clocks.stop() if rank == 0 else None
        return [a.elapsed_time(b) for a, b in ev], clk

    # ---- timed region: K steps, per-step CUDA events on the launching stream
    step_ms, clk = timed_steps(args.steps)
    status = h.device_status()
    mean_ms = reduce_max(statistics.mean(step_ms), dev)
    tokens_per_step = w.batch * w.T
    value = whole_job_rate(tokens_per_step, world, mean_ms / 1e3)
    state_norm = float(torch.linalg.vector_norm(W).item())

    # ---- the same workload on a state that stays live (gamma = 1): under the
    # E2-TTT draw W and M decay towards zero within a step, and GEMMs on zero
    # operands draw less power; this timing shows what that is worth.
    live = None
    if w.scalars == "e2ttt" and heads is None and not args.no_live_state:
        g1 = torch.ones_like(gamma)
        live_ms, live_clk = timed_steps(max(3, min(args.steps, 10)), g1)
        live_mean = reduce_max(statistics.mean(live_ms), dev)
        live = {"value": whole_job_rate(tokens_per_step, world, live_mean / 1e3), "unit": UNIT,
                "ms_per_step": live_mean, "steps": len(live_ms), "clocks": live_clk,
                "scalars": "eta and beta of the workload's draw, gamma = 1 (no decay)",
                "final_W_norm": float(torch.linalg.vector_norm(W).item())}
        if live_clk and live_clk.get("sm_mhz"):
            live["cycles_per_step"] = live_mean * 1e-3 * live_clk["sm_mhz"] * 1e6

    # ---- per-kernel breakdown from one profiled replay (same launches, eager, events per launch)
    W2, M2 = W0d.clone(), M0d.clone()
    _, stats = h.prefill_profiled(hidden, tokens, W2, M2, eta, beta, gamma, w.b, stream=st)
    del W2, M2
    launches_per_step = sum(s["launches"] for s in stats)
    pk = peaks()
    gemms = [s for s in stats if s["flops"] > 0]
    dom = max(gemms, key=lambda s: s["ms"])
    t_tensor = dom["flops"] / (pk["tflops_sustained"] * 1e12)
    t_hbm = dom["bytes"] / (pk["hbm"] * 1e9)
    bound = "tensor" if t_tensor >= t_hbm else "hbm"
    per_launch_ms = dom["ms"] / dom["launches"]
    if bound == "tensor":
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        peak, unit = pk["tflops_sustained"], "TFLOP/s"
    else:
        achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
        peak, unit = pk["hbm"], "GB/s"
    traffic = profiled_traffic(dom["name"], w.name)
    step_total = sum(s["ms"] for s in stats)
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": traffic, "kernel": dom["name"], "launches_per_step": dom["launches"],
                "ms_per_launch": per_launch_ms, "share_of_step": dom["ms"] / step_total,
                "algorithmic_flops_per_launch": dom["flops"] / dom["launches"],
                "algorithmic_bytes_per_launch": dom["bytes"] / dom["launches"],
                "peak_source": f"{pk['source']} (bf16 sustained; HBM copy)"}

    # ---- the scalar heads alone (when used): HBM-bound, one read of the hidden rows
    heads_line = None
    if heads is not None:
        reps = 10
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ttt.ttt_scalar_heads(hidden, *heads, stream=st)
        a_.record(st)
        for _ in range(reps):
            ttt.ttt_scalar_heads(hidden, *heads, stream=st)
        b_.record(st)
        torch.cuda.synchronize()
        hms = a_.elapsed_time(b_) / reps
        hbytes = 4.0 * hidden.numel() + 3 * 4.0 * w.batch * w.T + 12.0 * w.d
        heads_line = {"us_per_call": 1e3 * hms, "algorithmic_bytes": hbytes,
                      "achieved_GBs": hbytes / (hms / 1e3) / 1e9, "frac_hbm": hbytes / (hms / 1e3) / 1e9 / pk["hbm"],
                      "share_of_step": hms / mean_ms}

    # ---- end to end through the public API with host buffers
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    hx = [pin(x["hidden"]), pin(x["tokens"].astype(np.int32)), pin(x["W0"]), pin(x["M0"]), pin(x["eta"]),
          pin(x["beta"]), pin(x["gamma"])]
    h2d = sum(t.numel() * t.element_size() for t in (hx[:4] if heads is not None else hx))
    d2h = 2 * hx[2].numel() * 4 + w.batch * w.n_chunks * 4
    del hidden, tokens, W, M, W0d, M0d, eta, beta, gamma
    torch.cuda.empty_cache()
    h.prefill_host(*hx, b=w.b, stream=st, scalar_heads=heads)    # warm the host path once
    e_steps = max(1, min(args.steps, 3))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(e_steps):
        h.prefill_host(*hx, b=w.b, stream=st, scalar_heads=heads)
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e_steps, dev)
    e2e = {"value": whole_job_rate(tokens_per_step, world, e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e_steps}

    if world > 1:
        dist.barrier()
    if rank == 0:
        fl = flops_per_token(w)
        tflops = value * fl / 1e12
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.precision == "bf16" else "f32", "data": "synthetic",
                "config": workload_config(w),
                "algorithmic_tflops": tflops,
                "pct_of_bf16_peak": {"burst": tflops / world / pk["tflops"],
                                     "sustained": tflops / world / pk["tflops_sustained"], "source": pk["source"]},
                "clocks": clk, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
                "roofline": roofline, "device_status": status, "final_W_norm": state_norm,
                "breakdown": {st_["name"]: {"launches": st_["launches"], "ms": round(st_["ms"], 3),
                                            "us_per_launch": round(1e3 * st_["ms"] / st_["launches"], 2),
                                            "share": round(st_["ms"] / step_total, 4)}
                              for st_ in sorted(stats, key=lambda q: -q["ms"])},
                "us_per_chunk": 1e3 * mean_ms / w.n_chunks,
                "hbm": hbm_line(w, mean_ms, pk)}
        if clk and clk.get("sm_mhz"):
            line["cycles_per_step"] = mean_ms * 1e-3 * clk["sm_mhz"] * 1e6
        if live is not None:
            line["live_state"] = live
        if heads_line is not None:
            line["config"]["scalars"] = "input-dependent heads (eta_base 0.01, alpha_base 1, tau 16)"
            line["scalar_heads"] = heads_line
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ours_recon(args, w: I.Workload):
    """E2-TTT's own layer (ttt_prefill_recon): the same timing rules; the
    roofline is taken over the whole step (this head has no per-kernel replay)."""
    import torch
    from weight_long_context_b200 import ttt

    rank, world, local = dist_env()
    if world > 1:
        init_dist("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    st = torch.cuda.current_stream(dev)
    x = I.make_recon_inputs(w, seed=rank)
    T = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    h = ttt.Handle(w.d, w.hidden, w.vocab, 1, w.mlp, False, w.precision, None, None, None, w.rms_eps, w.reduction,
                   w.update_rule, head="recon", device=dev)
    K, V, Q, W, M = T(x["K"]), T(x["V"]), T(x["Q"]), T(x["W0"]), T(x["M0"])
    eta, beta, gamma = T(x["eta"]), T(x["beta"]), T(x["gamma"])
    O = torch.empty_like(K)
    flush = None
    if 3 * K.numel() * 4 + state_bytes(w) <= 2 * L2_BYTES:
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)

    def step():
        return h.prefill_recon(K, V, Q, W, M, eta, beta, gamma, w.b, O=O, stream=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert h.device_status() == 0, "device status after warm-up"
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(i & 0xff)
        ev[i][0].record(st)
        step()
        ev[i][1].record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else None
    step_ms = [a.elapsed_time(b) for a, b in ev]
    status = h.device_status()
    mean_ms = reduce_max(statistics.mean(step_ms), dev)
    tokens_per_step = w.batch * w.T
    value = whole_job_rate(tokens_per_step, world, mean_ms / 1e3)
    pk = peaks()
    # kernels per step in ttt_prefill_recon's launch sequence: the scalar scan and
    # the operand shadow, then per chunk two gathers, four forward GEMMs, the
    # row kernel, the chunk mean, the backward GEMM and the two aggregations
    launches = 2 + 11 * w.n_chunks

    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    hx = [pin(x[k]) for k in ("K", "V", "Q", "W0", "M0", "eta", "beta", "gamma")]
    h2d = sum(t.numel() * t.element_size() for t in hx)
    d2h = 2 * hx[3].numel() * 4 + w.batch * w.n_chunks * 4 + hx[0].numel() * 4
    del K, V, Q, W, M, eta, beta, gamma, O
    torch.cuda.empty_cache()
    h.prefill_recon_host(*hx, b=w.b, stream=st)
    e_steps = max(1, min(args.steps, 3))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(e_steps):
        h.prefill_recon_host(*hx, b=w.b, stream=st)
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e_steps, dev)
    if world > 1:
        dist.barrier()
    if rank == 0:
        fl = flops_per_token(w)
        tflops = value * fl / 1e12
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.precision == "bf16" else "f32", "data": "synthetic",
                "config": workload_config(w), "algorithmic_tflops": tflops,
                "pct_of_bf16_peak": {"burst": tflops / world / pk["tflops"],
                                     "sustained": tflops / world / pk["tflops_sustained"], "source": pk["source"]},
                "clocks": clk,
                "e2e": {"value": whole_job_rate(tokens_per_step, world, e2e_ms / 1e3), "unit": UNIT,
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                        "steps": e_steps},
                "gpu_launches": launches * args.steps,
                "roofline": {"bound": "tensor", "achieved": tflops / world, "peak": pk["tflops_sustained"],
                             "unit": "TFLOP/s", "frac": tflops / world / pk["tflops_sustained"], "traffic": None,
                             "kernel": "whole step (this head has no per-kernel replay)",
                             "peak_source": f"{pk['source']} (bf16 sustained)"},
                "device_status": status}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ours_predict(args, w: I.Workload):
    """Forward-only final prediction at fixed fast weights (ttt_predict) over
    the whole sequence, args.predict_rows rows per sequence per pass; the same
    timing rules as the inner loop, the roofline over the whole step."""
    import torch
    from weight_long_context_b200 import ttt

    rank, world, local = dist_env()
    if world > 1:
        init_dist("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    st = torch.cuda.current_stream(dev)
    rows = args.predict_rows
    if w.T % rows:
        raise SystemExit(f"--predict-rows must divide T = {w.T}")
    x = I.make_inputs(w, seed=rank)
    T = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    h = ttt.Handle(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.has_static, w.precision, T(x["lm_head"]),
                   T(x["rms_gain"]), T(x["static_w"]) if x["static_w"] is not None else None, w.rms_eps,
                   w.reduction, w.update_rule)
    hidden, tokens, W = T(x["hidden"]), T(x["tokens"], torch.int32), T(x["W0"])
    grp = torch.empty((w.batch, w.T // rows), dtype=torch.float32, device=dev)
    flush = None
    if input_bytes(w) + state_bytes(w) <= 2 * L2_BYTES:
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)

    def step():
        return h.predict(hidden, tokens, W, rows, group_loss=grp, stream=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert h.device_status() == 0, "device status after warm-up"
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(i & 0xff)
        ev[i][0].record(st)
        step()
        ev[i][1].record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else None
    step_ms = [a.elapsed_time(b) for a, b in ev]
    status = h.device_status()
    mean_ms = reduce_max(statistics.mean(step_ms), dev)
    tokens_per_step = w.batch * w.T
    value = whole_job_rate(tokens_per_step, world, mean_ms / 1e3)
    pk = peaks()
    # kernels per step in ttt_predict's launch sequence: the operand shadow of
    # W, then per pass the gather, two GEMMs per MLP, the RMSNorm, the logits
    # GEMM, the cross-entropy row reduction and the group mean
    n_mlp = w.n_blocks * (2 if w.has_static else 1)
    launches = 1 + (w.T // rows) * (5 + 2 * n_mlp)

    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    hx = [pin(x["hidden"]), pin(x["tokens"].astype(np.int32)), pin(x["W0"])]
    h2d = sum(t.numel() * t.element_size() for t in hx)
    d2h = grp.numel() * 4
    del hidden, tokens, W
    torch.cuda.empty_cache()
    h.predict_host(*hx, b=rows, stream=st)
    e_steps = max(1, min(args.steps, 3))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(e_steps):
        h.predict_host(*hx, b=rows, stream=st)
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e_steps, dev)
    if world > 1:
        dist.barrier()
    if rank == 0:
        tflops = value * predict_flops_per_token(w) / 1e12
        cfg = workload_config(w)
        cfg.update(workload=w.name + " final prediction", rows_per_pass=rows,
                   pass_kind="forward only at fixed fast weights (no backward, no update)")
        line = {"metric": "final-prediction tokens/sec at 1 B200 (forward only at W_T)", "value": value,
                "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if w.precision == "bf16" else "f32", "data": "synthetic", "config": cfg,
                "algorithmic_tflops": tflops, "clocks": clk,
                "e2e": {"value": whole_job_rate(tokens_per_step, world, e2e_ms / 1e3), "unit": UNIT,
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                        "steps": e_steps},
                "gpu_launches": launches * args.steps,
                "roofline": {"bound": "tensor", "achieved": tflops / world, "peak": pk["tflops_sustained"],
                             "unit": "TFLOP/s", "frac": tflops / world / pk["tflops_sustained"], "traffic": None,
                             "kernel": "whole step (forward GEMMs and the logits GEMM dominate)",
                             "peak_source": f"{pk['source']} (bf16 sustained)"},
                "device_status": status}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_predict(w)
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=I.WORKLOAD_ORDER + ["e2ttt_layer_128k", "stack_128k_swa"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-live-state", action="store_true",
                    help="skip the second timing on a state that stays live (gamma = 1)")
    ap.add_argument("--scalars", default="", choices=["", "e2ttt_live"],
                    help="override the workload's scalar recipe (e2ttt_live: the E2-TTT draw with gamma = 1)")
    ap.add_argument("--scalar-heads", action="store_true",
                    help="input-dependent scalars: eta, beta, gamma computed from the hidden rows on the device "
                         "inside every step (eta_base 0.01, alpha_base 1, tau 16, heads N(0, 1/d))")
    ap.add_argument("--update-rule", default="e2ttt", choices=["e2ttt", "lact"],
                    help="chunk update rule: Proposition 3.1 (default) or LaCT's chunk-wise rule")
    ap.add_argument("--chunks", type=int, default=0,
                    help="profiling captures only: run the first N chunks of each sequence instead of the full T "
                         "(every launch keeps its full-size shape; the line's config names the reduced T)")
    ap.add_argument("--final-prediction", action="store_true",
                    help="time the forward-only final prediction at fixed fast weights (ttt_predict) instead of "
                         "the inner loop")
    ap.add_argument("--predict-rows", type=int, default=8192,
                    help="rows per sequence in one pass of the final prediction")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    w = I.WORKLOADS[args.workload]
    if args.chunks > 0:
        w = w.with_(T=min(w.T, args.chunks * w.b))
    if args.update_rule != w.update_rule:
        w = w.with_(update_rule=args.update_rule)
    if args.scalars and args.scalars != w.scalars:
        w = w.with_(scalars=args.scalars, name=w.name + "_" + args.scalars)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.final_prediction:
        if w.head != "lm":
            ap.error("--final-prediction needs a next-token workload")
        return run_ours_predict(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
