"""Seeded synthetic inputs for the TTT inner loop.

This module is shared by the CPU oracle's tests, the CUDA parity tests and the
benchmark.  It holds random draws, shapes and the table of workloads, and none
of the method's arithmetic: no forward pass, no loss, no scalar kernel.

The pages train and evaluate on natural text (DCLM, Pile-Books, FineWeb-Edu:
"TTT-E2E：端到端测试时训练的长上下文语言建模", section 训练配置; "Rethinking
Expressivity and Efficiency in Test-Time Training", section 实验环境).  Those
corpora are not used here.  Synthetic inputs with the same shapes stand in for
them:

* hidden rows x ~ N(0, 1), each row divided by its own RMS (the scale a frozen
  backbone's normalised residual stream has);
* tokens uniform over [0, V) for the tiny check, otherwise a truncated
  Zipf(1.1) law P(k) proportional to (k+1)^-1.1 over [0, V), drawn by inverse
  CDF, because natural-text token frequencies are Zipf-like;
* LM head, static MLPs and the initial fast weights W0 ~ N(0, 0.02^2);
* scalars: plain SGD (eta = alpha, beta = 0, gamma = 1) or the E2-TTT draw
  eta = 0.01 * sigmoid(N(0,1)), beta ~ U(0.8, 0.99), gamma ~ U(0.99, 1.0);
  "e2ttt_live" is the same draw with gamma then set to 1 (no decay).  Under
  the plain E2-TTT draw a chunk of 1024 tokens scales the state by a product
  of gammas near 0.006, so over a long sequence W and M decay to zero; with
  gamma = 1 the state keeps its size, which is what an added parity case and
  a live-state timing need.

Draw order (one numpy Generator seeded once): hidden, tokens, LM head, static
weights, W0, M0 (only if requested), eta, beta, gamma.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, Optional

import numpy as np

GELU = "gelu"
SWIGLU = "swiglu"


@dataclass(frozen=True)
class Workload:
    """One inner-loop workload: model shape, sequence shape and scalar recipe."""

    name: str
    d: int
    hidden: int
    vocab: int
    n_blocks: int
    mlp: str  # "gelu" (W1[h,d], W2[d,h]) or "swiglu" (W1 gate[h,d], W2 up[h,d], W3 down[d,h])
    has_static: bool
    precision: str  # "fp32" or "bf16"
    T: int
    b: int
    batch: int
    scalars: str  # "sgd", "e2ttt" or "e2ttt_live" (the e2ttt draw with gamma = 1)
    sgd_lr: float = 0.0
    token_dist: str = "zipf"
    rms_eps: float = 1e-6
    reduction: str = "mean"  # chunk objective: mean (default) or sum of token losses
    update_rule: str = "e2ttt"  # chunk update: "e2ttt" (Proposition 3.1) or "lact" (chunk-wise rule)
    head: str = "lm"  # "lm": next-token cross-entropy; "recon": E2-TTT's key/value reconstruction layer
    attn_heads: int = 0   # > 0: frozen sliding-window attention in front of every updated block
    attn_window: int = 0

    @property
    def n_mats(self) -> int:
        return 2 if self.mlp == GELU else 3

    @property
    def block_params(self) -> int:
        return self.n_mats * self.hidden * self.d

    @property
    def n_chunks(self) -> int:
        return self.T // self.b

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the benchmark, in order.
WORKLOADS: Dict[str, Workload] = {
    # fp32 check: one GELU block, d=64, h=256, V=512, T=256, b=16, SGD alpha=0.1
    "tiny_sgd": Workload("tiny_sgd", 64, 256, 512, 1, GELU, False, "fp32",
                         256, 16, 1, "sgd", 0.1, "uniform"),
    # E2-TTT single GELU block, d=512, h=2048, V=8192, T=4096, b=64
    "e2ttt_block": Workload("e2ttt_block", 512, 2048, 8192, 1, GELU, False, "bf16",
                            4096, 64, 1, "e2ttt"),
    # 3B-class SwiGLU layer, d=3072, h=8192, V=32000, T=32768, b=1024, SGD eta=1e-3
    "sgd_3b": Workload("sgd_3b", 3072, 8192, 32000, 1, SWIGLU, False, "bf16",
                       32768, 1024, 1, "sgd", 1e-3),
    # 128K stack: 4 blocks, static + dynamic SwiGLU each, d=2048, h=5632, V=32000
    "stack_128k": Workload("stack_128k", 2048, 5632, 32000, 4, SWIGLU, True, "bf16",
                           131072, 1024, 1, "e2ttt"),
    # 16 independent sequences, GELU d=1024, h=4096, V=16384, T=8192, b=256
    "batched_16": Workload("batched_16", 1024, 4096, 16384, 1, GELU, False, "bf16",
                           8192, 256, 16, "e2ttt"),
    # E2-TTT's own layer (key/value reconstruction) at the 128K stack's layer
    # dimensions: one SwiGLU fast-weight MLP d=2048, h=5632, T=131072, b=1024
    "e2ttt_layer_128k": Workload("e2ttt_layer_128k", 2048, 5632, 16, 1, SWIGLU, False, "bf16",
                                 131072, 1024, 1, "e2ttt", head="recon"),
    # the 128K stack with frozen sliding-window attention in every block:
    # 32 heads of 64, window 8192 (the pages' k = 8K with b = 1K)
    "stack_128k_swa": Workload("stack_128k_swa", 2048, 5632, 32000, 4, SWIGLU, True, "bf16",
                               131072, 1024, 1, "e2ttt", attn_heads=32, attn_window=8192),
}
WORKLOAD_ORDER = ["tiny_sgd", "e2ttt_block", "sgd_3b", "stack_128k", "batched_16"]


def _normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def zipf_tokens(rng: np.random.Generator, vocab: int, shape, s: float = 1.1) -> np.ndarray:
    """Truncated Zipf(s) over [0, vocab), sampled by inverse CDF."""
    p = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    u = rng.random(size=shape)
    idx = np.searchsorted(cdf, u, side="right")
    return np.minimum(idx, vocab - 1).astype(np.int32)


def make_swa_inputs(w: Workload, seed: int = 0, scale: float = 0.02) -> Dict[str, np.ndarray]:
    """Frozen attention parameters of every updated block, drawn from their own
    generator (seed, 2): attn_w [n_blocks, 4, d, d] (Wq, Wk, Wv, Wo) ~
    N(0, scale^2), LayerNorm gain ~ U(0.8, 1.2) and bias ~ N(0, 0.1^2)
    [n_blocks, d]."""
    rng = np.random.default_rng([seed, 2])
    L, d = w.n_blocks, w.d
    attn_w = _normal(rng, (L, 4, d, d), scale)
    ln_gain = rng.uniform(0.8, 1.2, (L, d)).astype(np.float32)
    ln_bias = _normal(rng, (L, d), 0.1)
    return {"attn_w": attn_w, "ln_gain": ln_gain, "ln_bias": ln_bias}


def make_recon_inputs(w: Workload, seed: int = 0, T: Optional[int] = None, batch: Optional[int] = None,
                      m0_scale: float = 0.0, w0_per_sequence: bool = False) -> Dict[str, np.ndarray]:
    """Inputs of E2-TTT's own layer: everything make_inputs draws (its hidden
    rows serve as the keys K), then values V and queries Q [B,T,d] from a
    second generator seeded (seed, 1), rows scaled to unit RMS like K."""
    x = make_inputs(w, seed, T=T, batch=batch, m0_scale=m0_scale, w0_per_sequence=w0_per_sequence)
    rng = np.random.default_rng([seed, 1])
    B, T_, d = x["hidden"].shape

    def unit_rows():
        a = _normal(rng, (B, T_, d))
        if a.size:
            rms = np.sqrt(np.mean(a.astype(np.float64) ** 2, axis=-1, keepdims=True))
            a = (a / rms).astype(np.float32)
        return a
    x["K"] = x["hidden"]
    x["V"] = unit_rows()
    x["Q"] = unit_rows()
    return x


def make_inputs(w: Workload, seed: int = 0, T: Optional[int] = None,
                batch: Optional[int] = None, m0_scale: float = 0.0,
                w0_per_sequence: bool = False) -> Dict[str, np.ndarray]:
    """Draw every input of one prefill call.

    Returns float32 arrays (int32 tokens) in the layouts the C ABI takes:
    hidden [B,T,d], tokens [B,T] (the label of hidden row t), lm_head [V,d],
    rms_gain [d], static_w [n_blocks * m * h * d] (or None), W0 and M0
    [B * n_blocks * m * h * d] (matrix order W1, W2[, W3], each row-major),
    eta/beta/gamma [B,T].

    ``T``/``batch`` override the workload's sizes (for truncated parity runs).
    ``m0_scale`` > 0 draws a nonzero initial momentum (the workloads use M0=0).
    By default every sequence starts from the same W0 (the model's initial fast
    weights); ``w0_per_sequence`` draws one per sequence instead.
    """
    T = w.T if T is None else T
    B = w.batch if batch is None else batch
    rng = np.random.default_rng(seed)
    d, h, V = w.d, w.hidden, w.vocab

    hidden = _normal(rng, (B, T, d))
    if hidden.size:
        rms = np.sqrt(np.mean(hidden.astype(np.float64) ** 2, axis=-1, keepdims=True))
        hidden = (hidden / rms).astype(np.float32)

    if w.token_dist == "uniform":
        tokens = rng.integers(0, V, size=(B, T), dtype=np.int64).astype(np.int32)
    else:
        tokens = zipf_tokens(rng, V, (B, T))

    lm_head = _normal(rng, (V, d), 0.02)
    rms_gain = np.ones(d, dtype=np.float32)
    static_w = _normal(rng, (w.n_blocks * w.block_params,), 0.02) if w.has_static else None

    per_seq = w.n_blocks * w.block_params
    if w0_per_sequence:
        W0 = _normal(rng, (B * per_seq,), 0.02)
    else:
        W0 = np.tile(_normal(rng, (per_seq,), 0.02), B)
    if m0_scale > 0.0:
        M0 = _normal(rng, (B * per_seq,), m0_scale)
    else:
        M0 = np.zeros(B * per_seq, dtype=np.float32)

    if w.scalars == "sgd":
        eta = np.full((B, T), w.sgd_lr, dtype=np.float32)
        beta = np.zeros((B, T), dtype=np.float32)
        gamma = np.ones((B, T), dtype=np.float32)
    else:
        z = rng.standard_normal(size=(B, T))
        eta = (0.01 / (1.0 + np.exp(-z))).astype(np.float32)
        beta = rng.uniform(0.8, 0.99, size=(B, T)).astype(np.float32)
        gamma = rng.uniform(0.99, 1.0, size=(B, T)).astype(np.float32)
        if w.scalars == "e2ttt_live":
            gamma = np.ones_like(gamma)

    return dict(hidden=hidden, tokens=tokens, lm_head=lm_head, rms_gain=rms_gain,
                static_w=static_w, W0=W0, M0=M0, eta=eta, beta=beta, gamma=gamma)
