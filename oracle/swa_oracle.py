"""CPU oracle of the inner loop with frozen sliding-window attention inside the
updated blocks (the full TTT-E2E block).

TEST INFRASTRUCTURE ONLY, like ttt_oracle: only tests/, the smoke check and
the benchmark's baseline legs may import it; the product path never does.

Pages cited by title:
  [TTT-E2E]  "TTT-E2E：端到端测试时训练的长上下文语言建模"
  [E2-TTT]   "Rethinking Expressivity and Efficiency in Test-Time Training"
  [Review]   "NVIDIA开源TTT-E2E：128K上下文快2.7倍" (PaperDaily review)

What it computes
----------------
* Each updated block is h <- h + Attn(LN(h)), then h <- h + S(h) (the frozen
  static MLP, if any), then h <- h + D_W(h) (the dynamic MLP).  Attention is
  frozen: q, k, v, o projections without biases, a LayerNorm with frozen gain
  and bias in front ([TTT-E2E] the sketch's TTTE2EBlock and TTTSelfAttention;
  the static MLP next to the dynamic one as in [Review] 元学习 section).
* Rotary position embedding of q and k in the rotate-half form, angle
  pos * base^(-2i/d_head), base 10000 ([TTT-E2E] the sketch's RotaryEmbedding),
  at absolute sequence positions.
* Scores q.k / sqrt(d_head), softmax over the keys inside the window
  ([TTT-E2E] 滑动窗口注意力; window k = 8K, chunk b = 1K, k >= b in
  关键设计参数).
* A chunk's tokens attend to earlier chunks' keys and values inside the
  window; those were computed when their own chunk ran (at that chunk's
  start weights) and are constants for the current chunk's gradient.

Readings where the pages leave a step open (the sketch's mask is
|i - j| <= k/2, two-sided, which would let a token see its own label):
  * causal window: query t sees keys j with 0 <= t - j < k;
  * no attention biases (the MLP reading of ttt_oracle drops biases too);
  * the block order attention, static MLP, dynamic MLP.

Why the update needs weighted backward passes here
--------------------------------------------------
Without attention each token's loss depends on its own row only, so one
backward of sum_t l_t yields every G_t as a factor pair of row t and the
scalar kernels can weight the rows afterwards (ttt_oracle.chunk_backward).
Attention mixes the rows of a chunk: l_t depends on the lower blocks' rows of
earlier tokens too.  Proposition 3.1 needs only the sums sum_t K_t G_t, and
by linearity of the gradient sum_t K_t grad l_t = grad (sum_t K_t l_t).  The
oracle therefore runs one backward of the K_W-weighted and one of the
K_M-weighted chunk loss (a single one when the weights coincide, as under
LaCT's rule).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np

from .ttt_oracle import (Model, mlp_backward, mlp_forward, pack_blocks, scalar_kernels, unpack_blocks)


@dataclass
class Swa:
    """Frozen attention of every updated block: Wq, Wk, Wv, Wo [d, d] each and
    the LayerNorm gain and bias [d], one entry per block."""

    n_heads: int
    window: int
    Wq: List[np.ndarray]
    Wk: List[np.ndarray]
    Wv: List[np.ndarray]
    Wo: List[np.ndarray]
    ln_gain: List[np.ndarray]
    ln_bias: List[np.ndarray]
    ln_eps: float = 1e-5
    rope_base: float = 10000.0

    def astype(self, dtype) -> "Swa":
        c = lambda xs: [x.astype(dtype) for x in xs]
        return Swa(self.n_heads, self.window, c(self.Wq), c(self.Wk), c(self.Wv), c(self.Wo),
                   c(self.ln_gain), c(self.ln_bias), self.ln_eps, self.rope_base)


def make_swa(d, n_blocks, n_heads, window, attn_w, ln_gain, ln_bias, ln_eps=1e-5, dtype=np.float64) -> Swa:
    """attn_w [n_blocks, 4, d, d] (Wq, Wk, Wv, Wo); ln_gain, ln_bias [n_blocks, d]."""
    A = np.asarray(attn_w, dtype=dtype).reshape(n_blocks, 4, d, d)
    g = np.asarray(ln_gain, dtype=dtype).reshape(n_blocks, d)
    bb = np.asarray(ln_bias, dtype=dtype).reshape(n_blocks, d)
    return Swa(n_heads, window, [A[l, 0] for l in range(n_blocks)], [A[l, 1] for l in range(n_blocks)],
               [A[l, 2] for l in range(n_blocks)], [A[l, 3] for l in range(n_blocks)],
               [g[l] for l in range(n_blocks)], [bb[l] for l in range(n_blocks)], ln_eps)


# ---------------------------------------------------------------------------
# Pieces: LayerNorm with gain and bias, rotary embedding
# ---------------------------------------------------------------------------

def layer_norm_affine(x, gain, bias, eps):
    mu = x.mean(axis=-1, keepdims=True)
    xc = x - mu
    rs = 1.0 / np.sqrt((xc * xc).mean(axis=-1, keepdims=True) + eps)
    xhat = xc * rs
    return xhat * gain + bias, (xhat, rs)


def layer_norm_affine_backward(g, cache, gain):
    """Gradient w.r.t. the input of layer_norm_affine (gain and bias frozen)."""
    xhat, rs = cache
    gh = g * gain
    return rs * (gh - gh.mean(axis=-1, keepdims=True) - xhat * (gh * xhat).mean(axis=-1, keepdims=True))


def rope_angles(pos, d_head, base):
    """cos, sin [n, d_head]: angle pos * base^(-2i/d_head), repeated for both halves."""
    inv = base ** (-np.arange(0, d_head, 2, dtype=np.float64) / d_head)
    f = np.outer(np.asarray(pos, dtype=np.float64), inv)
    f = np.concatenate([f, f], axis=1)
    return np.cos(f), np.sin(f)


def rope(x, cos, sin):
    """Rotate-half form on the last axis: (x1, x2) -> (x1 c - x2 s, x1 s + x2 c)."""
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    c, s = cos[..., :h], sin[..., :h]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def rope_backward(g, cos, sin):
    """Transpose of the rotation (rotation by the negative angle)."""
    h = g.shape[-1] // 2
    g1, g2 = g[..., :h], g[..., h:]
    c, s = cos[..., :h], sin[..., :h]
    return np.concatenate([g1 * c + g2 * s, -g1 * s + g2 * c], axis=-1)


def window_mask(qpos, kpos, window):
    """Key j is visible to query t when 0 <= t - j < window."""
    delta = np.asarray(qpos)[:, None] - np.asarray(kpos)[None, :]
    return (delta >= 0) & (delta < window)


# ---------------------------------------------------------------------------
# Attention sub-layer of block l for one chunk of one sequence
# ---------------------------------------------------------------------------

def empty_kv(sw: Swa, d: int, dtype=np.float64):
    dh = d // sw.n_heads
    z = np.zeros((sw.n_heads, 0, dh), dtype=dtype)
    return (z, z.copy(), np.zeros(0, dtype=np.int64))


def attention_forward(sw: Swa, l: int, h, pos, kv_prev):
    """Returns (out [n, d], cache, (k_rot, v, pos)) for rows h at positions pos;
    kv_prev = (K [H, m, dh] rotated, V [H, m, dh], positions [m]) of earlier tokens."""
    n, d = h.shape
    H = sw.n_heads
    dh = d // H
    a, lnc = layer_norm_affine(h, sw.ln_gain[l], sw.ln_bias[l], sw.ln_eps)
    heads = lambda m: (a @ m.T).reshape(n, H, dh).transpose(1, 0, 2)
    q, k, v = heads(sw.Wq[l]), heads(sw.Wk[l]), heads(sw.Wv[l])
    cos, sin = rope_angles(pos, dh, sw.rope_base)
    cos, sin = cos.astype(h.dtype), sin.astype(h.dtype)
    qr, kr = rope(q, cos, sin), rope(k, cos, sin)
    Kp, Vp, ppos = kv_prev
    Ka = np.concatenate([Kp, kr], axis=1)
    Va = np.concatenate([Vp, v], axis=1)
    kpos = np.concatenate([ppos, np.asarray(pos)])
    mask = window_mask(pos, kpos, sw.window)
    s = (qr @ Ka.transpose(0, 2, 1)) / np.sqrt(dh)
    s = np.where(mask[None], s, -np.inf)
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    p = p / p.sum(axis=-1, keepdims=True)
    o = p @ Va
    oc = o.transpose(1, 0, 2).reshape(n, d)
    out = oc @ sw.Wo[l].T
    cache = (lnc, qr, Ka, Va, p, o, cos, sin, Kp.shape[1])
    return out, cache, (kr, v, np.asarray(pos))


def attention_backward(sw: Swa, l: int, cache, g_out):
    """Gradient w.r.t. the sub-layer's input rows; earlier tokens' keys and
    values are constants."""
    lnc, qr, Ka, Va, p, o, cos, sin, mprev = cache
    n, d = g_out.shape
    H = sw.n_heads
    dh = d // H
    do = (g_out @ sw.Wo[l]).reshape(n, H, dh).transpose(1, 0, 2)
    dp = do @ Va.transpose(0, 2, 1)
    D = np.sum(do * o, axis=-1, keepdims=True)
    ds = p * (dp - D) / np.sqrt(dh)
    dq = rope_backward(ds @ Ka, cos, sin)
    dk = rope_backward((ds.transpose(0, 2, 1) @ qr)[:, mprev:], cos, sin)
    dv = (p.transpose(0, 2, 1) @ do)[:, mprev:]
    flat = lambda x: x.transpose(1, 0, 2).reshape(n, d)
    da = flat(dq) @ sw.Wq[l] + flat(dk) @ sw.Wk[l] + flat(dv) @ sw.Wv[l]
    return layer_norm_affine_backward(da, lnc, sw.ln_gain[l])


# ---------------------------------------------------------------------------
# One chunk: forward at the chunk-start weights, weighted backward
# ---------------------------------------------------------------------------

def chunk_forward(model: Model, sw: Swa, W, X, y, pos0: int, kv):
    """Per-token losses of the chunk rows X [n, d] (positions pos0..pos0+n-1)
    at weights W; kv[l] holds block l's earlier keys and values.  Returns
    (loss [n], fwd, new_kv)."""
    n = X.shape[0]
    pos = np.arange(pos0, pos0 + n)
    caches, new_kv = [], []
    h = X
    for l in range(model.n_blocks):
        out, c, nkv = attention_forward(sw, l, h, pos, kv[l])
        caches.append(("attn", l, c))
        new_kv.append(nkv)
        h = h + out
        if model.static is not None:
            out, c = mlp_forward(model.mlp, model.static[l], h)
            caches.append(("static", l, c))
            h = h + out
        out, c = mlp_forward(model.mlp, W[l], h)
        caches.append(("dynamic", l, c))
        h = h + out
    ms = np.mean(h * h, axis=1)
    r = 1.0 / np.sqrt(ms + model.rms_eps)
    z = h * r[:, None] * model.rms_gain[None, :]
    logits = z @ model.lm_head.T
    mx = logits.max(axis=1)
    lse = mx + np.log(np.sum(np.exp(logits - mx[:, None]), axis=1))
    loss = lse - logits[np.arange(n), y]
    return loss, (caches, h, r, logits, lse), new_kv


def weighted_backward(model: Model, sw: Swa, W, y, fwd, weight):
    """grad_W of sum_t weight_t l_t for every dynamic matrix (dense, [l][j]).

    The backward stops at the lowest dynamic MLP: what lies below it (block
    0's static MLP and attention) reads only the frozen hidden rows."""
    caches, h, r, logits, lse = fwd
    n = h.shape[0]
    p = np.exp(logits - lse[:, None])
    p[np.arange(n), y] -= 1.0
    p *= np.asarray(weight, dtype=p.dtype)[:, None]
    gdz = (p @ model.lm_head) * model.rms_gain[None, :]
    dot = np.sum(gdz * h, axis=1)
    dh = gdz * r[:, None] - h * (r ** 3 * dot / model.d)[:, None]
    grads: List[Optional[List[np.ndarray]]] = [None] * model.n_blocks
    for kind, l, cache in reversed(caches):
        if kind == "attn":
            dh = dh + attention_backward(sw, l, cache, dh)
            continue
        mats = model.static[l] if kind == "static" else W[l]
        dx, pairs = mlp_backward(model.mlp, mats, cache, dh)
        if kind == "dynamic":
            grads[l] = [Lf.T @ Rf for (Lf, Rf) in pairs]
            if l == 0:
                break
        dh = dh + dx
    return grads


def rule_coefficients(rule: str, eta, beta, gamma):
    """(K_W, K_M, coefficient of W_0 in W_C, of M_0 in M_C, of M_0 in W_C)."""
    if rule == "lact":
        bbar = float(np.mean(np.asarray(beta, dtype=np.float64)))
        e = np.asarray(eta, dtype=np.float64)
        return e, e, 1.0, bbar, bbar
    return scalar_kernels(eta, beta, gamma)


def prefill_sequence(model: Model, sw: Swa, W0, M0, hidden, tokens, eta, beta, gamma, b,
                     rule: str = "e2ttt", reduction: str = "mean", n_chunks: Optional[int] = None,
                     pos0: int = 0, kv_in=None, return_kv: bool = False):
    """Chunk-serial inner loop of one sequence with attention in the blocks.
    Returns (W, M, chunk_loss [n_chunks]), and the key/value history too with
    return_kv.  To resume a sequence, pass the rows from position pos0 on, the
    state reached there and its history as kv_in."""
    gscale = 1.0 / b if reduction == "mean" else 1.0
    T, d = hidden.shape
    if T % b:
        raise ValueError("T must be a multiple of b")
    nc = T // b if n_chunks is None else n_chunks
    W = [[m.copy() for m in blk] for blk in W0]
    M = [[m.copy() for m in blk] for blk in M0]
    kv = list(kv_in) if kv_in is not None else [empty_kv(sw, d, hidden.dtype) for _ in range(model.n_blocks)]
    losses = np.zeros(nc)
    for c in range(nc):
        s = slice(c * b, (c + 1) * b)
        loss, fwd, new_kv = chunk_forward(model, sw, W, hidden[s], tokens[s], pos0 + c * b, kv)
        losses[c] = float(np.mean(loss))
        KW, KM, g0, b0, cM = rule_coefficients(rule, eta[s], beta[s], gamma[s])
        gW = weighted_backward(model, sw, W, tokens[s], fwd, KW)
        gM = gW if np.array_equal(KW, KM) else weighted_backward(model, sw, W, tokens[s], fwd, KM)
        dt = W[0][0].dtype
        W = [[(dt.type(g0) * W[l][j] + dt.type(cM) * M[l][j] - gscale * gW[l][j]).astype(dt)
              for j in range(len(W[l]))] for l in range(model.n_blocks)]
        M = [[(dt.type(b0) * M[l][j] - gscale * gM[l][j]).astype(dt) for j in range(len(M[l]))]
             for l in range(model.n_blocks)]
        for l in range(model.n_blocks):      # this chunk's keys and values join the window
            kr, v, p = new_kv[l]
            K0, V0, p0 = kv[l]
            kv[l] = (np.concatenate([K0, kr], axis=1), np.concatenate([V0, v], axis=1),
                     np.concatenate([p0, p]))
    if return_kv:
        return W, M, losses, kv
    return W, M, losses


def prefill(model: Model, sw: Swa, W0_flat, M0_flat, hidden, tokens, eta, beta, gamma, b,
            dtype=np.float64, rule: str = "e2ttt", reduction: str = "mean", n_chunks: Optional[int] = None):
    """Batched form with the C ABI's flat layouts (as ttt_oracle.prefill)."""
    mdl = model.astype(dtype)
    s_w = sw.astype(dtype)
    B = hidden.shape[0]
    shapes = mdl.mat_shapes()
    per_seq = mdl.n_blocks * sum(r * c for r, c in shapes)
    W0_flat = np.asarray(W0_flat, dtype=dtype).reshape(B, per_seq)
    M0_flat = np.asarray(M0_flat, dtype=dtype).reshape(B, per_seq)
    Ws, Ms, Ls = [], [], []
    for s in range(B):
        W0 = unpack_blocks(W0_flat[s].copy(), mdl.n_blocks, shapes)
        M0 = unpack_blocks(M0_flat[s].copy(), mdl.n_blocks, shapes)
        W, M, L = prefill_sequence(mdl, s_w, W0, M0, np.asarray(hidden[s], dtype=dtype), np.asarray(tokens[s]),
                                   eta[s], beta[s], gamma[s], b, rule=rule, reduction=reduction,
                                   n_chunks=n_chunks)
        Ws.append(pack_blocks(W))
        Ms.append(pack_blocks(M))
        Ls.append(L)
    return np.concatenate(Ws), np.concatenate(Ms), np.stack(Ls)


def final_prediction(model: Model, sw: Swa, W_flat, hidden, tokens, b, dtype=np.float64):
    """Forward-only pass of whole sequences at fixed fast weights with the
    attention blocks ([TTT-E2E] 持续学习框架, the 预测 step, and the sketch's
    最终预测 part): the rows are processed b at a time, and every key and value
    in the window is computed at the same weights W, so the result does not
    depend on b.  Returns (token_loss [B,T], group_loss [B, T // b]) as
    ttt_oracle.final_prediction does."""
    mdl = model.astype(dtype)
    s_w = sw.astype(dtype)
    B, T = np.asarray(tokens).shape
    if T % b:
        raise ValueError("T must be a multiple of b")
    shapes = mdl.mat_shapes()
    per_seq = mdl.n_blocks * sum(r * c for r, c in shapes)
    Wf = np.asarray(W_flat, dtype=dtype).reshape(B, per_seq)
    tok = np.zeros((B, T), dtype=dtype)
    for s_ in range(B):
        W = unpack_blocks(Wf[s_].copy(), mdl.n_blocks, shapes)
        X = np.asarray(hidden[s_], dtype=dtype)
        kv = [empty_kv(s_w, mdl.d, dtype) for _ in range(mdl.n_blocks)]
        for c in range(T // b):
            sl = slice(c * b, (c + 1) * b)
            loss, _, new_kv = chunk_forward(mdl, s_w, W, X[sl], np.asarray(tokens[s_])[sl], c * b, kv)
            tok[s_, sl] = loss
            kv = [(np.concatenate([kv[l][0], new_kv[l][0]], axis=1), np.concatenate([kv[l][1], new_kv[l][1]], axis=1),
                   np.concatenate([kv[l][2], new_kv[l][2]])) for l in range(mdl.n_blocks)]
    return tok, tok.reshape(B, -1, b).mean(axis=2)
