"""CPU oracle for the TTT-E2E inner loop with the E2-TTT closed-form chunk update.

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check in __graft_entry__ and
the benchmark's cpu_baseline / reference leg may import or run this module.
The product path (the CUDA library and its Python binding) never imports it
and shares no code with it.

What it computes, and where the pages define it
-----------------------------------------------
Pages cited by title:
  [TTT-E2E]  "TTT-E2E：端到端测试时训练的长上下文语言建模"
  [E2-TTT]   "Rethinking Expressivity and Efficiency in Test-Time Training"
  [Review]   "NVIDIA开源TTT-E2E：128K上下文快2.7倍" (PaperDaily review)

* The inner loop walks the sequence in chunks of b tokens; every token of a
  chunk is predicted with the chunk-start weights and contributes its
  next-token cross-entropy ([TTT-E2E] 内层循环：测试时训练; [E2-TTT]
  高效的逐块更新机制, O^[r] = f_{W^[r-1]}(Q^[r])).
* Only MLPs of the last blocks are updated; embedding, norms and attention
  are frozen; an updated block may carry a frozen "static" MLP next to the
  dynamic one ([Review] 元学习 section, dual-MLP paragraph).
* Fast-weight MLP forms: GELU  y = W2 GELU(W1 x),  SwiGLU  y = W3 (SiLU(W1 x)
  * (W2 x)), with a residual x + y ([E2-TTT] 快速权重网络实例化).  Reading: no
  norm inside the block and no biases.
* Frozen RMSNorm + LM head give the next-token loss ([TTT-E2E] 核心方法,
  the loss l_t is next-token prediction).
* G_t is the NEGATIVE gradient of token t's loss at the chunk-start weights;
  the per-token recursion is M_t = beta_t M_{t-1} + eta_t G_t,
  W_t = gamma_t W_{t-1} + M_t ([E2-TTT] 原始公式).
* The chunk-end state follows Proposition 3.1 ([E2-TTT] 命题3.1):
  M_C = btilde_0 M_0 + sum_t eta_t btilde_t G_t,
  W_C = gtilde_0 W_0 + btilde_0 R_1 M_0 + sum_t eta_t btilde_t R_t G_t,
  with suffix products btilde_t = prod_{i>t} beta_i, gtilde_t = prod_{i>t}
  gamma_i and R_t = sum_{i>=t} gtilde_i / btilde_i.
* After the inner loop the whole sequence is scored again at the final
  weights W_T, forward only ([TTT-E2E] 持续学习框架, 预测 step; the sketch's
  最终预测 part), per token and per group of b positions ([Review] 图6).

Readings where the pages leave a step open:
  * tokens[t] is the label of hidden row t (the caller pre-shifts);
  * the chunk objective is the MEAN next-token loss over the chunk (the default
    reduction of the first inner-loop sketch on [TTT-E2E]); the per-token loss
    entering the recursion is therefore l_t / b, so that with beta = 0,
    gamma = 1, eta_t = alpha one chunk is one mini-batch gradient step on the
    chunk's mean loss, and b = 1 is plain online SGD.  reduction="sum" (the
    second sketch's reduction='sum') uses l_t itself.  The reported chunk loss
    is the mean of the b token losses at chunk-start weights either way;
  * RMSNorm: z = g * h / sqrt(mean(h^2) + eps), computed per row;
  * GELU is the exact erf form; SiLU(x) = x sigmoid(x);
  * the coefficients eta_t btilde_t R_t and btilde_0 R_1 are evaluated in the
    division-free form the expanded equation of Proposition 3.1 gives
    (sum over j of prod beta * gtilde_j), which equals the ratio form
    wherever btilde > 0 and stays finite where a beta is 0.

Parity pins (tests/test_oracle_*.py) tie every function here to something
other than itself: exact-rational recursion, finite differences, torch
autograd, closed forms of cross-entropy, the SGD reduction, resume and
linearity.  No function here is "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np
from scipy.special import erf, expit

GELU = "gelu"
SWIGLU = "swiglu"


# ---------------------------------------------------------------------------
# Elementwise functions ([E2-TTT] 快速权重网络实例化; [TTT-E2E] nn.GELU)
# ---------------------------------------------------------------------------

def gelu(x):
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def gelu_grad(x):
    cdf = 0.5 * (1.0 + erf(x / math.sqrt(2.0)))
    pdf = np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
    return cdf + x * pdf


def sigmoid(x):
    # the logistic function from the library: no overflow of exp(-x) for large negative x
    return expit(x)


def silu(x):
    return x * sigmoid(x)


def silu_grad(x):
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


# ---------------------------------------------------------------------------
# Model description and weight packing
# ---------------------------------------------------------------------------

@dataclass
class Model:
    """Frozen parts of the model plus the shapes of the fast weights.

    lm_head E [V, d]; rms_gain g [d]; static[l] = list of the block's frozen
    MLP matrices (same kind and shape as the dynamic MLP) or None.
    """

    d: int
    hidden: int
    vocab: int
    n_blocks: int
    mlp: str
    rms_eps: float
    lm_head: np.ndarray
    rms_gain: np.ndarray
    static: Optional[List[List[np.ndarray]]] = None

    @property
    def n_mats(self) -> int:
        return 2 if self.mlp == GELU else 3

    def mat_shapes(self) -> List[Tuple[int, int]]:
        d, h = self.d, self.hidden
        if self.mlp == GELU:
            return [(h, d), (d, h)]
        return [(h, d), (h, d), (d, h)]

    def astype(self, dtype) -> "Model":
        st = None
        if self.static is not None:
            st = [[m.astype(dtype) for m in blk] for blk in self.static]
        return Model(self.d, self.hidden, self.vocab, self.n_blocks, self.mlp,
                     self.rms_eps, self.lm_head.astype(dtype),
                     self.rms_gain.astype(dtype), st)


def unpack_blocks(flat: np.ndarray, n_blocks: int, shapes) -> List[List[np.ndarray]]:
    """Flat [n_blocks][m] row-major matrices -> nested list (views)."""
    out, off = [], 0
    for _ in range(n_blocks):
        blk = []
        for (r, c) in shapes:
            blk.append(flat[off:off + r * c].reshape(r, c))
            off += r * c
        out.append(blk)
    assert off == flat.size, (off, flat.size)
    return out


def pack_blocks(blocks: List[List[np.ndarray]]) -> np.ndarray:
    return np.concatenate([m.reshape(-1) for blk in blocks for m in blk])


def make_model(d, hidden, vocab, n_blocks, mlp, rms_eps, lm_head, rms_gain,
               static_w=None, dtype=np.float64) -> Model:
    m = Model(d, hidden, vocab, n_blocks, mlp, rms_eps,
              np.asarray(lm_head, dtype=dtype), np.asarray(rms_gain, dtype=dtype))
    if static_w is not None:
        m.static = unpack_blocks(np.asarray(static_w, dtype=dtype), n_blocks, m.mat_shapes())
    return m


# ---------------------------------------------------------------------------
# Forward and per-token backward at fixed (chunk-start) weights
# ---------------------------------------------------------------------------

def mlp_forward(kind: str, mats: Sequence[np.ndarray], x: np.ndarray):
    """y = MLP(x) for rows x [n, d]; returns (y, cache)."""
    if kind == GELU:
        W1, W2 = mats
        U = x @ W1.T
        A = gelu(U)
        return A @ W2.T, (x, U, A)
    W1, W2, W3 = mats
    Ug = x @ W1.T
    Uu = x @ W2.T
    A = silu(Ug) * Uu
    return A @ W3.T, (x, Ug, Uu, A)


def mlp_backward(kind: str, mats, cache, d_out: np.ndarray):
    """Backward of y = MLP(x) given dL/dy rows.

    Returns (dL/dx through the MLP branch only, per-matrix factor pairs) where
    the per-token gradient of matrix j is outer(L_j[t], R_j[t]).
    """
    if kind == GELU:
        W1, W2 = mats
        x, U, A = cache
        dA = d_out @ W2
        dU = dA * gelu_grad(U)
        return dU @ W1, [(dU, x), (d_out, A)]
    W1, W2, W3 = mats
    x, Ug, Uu, A = cache
    dA = d_out @ W3
    dUg = dA * Uu * silu_grad(Ug)
    dUu = dA * silu(Ug)
    return dUg @ W1 + dUu @ W2, [(dUg, x), (dUu, x), (d_out, A)]


def chunk_forward(model: Model, W: List[List[np.ndarray]], X: np.ndarray, y: np.ndarray):
    """Per-token losses l_t at weights W for rows X [n, d] with labels y [n].

    Block l applies h <- h + S_l(h) (if a static MLP exists), then
    h <- h + D_l(h); then z = RMSNorm(h), logits = z E^T,
    l_t = logsumexp(logits_t) - logits_t[y_t].
    """
    caches = []
    h = X
    for l in range(model.n_blocks):
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
    rows = np.arange(X.shape[0])
    loss = lse - logits[rows, y]
    return loss, (caches, h, r, logits, lse)


def chunk_backward(model: Model, W, y, fwd):
    """Per-token gradient factors of every dynamic matrix.

    Returns grads[l][j] = (L, R) with dl_t/dW_{l,j} = outer(L[t], R[t]).
    Each token's loss depends only on its own row, so one batched backward of
    sum_t l_t yields every per-token gradient ([E2-TTT] 单次反向传播的链式法则分解).
    """
    caches, h, r, logits, lse = fwd
    n = h.shape[0]
    p = np.exp(logits - lse[:, None])
    p[np.arange(n), y] -= 1.0                       # dl/dlogits
    dz = p @ model.lm_head                          # dl/dz
    gdz = dz * model.rms_gain[None, :]
    d = model.d
    dot = np.sum(gdz * h, axis=1)
    dh = gdz * r[:, None] - h * (r ** 3 * dot / d)[:, None]   # RMSNorm backward

    grads: List[List] = [None] * model.n_blocks
    for kind, l, cache in reversed(caches):
        mats = model.static[l] if kind == "static" else W[l]
        dx_branch, pairs = mlp_backward(model.mlp, mats, cache, dh)
        if kind == "dynamic":
            grads[l] = pairs
        dh = dh + dx_branch                         # residual
    return grads


# ---------------------------------------------------------------------------
# Scalar kernels ([E2-TTT] 定义高效后缀乘积与比例和, 命题3.1)
# ---------------------------------------------------------------------------

def suffix_products(v: np.ndarray) -> np.ndarray:
    """out[t] = prod_{i=t+1}^{C} v_i for t = 0..C (1-indexed v), out[C] = 1."""
    C = v.shape[0]
    out = np.ones(C + 1, dtype=np.float64)
    for t in range(C - 1, -1, -1):
        out[t] = out[t + 1] * float(v[t])
    return out


def scalar_kernels(eta, beta, gamma):
    """Coefficients of Proposition 3.1 for one chunk of length C.

    Inputs are the chunk's eta, beta, gamma (0-based arrays; entry k is token
    t = k + 1).  Returns (K_W [C], K_M [C], gtilde_0, btilde_0, c_M) with
      K_M_t = eta_t btilde_t,
      K_W_t = eta_t btilde_t R_t = eta_t sum_{j=t}^{C} (prod_{i=t+1}^{j} beta_i) gtilde_j,
      c_M   = btilde_0 R_1       = sum_{j=1}^{C} (prod_{i=1}^{j} beta_i) gtilde_j,
    i.e. the gradient and momentum terms of the expanded chunk-end equation
    (the one printed just before the definitions of btilde, gtilde, R).
    Evaluated in float64.
    """
    eta = np.asarray(eta, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    gamma = np.asarray(gamma, dtype=np.float64)
    C = eta.shape[0]
    bt = suffix_products(beta)    # bt[k] = btilde_k, k = 0..C
    gt = suffix_products(gamma)   # gt[k] = gtilde_k
    KM = eta * bt[1:]
    KW = np.empty(C, dtype=np.float64)
    for k in range(C):            # token t = k+1
        # prod_{i=t+1}^{j} beta_i for j = t..C  ->  cumprod of beta[k+1:], with 1 for j = t
        run = np.concatenate(([1.0], np.cumprod(beta[k + 1:])))
        KW[k] = eta[k] * np.sum(run * gt[k + 1:])
    run0 = np.cumprod(beta)       # prod_{i=1}^{j} beta_i, j = 1..C
    cM = float(np.sum(run0 * gt[1:]))
    return KW, KM, float(gt[0]), float(bt[0]), cM


def scalar_heads(X, heads, bias, eta_base, alpha_base, tau):
    """Input-dependent update scalars ([E2-TTT] 依赖于输入的动态参数化):
      eta_t   = eta_base * sigmoid(w_eta . x_t + b_eta),
      beta_t  = sigmoid(w_beta . x_t + b_beta) ** (1 / tau),
      alpha_t = alpha_base * sigmoid(w_alpha . x_t + b_alpha),
      gamma_t = 1 - eta_t * alpha_t.
    X [..., d]; heads [3, d] rows (w_eta, w_beta, w_alpha); bias [3].
    Reading: each Linear has a bias.  Evaluated in float64."""
    X = np.asarray(X, dtype=np.float64)
    Wh = np.asarray(heads, dtype=np.float64)
    bh = np.asarray(bias, dtype=np.float64)
    z = X @ Wh.T + bh                     # [..., 3]
    sig = 1.0 / (1.0 + np.exp(-z))
    eta = eta_base * sig[..., 0]
    beta = sig[..., 1] ** (1.0 / tau)
    alpha = alpha_base * sig[..., 2]
    gamma = 1.0 - eta * alpha
    return eta, beta, gamma


def scalar_kernels_ratio_form(eta, beta, gamma):
    """The same coefficients through R_t = sum_{i>=t} gtilde_i / btilde_i.

    This is the form printed in the definitions; it divides by btilde and is
    only defined where every btilde_i > 0.  Kept for the pins.
    """
    eta = np.asarray(eta, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    gamma = np.asarray(gamma, dtype=np.float64)
    C = eta.shape[0]
    bt = suffix_products(beta)
    gt = suffix_products(gamma)
    R = np.array([np.sum(gt[t:C + 1] / bt[t:C + 1]) for t in range(1, C + 1)])  # R_1..R_C
    KW = eta * bt[1:] * R
    KM = eta * bt[1:]
    return KW, KM, float(gt[0]), float(bt[0]), float(bt[0] * R[0])


# ---------------------------------------------------------------------------
# Chunk update: closed form (Prop. 3.1 / Algorithm 1) and explicit recursion
# ---------------------------------------------------------------------------

def chunk_update_closed(W, M, grads, eta, beta, gamma, gscale=1.0):
    """Algorithm 1, the scalar-kernel and update steps: aggregate with K_W and K_M, then
    W_C = gtilde_0 W_0 + btilde_0 R_1 M_0 + dW and M_C = btilde_0 M_0 + dM.

    G_t = -gscale * outer(L[t], R[t]) (gscale = 1/b for the mean reduction),
    so sum_t K_t G_t = -gscale (K * L)^T R.
    """
    KW, KM, g0, b0, cM = scalar_kernels(eta, beta, gamma)
    dt = W[0][0].dtype
    KW = (KW * gscale).astype(dt)
    KM = (KM * gscale).astype(dt)
    newW, newM = [], []
    for l in range(len(W)):
        bw, bm = [], []
        for j in range(len(W[l])):
            Lf, Rf = grads[l][j]
            dW = -((Lf * KW[:, None]).T @ Rf)
            dM = -((Lf * KM[:, None]).T @ Rf)
            bw.append((dt.type(g0) * W[l][j] + dt.type(cM) * M[l][j] + dW).astype(dt))
            bm.append((dt.type(b0) * M[l][j] + dM).astype(dt))
        newW.append(bw)
        newM.append(bm)
    return newW, newM


def chunk_update_explicit(W, M, grads, eta, beta, gamma, gscale=1.0):
    """The per-token recursion itself ([E2-TTT] 原始公式), with every G_t
    materialised:  M_t = beta_t M_{t-1} + eta_t G_t,  W_t = gamma_t W_{t-1} + M_t."""
    newW, newM = [], []
    C = len(eta)
    for l in range(len(W)):
        bw, bm = [], []
        for j in range(len(W[l])):
            Lf, Rf = grads[l][j]
            Wt = W[l][j].copy()
            Mt = M[l][j].copy()
            for k in range(C):
                G = -gscale * np.outer(Lf[k], Rf[k])
                Mt = beta[k] * Mt + eta[k] * G
                Wt = gamma[k] * Wt + Mt
            bw.append(Wt)
            bm.append(Mt)
        newW.append(bw)
        newM.append(bm)
    return newW, newM


def chunk_update_lact(W, M, grads, eta, beta, gamma, gscale=1.0):
    """LaCT's chunk-wise rule ([E2-TTT] 高效的逐块（Chunk-wise）更新机制): a single
    update direction for the chunk, the negative gradient of the eta-weighted
    sum of the token losses at the chunk-start weights,
      G = -grad sum_t eta_t l_t = sum_t eta_t G_t,
    a momentum factor averaged over the chunk, and no decay:
      M_C = (1/C sum_t beta_t) M_0 + G,   W_C = W_0 + M_C.
    gamma is not used by this rule."""
    bbar = float(np.mean(np.asarray(beta, dtype=np.float64)))
    e = np.asarray(eta, dtype=np.float64)
    newW, newM = [], []
    for l in range(len(W)):
        bw, bm = [], []
        for j in range(len(W[l])):
            Lf, Rf = grads[l][j]
            dt = W[l][j].dtype
            G = (-gscale * ((Lf * e[:, None].astype(Lf.dtype)).T @ Rf)).astype(dt)
            Mn = (dt.type(bbar) * M[l][j] + G).astype(dt)
            bw.append((W[l][j] + Mn).astype(dt))
            bm.append(Mn)
        newW.append(bw)
        newM.append(bm)
    return newW, newM


UPDATE_RULES = ("closed", "explicit", "lact")


# ---------------------------------------------------------------------------
# The inner loop over a whole sequence
# ---------------------------------------------------------------------------

def prefill_sequence(model: Model, W0, M0, hidden, tokens, eta, beta, gamma, b,
                     update: str = "closed", n_chunks: Optional[int] = None,
                     reduction: str = "mean"):
    """Chunk-serial inner loop for one sequence.

    W0, M0: nested lists [n_blocks][m] of matrices; hidden [T, d]; tokens [T];
    eta/beta/gamma [T].  Returns (W_final, M_final, chunk_loss [n_chunks]).
    ``n_chunks`` limits the run to the first chunks (for sampled parity).
    ``reduction``: "mean" (per-token loss l_t / b) or "sum" (l_t).
    """
    if reduction not in ("mean", "sum"):
        raise ValueError("reduction must be 'mean' or 'sum'")
    gscale = 1.0 / b if reduction == "mean" else 1.0
    T = hidden.shape[0]
    if T % b != 0:
        raise ValueError("T must be a multiple of b")
    nc = T // b if n_chunks is None else n_chunks
    W = [[m.copy() for m in blk] for blk in W0]
    M = [[m.copy() for m in blk] for blk in M0]
    losses = np.zeros(nc, dtype=np.float64)
    if update not in UPDATE_RULES:
        raise ValueError("update must be one of " + ", ".join(UPDATE_RULES))
    # looked up at call time (the pins substitute planted mistakes)
    step = {"closed": chunk_update_closed, "explicit": chunk_update_explicit, "lact": chunk_update_lact}[update]
    for c in range(nc):
        s = slice(c * b, (c + 1) * b)
        X = hidden[s]
        y = tokens[s]
        loss, fwd = chunk_forward(model, W, X, y)     # forward at the chunk-start weights
        losses[c] = float(np.mean(loss))
        grads = chunk_backward(model, W, y, fwd)      # one backward for the whole chunk
        W, M = step(W, M, grads, eta[s], beta[s], gamma[s], gscale)
    return W, M, losses


def prefill(model: Model, W0_flat, M0_flat, hidden, tokens, eta, beta, gamma, b,
            dtype=np.float64, update: str = "closed", n_chunks: Optional[int] = None,
            reduction: str = "mean"):
    """Batched inner loop with the C-ABI's flat layouts.

    hidden [B,T,d], tokens [B,T], eta/beta/gamma [B,T],
    W0_flat / M0_flat [B * n_blocks * m * h * d].
    Returns (W_flat, M_flat, chunk_loss [B, n_chunks]) in ``dtype``.
    """
    mdl = model.astype(dtype)
    B = hidden.shape[0]
    shapes = mdl.mat_shapes()
    per_seq = mdl.n_blocks * sum(r * c for r, c in shapes)
    W0_flat = np.asarray(W0_flat, dtype=dtype).reshape(B, per_seq)
    M0_flat = np.asarray(M0_flat, dtype=dtype).reshape(B, per_seq)
    Ws, Ms, Ls = [], [], []
    for s in range(B):
        W0 = unpack_blocks(W0_flat[s].copy(), mdl.n_blocks, shapes)
        M0 = unpack_blocks(M0_flat[s].copy(), mdl.n_blocks, shapes)
        W, M, L = prefill_sequence(mdl, W0, M0, np.asarray(hidden[s], dtype=dtype),
                                   np.asarray(tokens[s]), eta[s], beta[s], gamma[s], b,
                                   update=update, n_chunks=n_chunks, reduction=reduction)
        Ws.append(pack_blocks(W))
        Ms.append(pack_blocks(M))
        Ls.append(L)
    return np.concatenate(Ws), np.concatenate(Ms), np.stack(Ls)


def state_without_gradients(W0_flat, M0_flat, eta, beta, gamma, b, n_chunks: Optional[int] = None,
                            update: str = "closed"):
    """The chunk-end states the inner loop would reach if every G_t were 0.

    Proposition 3.1 ([E2-TTT] 命题3.1) with the gradient sums dropped, chunk by
    chunk: W <- gtilde_0 W + btilde_0 R_1 M, M <- btilde_0 M; under LaCT's
    rule ([E2-TTT] 高效的逐块更新机制) M <- mean(beta) M, W <- W + M.  It is
    elementwise, so W0_flat / M0_flat may be any subset of the flat state of
    each sequence: arrays [B, n] (or [n] for one sequence), eta/beta/gamma
    [B, T].  Subtracting it from a final state leaves the part the gradients
    contributed (the update GEMMs' work), which the parity tests check on its
    own because the decayed initial state can dominate W.  float64.
    """
    W = np.array(W0_flat, dtype=np.float64, copy=True)
    M = np.array(M0_flat, dtype=np.float64, copy=True)
    one = W.ndim == 1
    if one:
        W, M = W[None], M[None]
    eta = np.asarray(eta, dtype=np.float64).reshape(W.shape[0], -1)
    beta = np.asarray(beta, dtype=np.float64).reshape(W.shape[0], -1)
    gamma = np.asarray(gamma, dtype=np.float64).reshape(W.shape[0], -1)
    nc = eta.shape[1] // b if n_chunks is None else n_chunks
    for s in range(W.shape[0]):
        for c in range(nc):
            sl = slice(c * b, (c + 1) * b)
            if update == "lact":
                bbar = float(np.mean(beta[s, sl]))
                M[s] = bbar * M[s]
                W[s] = W[s] + M[s]
            else:
                _, _, g0, b0, cM = scalar_kernels(eta[s, sl], beta[s, sl], gamma[s, sl])
                W[s] = g0 * W[s] + cM * M[s]
                M[s] = b0 * M[s]
    return (W[0], M[0]) if one else (W, M)


# ---------------------------------------------------------------------------
# Final prediction with the updated weights
# ([TTT-E2E] 持续学习框架 (预测 step) and the sketch's 最终预测 part;
#  per-position breakdown as in [Review] 图6)
# ---------------------------------------------------------------------------

def group_means(loss: np.ndarray, b: int) -> np.ndarray:
    """Mean of each run of b consecutive positions of one sequence."""
    return loss.reshape(-1, b).mean(axis=1)


def final_prediction(model: Model, W_flat, hidden, tokens, b, dtype=np.float64):
    """Forward-only pass of whole sequences at fixed fast weights.

    After the inner loop the weights W_T hold the context; the sequence is
    run again through the blocks, the frozen RMSNorm and the LM head at W_T,
    with no update, and scored by the next-token loss.  Every row is
    independent here (the weights do not change), so the whole sequence is
    one forward.  Reading: the losses are reported per token and as the mean
    of each group of b positions (the loss-by-position curve); the sketch's
    single final loss is the mean of all of them.

    hidden [B,T,d], tokens [B,T] (labels, as in ``prefill``),
    W_flat [B * n_blocks * m * h * d].  Returns (token_loss [B,T],
    group_loss [B, T // b]) in ``dtype``.
    """
    mdl = model.astype(dtype)
    B, T = np.asarray(tokens).shape
    if T % b != 0:
        raise ValueError("T must be a multiple of b")
    shapes = mdl.mat_shapes()
    per_seq = mdl.n_blocks * sum(r * c for r, c in shapes)
    Wf = np.asarray(W_flat, dtype=dtype).reshape(B, per_seq)
    tok = np.zeros((B, T), dtype=dtype)
    grp = np.zeros((B, T // b), dtype=dtype)
    for s in range(B):
        W = unpack_blocks(Wf[s].copy(), mdl.n_blocks, shapes)
        loss, _ = chunk_forward(mdl, W, np.asarray(hidden[s], dtype=dtype), np.asarray(tokens[s]))
        tok[s] = loss
        grp[s] = group_means(loss, b)
    return tok, grp


# ---------------------------------------------------------------------------
# E2-TTT's own layer: key/value reconstruction, query outputs
# ([E2-TTT] 背景知识 (TTT建模范式, 表达能力强的逐Token更新机制), 快速权重网络实例化, Algorithm 1)
# ---------------------------------------------------------------------------

def recon_shapes(kind: str, d: int, h: int):
    """Fast-weight matrices of the layer's MLP, [rows, cols] each."""
    return [(h, d), (d, h)] if kind == GELU else [(h, d), (h, d), (d, h)]


def layer_norm(y, eps):
    """Parameter-free LayerNorm over the last axis; returns (LN(y), 1/std)."""
    mu = y.mean(axis=-1, keepdims=True)
    var = ((y - mu) ** 2).mean(axis=-1, keepdims=True)
    rs = 1.0 / np.sqrt(var + eps)
    return (y - mu) * rs, rs


def layer_norm_backward(g, ln, rs):
    """dL/dy from dL/dLN(y) for the parameter-free LayerNorm."""
    return rs * (g - g.mean(axis=-1, keepdims=True) - ln * (g * ln).mean(axis=-1, keepdims=True))


def recon_forward(kind: str, mats, X, eps):
    """f_W(x) = x + LN(MLP_W(x)) ([E2-TTT] 快速权重网络实例化); rows of X."""
    y, cache = mlp_forward(kind, mats, X)
    ln, rs = layer_norm(y, eps)
    return X + ln, (cache, ln, rs)


def recon_chunk(kind: str, mats, K, V, eps):
    """Per-token reconstruction losses L_t = mean_j (f_W(k_t) - v_t)_j^2 (the
    mean squared error) at the chunk-start weights, and the factor pairs of
    their gradients (one backward for the chunk)."""
    f, (cache, ln, rs) = recon_forward(kind, mats, K, eps)
    r = f - V
    loss = (r * r).mean(axis=1)
    gf = 2.0 * r / r.shape[1]
    gy = layer_norm_backward(gf, ln, rs)
    _, pairs = mlp_backward(kind, mats, cache, gy)
    return loss, pairs


def prefill_recon(kind: str, d: int, h: int, W0_flat, M0_flat, K, V, Q, eta, beta, gamma, b, eps,
                  dtype=np.float64, update: str = "closed", reduction: str = "mean",
                  n_chunks: Optional[int] = None):
    """The layer over batched sequences (Algorithm 1 chunk after chunk): for each
    chunk, outputs o_t = f_{W_0}(q_t) and losses at the chunk-start weights, one
    backward, then the chunk update (Proposition 3.1, or LaCT's rule).
    K, V, Q [B, T, d]; W0_flat / M0_flat [B * m * h * d].  Returns
    (W_flat, M_flat, chunk_loss [B, n_chunks], O [B, T, d])."""
    if update not in UPDATE_RULES:
        raise ValueError("update must be one of " + ", ".join(UPDATE_RULES))
    step = {"closed": chunk_update_closed, "explicit": chunk_update_explicit, "lact": chunk_update_lact}[update]
    gscale = 1.0 / b if reduction == "mean" else 1.0
    shapes = recon_shapes(kind, d, h)
    per_seq = sum(r * c for r, c in shapes)
    Bn, T, _ = np.shape(K)
    nc = T // b if n_chunks is None else n_chunks
    W0_flat = np.asarray(W0_flat, dtype=dtype).reshape(Bn, per_seq)
    M0_flat = np.asarray(M0_flat, dtype=dtype).reshape(Bn, per_seq)
    Ws, Ms, Ls = [], [], []
    O = np.zeros((Bn, nc * b, d), dtype=dtype)
    for s in range(Bn):
        W = unpack_blocks(W0_flat[s].copy(), 1, shapes)
        M = unpack_blocks(M0_flat[s].copy(), 1, shapes)
        losses = np.zeros(nc)
        for c in range(nc):
            sl = slice(c * b, (c + 1) * b)
            Kc, Vc, Qc = (np.asarray(a[s][sl], dtype=dtype) for a in (K, V, Q))
            O[s, sl] = recon_forward(kind, W[0], Qc, eps)[0]
            loss, pairs = recon_chunk(kind, W[0], Kc, Vc, eps)
            losses[c] = float(np.mean(loss))
            W, M = step(W, M, [pairs], eta[s][sl], beta[s][sl], gamma[s][sl], gscale)
        Ws.append(pack_blocks(W))
        Ms.append(pack_blocks(M))
        Ls.append(losses)
    return np.concatenate(Ws), np.concatenate(Ms), np.stack(Ls), O


def token_losses(model: Model, W_flat, X, y, dtype=np.float64):
    """Per-token losses of rows X at fast weights W_flat (one sequence)."""
    mdl = model.astype(dtype)
    W = unpack_blocks(np.asarray(W_flat, dtype=dtype), mdl.n_blocks, mdl.mat_shapes())
    loss, _ = chunk_forward(mdl, W, np.asarray(X, dtype=dtype), np.asarray(y))
    return loss


def token_gradients(model: Model, W_flat, X, y, dtype=np.float64):
    """Per-token gradients dl_t/dW as a dense array [n, n_params] (tiny shapes only)."""
    mdl = model.astype(dtype)
    W = unpack_blocks(np.asarray(W_flat, dtype=dtype), mdl.n_blocks, mdl.mat_shapes())
    X = np.asarray(X, dtype=dtype)
    y = np.asarray(y)
    _, fwd = chunk_forward(mdl, W, X, y)
    grads = chunk_backward(mdl, W, y, fwd)
    n = X.shape[0]
    rows = []
    for t in range(n):
        parts = []
        for l in range(mdl.n_blocks):
            for (Lf, Rf) in grads[l]:
                parts.append(np.outer(Lf[t], Rf[t]).reshape(-1))
        rows.append(np.concatenate(parts))
    return np.stack(rows)
