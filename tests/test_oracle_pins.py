"""Pins of the CPU oracle to things other than itself (CPU only).

Each pin cites the passage it checks.  Pages by title:
  [E2-TTT]  "Rethinking Expressivity and Efficiency in Test-Time Training"
  [TTT-E2E] "TTT-E2E：端到端测试时训练的长上下文语言建模"
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import ttt_oracle as O
from tests import autograd_model as AM


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def tiny_setup(kind="gelu", d=4, h=6, V=7, L=2, static=True, T=12, seed=1,
               m0=0.05, scalars="e2ttt"):
    rng = np.random.default_rng(seed)
    shapes = AM.shapes_of(kind, d, h)
    per_block = sum(r * c for r, c in shapes)
    E = rng.normal(0, 0.5, (V, d))
    g = rng.uniform(0.5, 1.5, d)
    static_w = rng.normal(0, 0.4, L * per_block) if static else None
    W0 = rng.normal(0, 0.4, L * per_block)
    M0 = rng.normal(0, m0, L * per_block) if m0 else np.zeros(L * per_block)
    X = rng.normal(0, 1, (T, d))
    y = rng.integers(0, V, T)
    if scalars == "sgd":
        eta = np.full(T, 0.1)
        beta = np.zeros(T)
        gamma = np.ones(T)
    else:
        eta = 0.05 / (1 + np.exp(-rng.normal(size=T)))
        beta = rng.uniform(0.8, 0.99, T)
        gamma = rng.uniform(0.99, 1.0, T)
    model = O.make_model(d, h, V, L, kind, 1e-6, E, g, static_w)
    return dict(model=model, kind=kind, d=d, h=h, V=V, L=L, E=E, g=g, static_w=static_w,
                W0=W0, M0=M0, X=X, y=y, eta=eta, beta=beta, gamma=gamma)


def run_prefill(s, b, update="closed", reduction="mean", **over):
    p = dict(s)
    p.update(over)
    W, M, Ls = O.prefill(p["model"], p["W0"], p["M0"], p["X"][None], p["y"][None],
                         p["eta"][None], p["beta"][None], p["gamma"][None], b,
                         update=update, reduction=reduction)
    return W, M, Ls[0]


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300))


# ---------------------------------------------------------------------------
# 1. Scalar kernels against the exact recursion in rational arithmetic
#    ([E2-TTT] 原始公式 vs 命题3.1)
# ---------------------------------------------------------------------------

def exact_coefficients(eta, beta, gamma):
    """Run M_t = beta_t M_{t-1} + eta_t G_t, W_t = gamma_t W_{t-1} + M_t exactly,
    with W_0, M_0, G_1..G_C as independent basis vectors.  Returns the
    coefficient vectors of W_C and M_C over (W_0, M_0, G_1..G_C)."""
    C = len(eta)
    n = C + 2
    W = [Fraction(0)] * n
    M = [Fraction(0)] * n
    W[0] = Fraction(1)
    M[1] = Fraction(1)
    for t in range(C):
        M = [beta[t] * m for m in M]
        M[2 + t] += eta[t]
        W = [gamma[t] * w + m for w, m in zip(W, M)]
    return W, M


@pytest.mark.parametrize("case", ["random", "beta_zero", "ones", "mixed_zero"])
def test_scalar_kernels_match_exact_recursion(case):
    rng = np.random.default_rng(7)
    C = 9
    den = 97
    eta = [Fraction(int(rng.integers(1, 50)), 1000) for _ in range(C)]
    if case == "random":
        beta = [Fraction(int(rng.integers(60, 97)), den) for _ in range(C)]
        gamma = [Fraction(int(rng.integers(80, 97)), den) for _ in range(C)]
    elif case == "beta_zero":          # plain SGD-like momentum-free chunk
        beta = [Fraction(0)] * C
        gamma = [Fraction(1)] * C
    elif case == "ones":
        beta = [Fraction(1)] * C
        gamma = [Fraction(1)] * C
    else:                              # a zero momentum factor in mid-chunk
        beta = [Fraction(int(rng.integers(60, 97)), den) for _ in range(C)]
        beta[4] = Fraction(0)
        gamma = [Fraction(int(rng.integers(80, 97)), den) for _ in range(C)]
    Wc, Mc = exact_coefficients(eta, beta, gamma)
    KW, KM, g0, b0, cM = O.scalar_kernels([float(x) for x in eta], [float(x) for x in beta],
                                          [float(x) for x in gamma])
    tol = 1e-14
    assert abs(g0 - float(Wc[0])) <= tol * max(1, abs(float(Wc[0])))
    assert abs(cM - float(Wc[1])) <= tol * max(1, abs(float(Wc[1])))
    assert abs(b0 - float(Mc[1])) <= tol
    assert float(Mc[0]) == 0.0
    np.testing.assert_allclose(KW, [float(x) for x in Wc[2:]], rtol=1e-13, atol=1e-18)
    np.testing.assert_allclose(KM, [float(x) for x in Mc[2:]], rtol=1e-13, atol=1e-18)


def test_scalar_kernels_match_ratio_form():
    """Division-free evaluation == the printed R_t = sum gtilde_i / btilde_i form."""
    rng = np.random.default_rng(3)
    for C in (1, 2, 16, 64):
        eta = 0.01 / (1 + np.exp(-rng.normal(size=C)))
        beta = rng.uniform(0.8, 0.99, C)
        gamma = rng.uniform(0.99, 1.0, C)
        a = O.scalar_kernels(eta, beta, gamma)
        r = O.scalar_kernels_ratio_form(eta, beta, gamma)
        np.testing.assert_allclose(a[0], r[0], rtol=1e-12)
        np.testing.assert_allclose(a[1], r[1], rtol=1e-12)
        np.testing.assert_allclose(a[2:], r[2:], rtol=1e-12)


def test_R_limits_and_bounds():
    """[E2-TTT] 累积核 R_t 的稳定性分析: beta, gamma -> 1 gives R_t = C - t + 1,
    so K_W <= eta * C; and 0 <= K_M <= eta, 0 <= K_W <= eta (C - t + 1)."""
    C = 32
    eta = np.linspace(0.001, 0.01, C)
    KW, KM, g0, b0, cM = O.scalar_kernels(eta, np.ones(C), np.ones(C))
    t = np.arange(1, C + 1)
    np.testing.assert_allclose(KW, eta * (C - t + 1), rtol=1e-15)
    np.testing.assert_allclose(KM, eta, rtol=1e-15)
    assert g0 == 1.0 and b0 == 1.0 and cM == pytest.approx(C, rel=1e-15)
    rng = np.random.default_rng(0)
    for _ in range(20):
        beta = rng.uniform(0, 1, C)
        gamma = rng.uniform(0, 1, C)
        KW, KM, g0, b0, cM = O.scalar_kernels(eta, beta, gamma)
        assert np.all(KM >= 0) and np.all(KM <= eta * (1 + 1e-15))
        assert np.all(KW >= 0) and np.all(KW <= eta * (C - t + 1) * (1 + 1e-15))
        assert 0 <= cM <= C


def test_scalar_kernels_underflow_finite():
    """b = 1024 with beta ~ U(.8,.99): prod beta underflows float32 (about 1e-47),
    the ratio form would divide by it; the coefficients must stay finite."""
    rng = np.random.default_rng(0)
    C = 1024
    beta = rng.uniform(0.8, 0.99, C)
    gamma = rng.uniform(0.99, 1.0, C)
    eta = np.full(C, 0.01)
    KW, KM, g0, b0, cM = O.scalar_kernels(eta, beta, gamma)
    assert np.all(np.isfinite(KW)) and np.all(np.isfinite(KM))
    assert np.float32(b0) == 0.0          # would underflow in float32
    assert np.all(KW <= 0.01 * (C - np.arange(C)))


# ---------------------------------------------------------------------------
# 2. Closed form == explicit per-token recursion on the full model
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind,static,red", [("gelu", False, "mean"), ("gelu", True, "sum"),
                                             ("swiglu", True, "mean"), ("swiglu", False, "sum")])
def test_closed_form_equals_recursion(kind, static, red):
    s = tiny_setup(kind=kind, static=static, h=6 if kind == "gelu" else 5, T=12)
    W1, M1, L1 = run_prefill(s, 4, "closed", reduction=red)
    W2, M2, L2 = run_prefill(s, 4, "explicit", reduction=red)
    assert rel(W1, W2) < 1e-12
    assert rel(M1, M2) < 1e-12
    np.testing.assert_allclose(L1, L2, rtol=1e-13)


# ---------------------------------------------------------------------------
# 3. Per-token gradients: finite differences and autograd
#    ([E2-TTT] 单次反向传播的链式法则分解)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["gelu", "swiglu"])
def test_gradients_match_finite_differences(kind):
    s = tiny_setup(kind=kind, d=3, h=4, V=5, L=2, static=True, T=3)
    model, W, X, y = s["model"], s["W0"], s["X"], s["y"]
    G = O.token_gradients(model, W, X, y)
    eps = 1e-6
    fd = np.zeros_like(G)
    for i in range(W.size):
        Wp = W.copy(); Wp[i] += eps
        Wm = W.copy(); Wm[i] -= eps
        fd[:, i] = (O.token_losses(model, Wp, X, y) - O.token_losses(model, Wm, X, y)) / (2 * eps)
    np.testing.assert_allclose(G, fd, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("kind,static,L", [("gelu", False, 1), ("gelu", True, 3), ("swiglu", True, 2)])
def test_gradients_and_losses_match_autograd(kind, static, L):
    s = tiny_setup(kind=kind, d=6, h=8, V=11, L=L, static=static, T=5)
    T_ = lambda a: None if a is None else torch.tensor(a, dtype=torch.float64)
    Ga, La = AM.per_token_grads(kind, 6, 8, L, 1e-6, T_(s["E"]), T_(s["g"]), T_(s["static_w"]),
                                T_(s["W0"]), T_(s["X"]), torch.tensor(s["y"]))
    G = O.token_gradients(s["model"], s["W0"], s["X"], s["y"])
    Lo = O.token_losses(s["model"], s["W0"], s["X"], s["y"])
    np.testing.assert_allclose(Lo, La.numpy(), rtol=1e-12)
    np.testing.assert_allclose(G, Ga.numpy(), rtol=1e-10, atol=1e-13)


# ---------------------------------------------------------------------------
# 4. SGD reduction ([TTT-E2E] 持续学习框架: W_t = W_{t-1} - alpha grad l_t)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["gelu", "swiglu"])
def test_b1_sgd_is_online_sgd(kind):
    """b = 1, beta = 0, gamma = 1, eta = alpha: the chunk update is exactly one
    online SGD step per token, with the loss taken before the step."""
    s = tiny_setup(kind=kind, d=5, h=7, V=9, L=2, static=True, T=10, scalars="sgd", m0=0.3)
    alpha = 0.1
    W, M, Ls = run_prefill(s, 1)
    T_ = lambda a: None if a is None else torch.tensor(a, dtype=torch.float64)
    Wt = T_(s["W0"])
    ref_losses = []
    for t in range(10):
        Wv = Wt.clone().requires_grad_(True)
        l = AM.losses(kind, 5, 7, 2, 1e-6, T_(s["E"]), T_(s["g"]), T_(s["static_w"]), Wv,
                      T_(s["X"][t:t + 1]), torch.tensor(s["y"][t:t + 1]))[0]
        (gr,) = torch.autograd.grad(l, Wv)
        ref_losses.append(float(l))
        Wt = Wt - alpha * gr
    assert rel(W, Wt.numpy()) < 1e-12
    np.testing.assert_allclose(Ls, ref_losses, rtol=1e-12)


@pytest.mark.parametrize("red", ["mean", "sum"])
def test_chunked_sgd_uses_chunk_start_gradients(red):
    """b = 4 SGD: one mini-batch step at the chunk-start weights,
    W_C = W_0 - alpha grad (mean_t l_t)(W_0) (reduction "mean"; the sum for
    "sum"), and M_C = eta_C G_C (only the last token survives when beta = 0)."""
    s = tiny_setup(kind="gelu", d=5, h=7, V=9, L=1, static=False, T=4, scalars="sgd", m0=0.3)
    W, M, Ls = run_prefill(s, 4, reduction=red)
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    Wv = T_(s["W0"]).requires_grad_(True)
    l = AM.losses("gelu", 5, 7, 1, 1e-6, T_(s["E"]), T_(s["g"]), None, Wv, T_(s["X"]), torch.tensor(s["y"]))
    obj = l.mean() if red == "mean" else l.sum()
    (gobj,) = torch.autograd.grad(obj, Wv, retain_graph=True)
    (glast,) = torch.autograd.grad(l[3], Wv)
    scale = 0.25 if red == "mean" else 1.0
    assert rel(W, (T_(s["W0"]) - 0.1 * gobj).numpy()) < 1e-12
    assert rel(M, (-0.1 * scale * glast).numpy()) < 1e-12
    assert Ls[0] == pytest.approx(float(l.mean()), rel=1e-12)


# ---------------------------------------------------------------------------
# 4b. LaCT's chunk-wise rule ([E2-TTT] 高效的逐块（Chunk-wise）更新机制)
# ---------------------------------------------------------------------------

def test_lact_without_momentum_matches_closed_form_w():
    """beta = 0: LaCT's W_C = W_0 + sum_t eta_t G_t, which is also the E2-TTT
    chunk end with beta = 0, gamma = 1; LaCT's M_C is the whole chunk step."""
    s = tiny_setup(kind="swiglu", d=4, h=6, V=7, L=2, static=True, T=8, seed=3)
    T = len(s["eta"])
    Wl, Ml, _ = run_prefill(s, 4, update="lact", beta=np.zeros(T), gamma=s["gamma"])
    Wc, _, _ = run_prefill(s, 4, update="closed", beta=np.zeros(T), gamma=np.ones(T))
    assert rel(Wl, Wc) < 1e-12
    # the last chunk's step is the last chunk's M
    Wp, _, _ = run_prefill(s, 4, update="lact", beta=np.zeros(T), gamma=s["gamma"],
                           X=s["X"][:4], y=s["y"][:4], eta=s["eta"][:4])
    assert rel(Ml, Wl - Wp) < 1e-10


@pytest.mark.parametrize("red", ["mean", "sum"])
def test_lact_direction_is_gradient_of_weighted_loss(red):
    """One chunk from M_0 = 0: M_C = -grad_W sum_t eta_t l_t (l_t / b for the
    mean reduction) at W_0, taken by torch autograd of an independent model."""
    s = tiny_setup(kind="gelu", d=5, h=7, V=9, L=1, static=False, T=6, seed=4, m0=0.0)
    W, M, _ = run_prefill(s, 6, update="lact", reduction=red)
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    Wv = T_(s["W0"]).requires_grad_(True)
    l = AM.losses("gelu", 5, 7, 1, 1e-6, T_(s["E"]), T_(s["g"]), None, Wv, T_(s["X"]), torch.tensor(s["y"]))
    scale = 1.0 / 6 if red == "mean" else 1.0
    (g,) = torch.autograd.grad((T_(s["eta"]) * l).sum() * scale, Wv)
    assert rel(M, (-g).numpy()) < 1e-12
    assert rel(W, (T_(s["W0"]) - g).numpy()) < 1e-12


def test_lact_momentum_factor_is_the_chunk_average():
    """beta alternating 0, 1 averages to 1/2 exactly (a product would give 0,
    the last token's factor 1): M_C - M_C(M_0 = 0) = M_0 / 2."""
    s = tiny_setup(kind="gelu", d=4, h=5, V=6, L=1, static=False, T=4, seed=5, m0=0.3)
    beta = np.array([0.0, 1.0, 0.0, 1.0])
    _, M, _ = run_prefill(s, 4, update="lact", beta=beta)
    _, M0run, _ = run_prefill(s, 4, update="lact", beta=beta, M0=np.zeros_like(s["M0"]))
    assert rel(M - M0run, 0.5 * s["M0"]) < 1e-12


def test_lact_ignores_decay():
    """LaCT's rule has no decay term: gamma does not change the result."""
    s = tiny_setup(kind="gelu", d=4, h=5, V=6, L=1, static=False, T=8, seed=6)
    W1, M1, _ = run_prefill(s, 4, update="lact", gamma=np.full(8, 0.5))
    W2, M2, _ = run_prefill(s, 4, update="lact", gamma=np.ones(8))
    assert rel(W1, W2) == 0.0 and rel(M1, M2) == 0.0


# ---------------------------------------------------------------------------
# 4c. Input-dependent scalars ([E2-TTT] 依赖于输入的动态参数化)
# ---------------------------------------------------------------------------

def test_scalar_heads_at_zero_logits():
    """Zero weights and biases: every gate is sigmoid(0) = 1/2 exactly, so
    eta = eta_base / 2, beta = 2^(-1/tau), gamma = 1 - eta_base alpha_base / 4."""
    X = np.random.default_rng(0).normal(size=(5, 7))
    eta, beta, gamma = O.scalar_heads(X, np.zeros((3, 7)), np.zeros(3), 0.02, 0.5, 8.0)
    np.testing.assert_allclose(eta, 0.01, rtol=1e-15)
    np.testing.assert_allclose(beta, 2.0 ** (-1.0 / 8.0), rtol=1e-15)
    np.testing.assert_allclose(gamma, 1.0 - 0.02 * 0.5 / 4.0, rtol=1e-15)


def test_scalar_heads_saturation_and_heads_are_separate():
    """A large positive logit on one head only saturates that head's gate:
    eta -> eta_base while beta and alpha stay at sigmoid(0) = 1/2."""
    X = np.ones((1, 4))
    heads = np.zeros((3, 4))
    heads[0] = 50.0                       # eta head only
    eta, beta, gamma = O.scalar_heads(X, heads, np.zeros(3), 0.01, 1.0, 4.0)
    assert eta[0] == pytest.approx(0.01, rel=1e-15)
    assert beta[0] == pytest.approx(0.5 ** 0.25, rel=1e-15)
    assert gamma[0] == pytest.approx(1.0 - 0.01 * 0.5, rel=1e-15)
    heads = np.zeros((3, 4))
    heads[1] = -50.0                      # beta head only: sigmoid -> 0
    _, beta, _ = O.scalar_heads(X, heads, np.zeros(3), 0.01, 1.0, 4.0)
    assert beta[0] < 1e-20


def test_scalar_heads_linear_in_x_and_bias():
    """The gate logits are affine in x: moving x along w_beta by s changes
    sigmoid^-1(beta^tau) by s |w_beta|^2, and the bias enters additively."""
    rng = np.random.default_rng(1)
    d = 6
    heads = rng.normal(size=(3, d))
    bias = rng.normal(size=3)
    x = rng.normal(size=(1, d))
    logit = lambda b: np.log(b ** 4.0 / (1.0 - b ** 4.0))
    _, b1, _ = O.scalar_heads(x, heads, bias, 0.01, 1.0, 4.0)
    _, b2, _ = O.scalar_heads(x + 0.1 * heads[1], heads, bias, 0.01, 1.0, 4.0)
    assert logit(b2[0]) - logit(b1[0]) == pytest.approx(0.1 * float(heads[1] @ heads[1]), rel=1e-9)
    _, b3, _ = O.scalar_heads(x, heads, bias + np.array([0.0, 0.3, 0.0]), 0.01, 1.0, 4.0)
    assert logit(b3[0]) - logit(b1[0]) == pytest.approx(0.3, rel=1e-9)


# ---------------------------------------------------------------------------
# 4d. E2-TTT's own layer: reconstruction loss, query outputs, inner LayerNorm
# ---------------------------------------------------------------------------

def recon_setup(kind="gelu", d=6, h=9, T=8, seed=7, m0=0.05):
    rng = np.random.default_rng(seed)
    n = sum(r * c for r, c in AM.shapes_of(kind, d, h))
    return dict(kind=kind, d=d, h=h, W0=rng.normal(0, 0.4, n), M0=rng.normal(0, m0, n),
                K=rng.normal(size=(T, d)), V=rng.normal(size=(T, d)), Q=rng.normal(size=(T, d)),
                eta=0.05 / (1 + np.exp(-rng.normal(size=T))), beta=rng.uniform(0.8, 0.99, T),
                gamma=rng.uniform(0.99, 1.0, T))


def _recon_pairs_as_grads(kind, d, h, W, K, V, eps):
    """Per-token gradients [T, n] from the oracle's factor pairs."""
    mats = AM.split_blocks(W, 1, AM.shapes_of(kind, d, h))[0]
    loss, pairs = O.recon_chunk(kind, mats, K, V, eps)
    cols = [np.einsum("ti,tj->tij", Lf, Rf).reshape(len(K), -1) for Lf, Rf in pairs]
    return loss, np.concatenate(cols, axis=1)


@pytest.mark.parametrize("kind", ["gelu", "swiglu"])
def test_recon_losses_and_gradients_match_autograd(kind):
    s = recon_setup(kind)
    d, h, eps = s["d"], s["h"], 1e-6
    loss, G = _recon_pairs_as_grads(kind, d, h, s["W0"], s["K"], s["V"], eps)
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    Wv = T_(s["W0"]).requires_grad_(True)
    L = AM.recon_losses(kind, d, h, eps, Wv, T_(s["K"]), T_(s["V"]))
    np.testing.assert_allclose(loss, L.detach().numpy(), rtol=1e-12)
    for t in range(len(s["K"])):
        (g,) = torch.autograd.grad(L[t], Wv, retain_graph=True)
        assert rel(G[t], g.numpy()) < 1e-10
    Ot = AM.recon_outputs(kind, d, h, eps, T_(s["W0"]), T_(s["Q"])).numpy()
    mats = AM.split_blocks(s["W0"], 1, AM.shapes_of(kind, d, h))[0]
    assert rel(O.recon_forward(kind, mats, s["Q"], eps)[0], Ot) < 1e-13


def test_recon_gradients_match_finite_differences():
    s = recon_setup("swiglu", d=5, h=7, T=3, seed=8)
    d, h, eps = s["d"], s["h"], 1e-6
    _, G = _recon_pairs_as_grads("swiglu", d, h, s["W0"], s["K"], s["V"], eps)
    mats_of = lambda W: AM.split_blocks(W, 1, AM.shapes_of("swiglu", d, h))[0]
    rng = np.random.default_rng(0)
    for idx in rng.choice(len(s["W0"]), 12, replace=False):
        e = np.zeros_like(s["W0"])
        e[idx] = 1e-6
        lp, _ = O.recon_chunk("swiglu", mats_of(s["W0"] + e), s["K"], s["V"], eps)
        lm, _ = O.recon_chunk("swiglu", mats_of(s["W0"] - e), s["K"], s["V"], eps)
        np.testing.assert_allclose(G[:, idx], (lp - lm) / 2e-6, rtol=1e-5, atol=1e-8)


def test_recon_zero_output_matrix():
    """A zero output matrix makes the MLP branch zero and LayerNorm(0) = 0, so
    the layer is the identity: o_t = q_t and L_t = mean_j (k_t - v_t)_j^2 exactly."""
    s = recon_setup("gelu", d=6, h=9)
    W = s["W0"].copy()
    W[9 * 6:] = 0.0                              # W2 [d, h]
    Wf, Mf, Ls, Oo = O.prefill_recon("gelu", 6, 9, W, s["M0"], s["K"][None], s["V"][None], s["Q"][None],
                                     s["eta"][None], s["beta"][None], s["gamma"][None], 8, 1e-6)
    np.testing.assert_array_equal(Oo[0], s["Q"])
    assert Ls[0, 0] == pytest.approx(float(((s["K"] - s["V"]) ** 2).mean()), rel=1e-14)


@pytest.mark.parametrize("rule", ["closed", "lact"])
def test_recon_prefill_closed_form_equals_recursion(rule):
    """Over several chunks the Proposition 3.1 chunk end equals the per-token
    recursion (and LaCT's rule runs through the same driver)."""
    s = recon_setup("swiglu", T=12)
    args = ("swiglu", s["d"], s["h"], s["W0"], s["M0"], s["K"][None], s["V"][None], s["Q"][None],
            s["eta"][None], s["beta"][None], s["gamma"][None], 4, 1e-6)
    Wc, Mc, Lc, Oc = O.prefill_recon(*args, update=rule)
    if rule == "closed":
        We, Me, Le, Oe = O.prefill_recon(*args, update="explicit")
        assert rel(Wc, We) < 1e-12 and rel(Mc, Me) < 1e-12
        np.testing.assert_allclose(Lc, Le, rtol=1e-12)
        np.testing.assert_allclose(Oc, Oe, rtol=1e-12)
    else:
        assert np.all(np.isfinite(Wc)) and Lc.shape == (1, 3)


# ---------------------------------------------------------------------------
# 5. Cross-entropy closed forms
# ---------------------------------------------------------------------------

def test_zero_lm_head_gives_log_v_and_no_gradient():
    s = tiny_setup(kind="swiglu", d=4, h=5, V=13, L=2, static=True, T=8)
    s["model"].lm_head[:] = 0.0
    W, M, Ls = run_prefill(s, 4)
    np.testing.assert_allclose(Ls, np.log(13.0), rtol=1e-14)
    # no gradient: only decay / momentum act
    W_ref, M_ref = s["W0"].copy(), s["M0"].copy()
    for c in range(2):
        sl = slice(4 * c, 4 * c + 4)
        KW, KM, g0, b0, cM = O.scalar_kernels(s["eta"][sl], s["beta"][sl], s["gamma"][sl])
        W_ref, M_ref = g0 * W_ref + cM * M_ref, b0 * M_ref
    assert rel(W, W_ref) < 1e-13 and rel(M, M_ref) < 1e-13


def test_two_class_loss_is_softplus():
    """V = 2: l = softplus(logit_other - logit_target).  With W1 = 0 every
    dynamic MLP outputs 0 (GELU(0) = 0), so h = x and the logits are
    RMSNorm(x) E^T, computed here directly."""
    s = tiny_setup(kind="gelu", d=6, h=4, V=2, L=1, static=False, T=8)
    W = s["W0"].copy()
    W[:4 * 6] = 0.0
    X, y, E, g = s["X"], s["y"], s["E"], s["g"]
    z = X / np.sqrt(np.mean(X ** 2, axis=1, keepdims=True) + 1e-6) * g
    lg = z @ E.T
    other = lg[np.arange(8), 1 - y]
    target = lg[np.arange(8), y]
    expect = np.log1p(np.exp(other - target))
    np.testing.assert_allclose(O.token_losses(s["model"], W, X, y), expect, rtol=1e-13)


# ---------------------------------------------------------------------------
# 6. Resume, linearity, chunk-start losses
# ---------------------------------------------------------------------------

def test_resume_equivalence():
    """Only the chunk-end state crosses chunk boundaries ([E2-TTT] 原始公式,
    last sentence): prefill(T) == prefill(T1) then prefill(T - T1)."""
    s = tiny_setup(kind="swiglu", d=4, h=5, V=7, L=2, static=True, T=12)
    W, M, Ls = run_prefill(s, 3)
    T1 = 6
    s1 = dict(s, X=s["X"][:T1], y=s["y"][:T1], eta=s["eta"][:T1], beta=s["beta"][:T1], gamma=s["gamma"][:T1])
    Wa, Ma, La = run_prefill(s1, 3)
    s2 = dict(s, X=s["X"][T1:], y=s["y"][T1:], eta=s["eta"][T1:], beta=s["beta"][T1:], gamma=s["gamma"][T1:],
              W0=Wa, M0=Ma)
    Wb, Mb, Lb = run_prefill(s2, 3)
    assert rel(Wb, W) < 1e-14 and rel(Mb, M) < 1e-14
    np.testing.assert_allclose(np.concatenate([La, Lb]), Ls, rtol=1e-14)


def test_single_chunk_update_is_linear_in_eta():
    s = tiny_setup(kind="gelu", d=4, h=6, V=7, L=2, static=True, T=6)
    W1, M1, _ = run_prefill(s, 6)
    W3, M3, _ = run_prefill(s, 6, eta=3.0 * s["eta"])
    KW, KM, g0, b0, cM = O.scalar_kernels(s["eta"], s["beta"], s["gamma"])
    base_W = g0 * s["W0"] + cM * s["M0"]
    base_M = b0 * s["M0"]
    assert rel(W3 - base_W, 3.0 * (W1 - base_W)) < 1e-12
    assert rel(M3 - base_M, 3.0 * (M1 - base_M)) < 1e-12


def test_chunk_loss_is_mean_at_chunk_start_weights():
    """[E2-TTT] O^[r] = f_{W^[r-1]}(Q^[r]): chunk c's loss uses the state after c chunks."""
    s = tiny_setup(kind="swiglu", d=4, h=5, V=7, L=2, static=True, T=12)
    _, _, Ls = run_prefill(s, 4)
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    for c in range(3):
        if c == 0:
            Wc = s["W0"]
        else:
            sc = dict(s, X=s["X"][:4 * c], y=s["y"][:4 * c], eta=s["eta"][:4 * c],
                      beta=s["beta"][:4 * c], gamma=s["gamma"][:4 * c])
            Wc, _, _ = run_prefill(sc, 4)
        l = AM.losses("swiglu", 4, 5, 2, 1e-6, T_(s["E"]), T_(s["g"]), T_(s["static_w"]), T_(Wc),
                      T_(s["X"][4 * c:4 * c + 4]), torch.tensor(s["y"][4 * c:4 * c + 4]))
        assert Ls[c] == pytest.approx(float(l.mean()), rel=1e-12)


# ---------------------------------------------------------------------------
# 6b. Final prediction at the updated weights ([TTT-E2E] 持续学习框架, the
#     预测 step, and the sketch's 最终预测 part)
# ---------------------------------------------------------------------------

def test_final_prediction_matches_autograd_restatement():
    """Two sequences, each at its own W_T from the inner loop: every token's
    loss equals the independent torch restatement over the whole sequence."""
    s = tiny_setup(kind="gelu", d=4, h=6, V=7, L=2, static=True, T=12)
    s2 = tiny_setup(kind="gelu", d=4, h=6, V=7, L=2, static=True, T=12, seed=5)
    WA, _, _ = run_prefill(s, 4)
    WB, _, _ = run_prefill(dict(s, X=s2["X"], y=s2["y"], W0=s2["W0"]), 3)
    X = np.stack([s["X"], s2["X"]])
    y = np.stack([s["y"], s2["y"]])
    tok, grp = O.final_prediction(s["model"], np.concatenate([WA, WB]), X, y, 4)
    assert tok.shape == (2, 12) and grp.shape == (2, 3)
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    for i, W in enumerate((WA, WB)):
        l = AM.losses("gelu", 4, 6, 2, 1e-6, T_(s["E"]), T_(s["g"]), T_(s["static_w"]), T_(W),
                      T_(X[i]), torch.tensor(y[i])).numpy()
        np.testing.assert_allclose(tok[i], l, rtol=1e-12)


def test_final_prediction_groups_are_chunk_start_losses():
    """At the chunk-start weights W_c, group c of a forward-only pass is the
    loss the inner loop reports for chunk c ([E2-TTT] O^[r] = f_{W^[r-1]}(Q^[r]))."""
    s = tiny_setup(kind="swiglu", d=4, h=5, V=7, L=2, static=True, T=12)
    _, _, Ls = run_prefill(s, 4)
    for c in range(3):
        if c == 0:
            Wc = s["W0"]
        else:
            sc = dict(s, X=s["X"][:4 * c], y=s["y"][:4 * c], eta=s["eta"][:4 * c],
                      beta=s["beta"][:4 * c], gamma=s["gamma"][:4 * c])
            Wc, _, _ = run_prefill(sc, 4)
        _, grp = O.final_prediction(s["model"], Wc, s["X"][None], s["y"][None], 4)
        assert grp[0, c] == pytest.approx(Ls[c], rel=1e-13)


def test_final_prediction_zero_head_is_log_v():
    s = tiny_setup(kind="swiglu", d=4, h=5, V=11, L=1, static=False, T=8)
    s["model"].lm_head[:] = 0.0
    tok, grp = O.final_prediction(s["model"], s["W0"], s["X"][None], s["y"][None], 2)
    np.testing.assert_allclose(tok, np.log(11.0), rtol=1e-14)
    np.testing.assert_allclose(grp, np.log(11.0), rtol=1e-14)


# ---------------------------------------------------------------------------
# 7. Planted mistakes: a plausible bug anywhere must fail one of the pins
# ---------------------------------------------------------------------------

def _must_fail(fn, *a, **k):
    with pytest.raises(AssertionError):
        fn(*a, **k)


def test_planted_mistakes_are_caught(monkeypatch):
    # (a) wrong sign of G in the aggregation
    orig = O.chunk_update_closed

    def flipped(W, M, grads, eta, beta, gamma, gscale=1.0):
        g2 = [[(-Lf, Rf) for (Lf, Rf) in blk] for blk in grads]
        return orig(W, M, g2, eta, beta, gamma, gscale)
    monkeypatch.setattr(O, "chunk_update_closed", flipped)
    _must_fail(test_chunked_sgd_uses_chunk_start_gradients, "mean")
    monkeypatch.setattr(O, "chunk_update_closed", orig)

    # (b) dropped momentum carry c_M in W_C
    orig_sk = O.scalar_kernels

    def no_cm(eta, beta, gamma):
        KW, KM, g0, b0, cM = orig_sk(eta, beta, gamma)
        return KW, KM, g0, b0, 0.0
    monkeypatch.setattr(O, "scalar_kernels", no_cm)
    _must_fail(test_closed_form_equals_recursion, "gelu", True, "mean")
    monkeypatch.setattr(O, "scalar_kernels", orig_sk)

    # (c) off-by-one suffix product (btilde_{t-1} instead of btilde_t)
    def shifted(eta, beta, gamma):
        KW, KM, g0, b0, cM = orig_sk(eta, beta, gamma)
        bt = O.suffix_products(np.asarray(beta, dtype=np.float64))
        return KW, np.asarray(eta) * bt[:-1], g0, b0, cM
    monkeypatch.setattr(O, "scalar_kernels", shifted)
    _must_fail(test_scalar_kernels_match_exact_recursion, "random")
    monkeypatch.setattr(O, "scalar_kernels", orig_sk)

    # (d) GELU derivative missing its x * pdf term
    monkeypatch.setattr(O, "gelu_grad", lambda x: 0.5 * (1.0 + O.erf(x / np.sqrt(2.0))))
    _must_fail(test_gradients_match_finite_differences, "gelu")
    monkeypatch.undo()

    # (e) RMSNorm backward without the projection term
    def _bwd_no_proj(model, W, y, fwd):
        caches, h, r, logits, lse = fwd
        n = h.shape[0]
        p = np.exp(logits - lse[:, None])
        p[np.arange(n), y] -= 1.0
        dh = (p @ model.lm_head) * model.rms_gain[None, :] * r[:, None]
        grads = [None] * model.n_blocks
        for kind, l, cache in reversed(caches):
            mats = model.static[l] if kind == "static" else W[l]
            dxb, pairs = O.mlp_backward(model.mlp, mats, cache, dh)
            if kind == "dynamic":
                grads[l] = pairs
            dh = dh + dxb
        return grads
    monkeypatch.setattr(O, "chunk_backward", _bwd_no_proj)
    _must_fail(test_gradients_match_finite_differences, "swiglu")
    monkeypatch.undo()

    # (g) LaCT: the product of the momentum factors instead of their average
    orig_lact = O.chunk_update_lact

    def lact_prod(W, M, grads, eta, beta, gamma, gscale=1.0):
        b = np.full(len(beta), np.prod(np.asarray(beta, dtype=np.float64)) ** (1.0 / len(beta)))
        return orig_lact(W, M, grads, eta, b, gamma, gscale)
    monkeypatch.setattr(O, "chunk_update_lact", lact_prod)
    _must_fail(test_lact_momentum_factor_is_the_chunk_average)
    monkeypatch.setattr(O, "chunk_update_lact", orig_lact)

    # (h) scalar heads: tau instead of 1 / tau as the momentum exponent
    orig_heads = O.scalar_heads

    def heads_tau(X, heads, bias, eta_base, alpha_base, tau):
        return orig_heads(X, heads, bias, eta_base, alpha_base, 1.0 / tau)
    monkeypatch.setattr(O, "scalar_heads", heads_tau)
    _must_fail(test_scalar_heads_at_zero_logits)
    monkeypatch.setattr(O, "scalar_heads", orig_heads)

    # (i) LayerNorm backward without its projection term
    orig_lnb = O.layer_norm_backward
    monkeypatch.setattr(O, "layer_norm_backward", lambda g, ln, rs: rs * (g - g.mean(axis=-1, keepdims=True)))
    _must_fail(test_recon_gradients_match_finite_differences)
    monkeypatch.setattr(O, "layer_norm_backward", orig_lnb)

    # (j) final prediction: groups of strided positions instead of consecutive ones
    orig_gm = O.group_means
    monkeypatch.setattr(O, "group_means", lambda loss, b: loss.reshape(b, -1).mean(axis=0))
    _must_fail(test_final_prediction_groups_are_chunk_start_losses)
    monkeypatch.setattr(O, "group_means", orig_gm)

    # (f) the residual dropped from the backward of a block
    orig_mb = O.mlp_backward

    def no_resid(kind, mats, cache, d_out):
        dx, pairs = orig_mb(kind, mats, cache, d_out)
        return dx - d_out, pairs   # cancels the residual the caller adds
    monkeypatch.setattr(O, "mlp_backward", no_resid)
    _must_fail(test_gradients_and_losses_match_autograd, "gelu", True, 3)
    monkeypatch.undo()


# ---------------------------------------------------------------------------
# The state without gradients (what the parity tests subtract to isolate the
# gradient-driven part of the final state)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rule", ["closed", "lact"])
def test_state_without_gradients_is_the_zero_head_run(rule):
    """A zero LM head gives zero gradients everywhere ([TTT-E2E] 核心方法: the
    loss reaches the weights only through the head), so the full inner loop
    must end exactly where the gradient-free recursion of Proposition 3.1 /
    LaCT's rule ends."""
    s = tiny_setup(kind="swiglu", d=4, h=6, V=7, L=2, static=True, T=12, m0=0.3)
    E0 = np.zeros_like(s["E"])
    model0 = O.make_model(s["d"], s["h"], s["V"], s["L"], "swiglu", 1e-6, E0, s["g"], s["static_w"])
    W, M, _ = run_prefill(s, 4, update=rule, model=model0)
    Wn, Mn = O.state_without_gradients(s["W0"], s["M0"], s["eta"][None], s["beta"][None], s["gamma"][None], 4,
                                       update=rule)
    np.testing.assert_allclose(W, Wn, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(M, Mn, rtol=1e-13, atol=1e-15)
    # and a nonzero head moves the state away from it
    W1, _, _ = run_prefill(s, 4, update=rule)
    assert rel(W1, Wn) > 1e-6


def test_state_without_gradients_matches_token_recursion():
    """Per-token recursion of [E2-TTT] 原始公式 with G_t = 0, token by token:
    M_t = beta_t M_{t-1}, W_t = gamma_t W_{t-1} + M_t; includes a beta = 0 and a
    gamma = 1 inside a chunk, and two sequences with their own scalars."""
    rng = np.random.default_rng(3)
    B, T, b, n = 2, 15, 5, 9
    W0 = rng.normal(size=(B, n))
    M0 = rng.normal(size=(B, n))
    eta = rng.uniform(0.0, 0.1, (B, T))
    beta = rng.uniform(0.5, 0.99, (B, T))
    gamma = rng.uniform(0.9, 1.0, (B, T))
    beta[0, 7] = 0.0
    gamma[1, 3] = 1.0
    Wn, Mn = O.state_without_gradients(W0, M0, eta, beta, gamma, b)
    for s in range(B):
        Wt, Mt = W0[s].copy(), M0[s].copy()
        for t in range(T):
            Mt = beta[s, t] * Mt
            Wt = gamma[s, t] * Wt + Mt
        np.testing.assert_allclose(Wn[s], Wt, rtol=1e-13)
        np.testing.assert_allclose(Mn[s], Mt, rtol=1e-13)
    # n_chunks stops early: two chunks = the recursion over the first 2 b tokens
    W2, M2 = O.state_without_gradients(W0[0], M0[0], eta[:1], beta[:1], gamma[:1], b, n_chunks=2)
    Wt, Mt = W0[0].copy(), M0[0].copy()
    for t in range(2 * b):
        Mt = beta[0, t] * Mt
        Wt = gamma[0, t] * Wt + Mt
    np.testing.assert_allclose(W2, Wt, rtol=1e-13)
    np.testing.assert_allclose(M2, Mt, rtol=1e-13)
