"""Pins of the sliding-window-attention oracle (oracle/swa_oracle.py), CPU only.

Pages by title:
  [TTT-E2E] "TTT-E2E：端到端测试时训练的长上下文语言建模" (the sketch's block,
            attention and rotary embedding; 滑动窗口注意力, 关键设计参数)
  [E2-TTT]  "Rethinking Expressivity and Efficiency in Test-Time Training"
            (原始公式, 命题3.1, 高效的逐块更新机制)
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import swa_oracle as S
from oracle import ttt_oracle as O
from tests import autograd_model as AM


def setup(kind="swiglu", d=8, H=2, h=6, V=7, L=2, static=True, T=8, window=5, seed=3, m0=0.05):
    rng = np.random.default_rng(seed)
    shapes = AM.shapes_of(kind, d, h)
    per_block = sum(r * c for r, c in shapes)
    s = dict(kind=kind, d=d, H=H, h=h, V=V, L=L, T=T, window=window)
    s["E"] = rng.normal(0, 0.5, (V, d))
    s["g"] = rng.uniform(0.5, 1.5, d)
    s["static_w"] = rng.normal(0, 0.3, L * per_block) if static else None
    s["W0"] = rng.normal(0, 0.3, L * per_block)
    s["M0"] = rng.normal(0, m0, L * per_block)
    s["attn_w"] = rng.normal(0, 0.4, (L, 4, d, d))
    s["ln_gain"] = rng.uniform(0.5, 1.5, (L, d))
    s["ln_bias"] = rng.normal(0, 0.2, (L, d))
    s["X"] = rng.normal(0, 1, (T, d))
    s["y"] = rng.integers(0, V, T)
    s["eta"] = 0.2 / (1 + np.exp(-rng.normal(size=T)))
    s["beta"] = rng.uniform(0.7, 0.99, T)
    s["gamma"] = rng.uniform(0.95, 1.0, T)
    s["model"] = O.make_model(d, h, V, L, kind, 1e-6, s["E"], s["g"], s["static_w"])
    s["swa"] = S.make_swa(d, L, H, window, s["attn_w"], s["ln_gain"], s["ln_bias"])
    return s


def run_oracle(s, b, rule="e2ttt", reduction="mean", **over):
    p = dict(s)
    p.update(over)
    W, M, Ls = S.prefill(p["model"], p["swa"], p["W0"], p["M0"], p["X"][None], p["y"][None], p["eta"][None],
                         p["beta"][None], p["gamma"][None], b, rule=rule, reduction=reduction)
    return W, M, Ls[0]


def torch_swa(s):
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    L = s["L"]
    A = s["attn_w"]
    return dict(n_heads=s["H"], window=s["window"], ln_eps=1e-5,
                Wq=[T_(A[l, 0]) for l in range(L)], Wk=[T_(A[l, 1]) for l in range(L)],
                Wv=[T_(A[l, 2]) for l in range(L)], Wo=[T_(A[l, 3]) for l in range(L)],
                ln_gain=[T_(s["ln_gain"][l]) for l in range(L)], ln_bias=[T_(s["ln_bias"][l]) for l in range(L)])


def recursion_reference(s, b, rule="e2ttt"):
    """The inner loop by its definition: per chunk, each token's gradient G_t
    = -grad (l_t / b) at the chunk-start weights (torch autograd of the
    independent restatement, earlier chunks' keys and values held fixed), then
    the per-token recursion M_t = beta_t M_{t-1} + eta_t G_t,
    W_t = gamma_t W_{t-1} + M_t ([E2-TTT] 原始公式), or LaCT's chunk rule
    ([E2-TTT] 高效的逐块更新机制)."""
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    sw = torch_swa(s)
    d, H, L = s["d"], s["H"], s["L"]
    dh = d // H
    W = T_(s["W0"])
    M = T_(s["M0"])
    kv = [(torch.zeros(H, 0, dh, dtype=torch.float64), torch.zeros(H, 0, dh, dtype=torch.float64),
           torch.zeros(0, dtype=torch.long)) for _ in range(L)]
    losses = []
    for c in range(s["T"] // b):
        sl = slice(c * b, (c + 1) * b)
        Wc = W.clone().requires_grad_(True)
        l, new_kv = AM.swa_losses(s["kind"], d, s["h"], L, 1e-6, T_(s["E"]), T_(s["g"]),
                                  T_(s["static_w"]) if s["static_w"] is not None else None, Wc,
                                  T_(s["X"][sl]), torch.tensor(s["y"][sl]), c * b, sw, kv)
        G = [-torch.autograd.grad(l[t] / b, Wc, retain_graph=True)[0] for t in range(b)]
        eta, beta, gamma = s["eta"][sl], s["beta"][sl], s["gamma"][sl]
        if rule == "lact":
            Gs = sum(float(eta[t]) * G[t] for t in range(b))
            M = float(np.mean(beta)) * M + Gs
            W = W + M
        else:
            for t in range(b):
                M = float(beta[t]) * M + float(eta[t]) * G[t]
                W = float(gamma[t]) * W + M
        W, M = W.detach(), M.detach()
        kv = [(torch.cat([kv[i][0], new_kv[i][0]], 1), torch.cat([kv[i][1], new_kv[i][1]], 1),
               torch.cat([kv[i][2], new_kv[i][2]])) for i in range(L)]
        losses.append(float(l.detach().mean()))
    return W.numpy(), M.numpy(), np.array(losses)


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300))


# ---------------------------------------------------------------------------
# Pieces against library routines and closed forms
# ---------------------------------------------------------------------------

def test_rope_is_complex_rotation():
    """Rotate-half form == (x1 + i x2) e^{i pos theta}, theta_j = base^(-2j/dh)."""
    rng = np.random.default_rng(0)
    x = rng.normal(size=(3, 5, 8))
    pos = np.array([0, 1, 7, 100, 4095])
    cos, sin = S.rope_angles(pos, 8, 10000.0)
    y = S.rope(x, cos, sin)
    theta = 10000.0 ** (-2.0 * np.arange(4) / 8)
    z = (x[..., :4] + 1j * x[..., 4:]) * np.exp(1j * pos[:, None] * theta[None, :])
    np.testing.assert_allclose(y, np.concatenate([z.real, z.imag], axis=-1), rtol=1e-12, atol=1e-12)
    # the backward is the inverse rotation (rotations are orthogonal)
    np.testing.assert_allclose(S.rope_backward(y, cos, sin), x, rtol=1e-12, atol=1e-12)


def test_layer_norm_matches_torch():
    rng = np.random.default_rng(1)
    x, g, bb = rng.normal(size=(6, 16)), rng.uniform(0.5, 1.5, 16), rng.normal(size=16)
    y, _ = S.layer_norm_affine(x, g, bb, 1e-5)
    ref = F.layer_norm(torch.tensor(x), (16,), torch.tensor(g), torch.tensor(bb), 1e-5).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_window_mask_brute_force():
    q = np.arange(8, 12)
    k = np.arange(0, 12)
    m = S.window_mask(q, k, 5)
    for i, t in enumerate(q):
        for j, kk in enumerate(k):
            assert m[i, j] == (kk <= t and t - kk < 5)


def test_attention_matches_sdpa_with_cache():
    """The sub-layer against torch's scaled_dot_product_attention with the
    same boolean window mask, earlier keys/values included."""
    s = setup(d=8, H=2, window=6)
    sw = s["swa"]
    rng = np.random.default_rng(4)
    m = 5
    Kp, Vp = rng.normal(size=(2, m, 4)), rng.normal(size=(2, m, 4))
    ppos = np.arange(3, 3 + m)
    h = rng.normal(size=(4, 8))
    pos = np.arange(8, 12)
    out, cache, (kr, v, _) = S.attention_forward(sw, 1, h, pos, (Kp, Vp, ppos))
    a = F.layer_norm(torch.tensor(h), (8,), torch.tensor(sw.ln_gain[1]), torch.tensor(sw.ln_bias[1]), 1e-5)
    q = AM.rope_complex((a @ torch.tensor(sw.Wq[1]).T).reshape(4, 2, 4).transpose(0, 1), torch.tensor(pos))
    k = AM.rope_complex((a @ torch.tensor(sw.Wk[1]).T).reshape(4, 2, 4).transpose(0, 1), torch.tensor(pos))
    vv = (a @ torch.tensor(sw.Wv[1]).T).reshape(4, 2, 4).transpose(0, 1)
    Ka = torch.cat([torch.tensor(Kp), k], 1)
    Va = torch.cat([torch.tensor(Vp), vv], 1)
    kp = torch.cat([torch.tensor(ppos), torch.tensor(pos)])
    d_ = torch.tensor(pos)[:, None] - kp[None, :]
    o = F.scaled_dot_product_attention(q, Ka, Va, attn_mask=(d_ >= 0) & (d_ < 6))
    ref = o.transpose(0, 1).reshape(4, 8) @ torch.tensor(sw.Wo[1]).T
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_window_one_is_the_value_path():
    """Window 1: each token sees only itself, the softmax is 1 and the
    sub-layer is LN(h) Wv^T Wo^T."""
    s = setup(d=8, H=2, window=1)
    sw = s["swa"]
    h = np.random.default_rng(5).normal(size=(4, 8))
    out, _, _ = S.attention_forward(sw, 0, h, np.arange(4), S.empty_kv(sw, 8))
    a, _ = S.layer_norm_affine(h, sw.ln_gain[0], sw.ln_bias[0], 1e-5)
    np.testing.assert_allclose(out, a @ sw.Wv[0].T @ sw.Wo[0].T, rtol=1e-12, atol=1e-12)


def test_window_covering_the_sequence_is_causal_attention():
    """Window >= T: a chunk's rows over the earlier chunks' history give the
    rows of plain causal attention over the whole sequence (torch SDPA with
    is_causal on equal query and key lengths)."""
    s = setup(d=8, H=2, window=10 ** 6)
    sw = s["swa"]
    rng = np.random.default_rng(11)
    h = rng.normal(size=(12, 8))
    pos = np.arange(12)
    out_all, _, (kr, v, _) = S.attention_forward(sw, 0, h, pos, S.empty_kv(sw, 8))
    _, _, hist = S.attention_forward(sw, 0, h[:8], pos[:8], S.empty_kv(sw, 8))
    out_tail, _, _ = S.attention_forward(sw, 0, h[8:], pos[8:], hist)
    np.testing.assert_allclose(out_tail, out_all[8:], rtol=1e-12, atol=1e-12)
    a = F.layer_norm(torch.tensor(h), (8,), torch.tensor(sw.ln_gain[0]), torch.tensor(sw.ln_bias[0]), 1e-5)
    split = lambda m: (a @ torch.tensor(m).T).reshape(12, 2, 4).transpose(0, 1)
    q = AM.rope_complex(split(sw.Wq[0]), torch.tensor(pos))
    k = AM.rope_complex(split(sw.Wk[0]), torch.tensor(pos))
    o = F.scaled_dot_product_attention(q, k, split(sw.Wv[0]), is_causal=True)
    ref = o.transpose(0, 1).reshape(12, 8) @ torch.tensor(sw.Wo[0]).T
    np.testing.assert_allclose(out_all, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_common_position_shift_leaves_attention_unchanged():
    """The rotary embedding makes scores depend on position differences only:
    shifting the queries' and the history's positions together changes nothing."""
    s = setup(d=8, H=2, window=6)
    sw = s["swa"]
    rng = np.random.default_rng(12)
    h0, h1 = rng.normal(size=(5, 8)), rng.normal(size=(4, 8))
    outs = []
    for shift in (0, 1000):
        _, _, hist = S.attention_forward(sw, 1, h0, np.arange(5) + shift, S.empty_kv(sw, 8))
        out, _, _ = S.attention_forward(sw, 1, h1, np.arange(5, 9) + shift, hist)
        outs.append(out)
    np.testing.assert_allclose(outs[1], outs[0], rtol=1e-9, atol=1e-11)


def test_resume_with_the_history():
    """Only (W, M) and the key/value history cross chunk boundaries: two runs
    that hand both over equal one run, bit for bit."""
    s = setup(kind="swiglu", T=12, window=7)
    mdl, sw = s["model"], s["swa"]
    shapes = mdl.mat_shapes()
    W0 = O.unpack_blocks(s["W0"].copy(), mdl.n_blocks, shapes)
    M0 = O.unpack_blocks(s["M0"].copy(), mdl.n_blocks, shapes)
    args = lambda sl: (s["X"][sl], s["y"][sl], s["eta"][sl], s["beta"][sl], s["gamma"][sl])
    W, M, L = S.prefill_sequence(mdl, sw, W0, M0, *args(slice(0, 12)), 4)
    Wa, Ma, La, kv = S.prefill_sequence(mdl, sw, W0, M0, *args(slice(0, 4)), 4, return_kv=True)
    Wb, Mb, Lb = S.prefill_sequence(mdl, sw, Wa, Ma, *args(slice(4, 12)), 4, pos0=4, kv_in=kv)
    assert all(np.array_equal(x, y) for bx, by in zip(Wb, W) for x, y in zip(bx, by))
    assert all(np.array_equal(x, y) for bx, by in zip(Mb, M) for x, y in zip(bx, by))
    np.testing.assert_array_equal(np.concatenate([La, Lb]), L)


# ---------------------------------------------------------------------------
# The inner loop against its definition
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["gelu", "swiglu"])
@pytest.mark.parametrize("rule", ["e2ttt", "lact"])
def test_prefill_matches_per_token_recursion(kind, rule):
    """Two chunks, a window shorter than two chunks (chunk 1 sees part of
    chunk 0): Proposition 3.1 over weighted backward passes == the per-token
    recursion over autograd gradients of the independent restatement."""
    s = setup(kind=kind, T=8, window=5)
    W, M, Ls = run_oracle(s, 4, rule=rule)
    Wr, Mr, Lr = recursion_reference(s, 4, rule=rule)
    assert rel(W, Wr) < 1e-10 and rel(M, Mr) < 1e-10, (rel(W, Wr), rel(M, Mr))
    np.testing.assert_allclose(Ls, Lr, rtol=1e-11)


def test_zero_output_projection_is_the_plain_loop():
    """Wo = 0 removes the attention sub-layers: the result is the pinned
    inner loop without attention (row-local gradients, one backward)."""
    s = setup(kind="swiglu", T=12, window=5, L=3)
    s["attn_w"][:, 3] = 0.0
    s["swa"] = S.make_swa(s["d"], s["L"], s["H"], s["window"], s["attn_w"], s["ln_gain"], s["ln_bias"])
    W, M, Ls = run_oracle(s, 4)
    Wp, Mp, Lp = O.prefill(s["model"], s["W0"], s["M0"], s["X"][None], s["y"][None], s["eta"][None],
                           s["beta"][None], s["gamma"][None], 4)
    assert rel(W, Wp) < 1e-12 and rel(M, Mp) < 1e-12
    np.testing.assert_allclose(Ls, Lp[0], rtol=1e-12)


def test_attention_makes_gradients_non_local():
    """With attention, weighting each token's own row afterwards (the row-local
    shortcut of the plain loop) is not the update: the weighted backward
    differs from it, and only the weighted backward matches the recursion."""
    s = setup(kind="gelu", T=4, window=4)
    W, M, _ = run_oracle(s, 4)
    Wl, _ = _row_local_update(s, 4)
    assert rel(W, O.pack_blocks(Wl)) > 1e-4


def _row_local_update(s, b):
    """One chunk with the plain loop's shortcut: one unweighted backward, each
    row's factor pair weighted by that token's K afterwards."""
    mdl, sw = s["model"], s["swa"]
    W0 = O.unpack_blocks(s["W0"].copy(), mdl.n_blocks, mdl.mat_shapes())
    M0 = O.unpack_blocks(s["M0"].copy(), mdl.n_blocks, mdl.mat_shapes())
    kv = [S.empty_kv(sw, s["d"]) for _ in range(mdl.n_blocks)]
    _, fwd, _ = S.chunk_forward(mdl, sw, W0, s["X"][:b], s["y"][:b], 0, kv)
    caches, h, r, logits, lse = fwd
    p = np.exp(logits - lse[:, None])
    p[np.arange(b), s["y"][:b]] -= 1.0
    gdz = (p @ mdl.lm_head) * mdl.rms_gain[None, :]
    dot = np.sum(gdz * h, axis=1)
    dh = gdz * r[:, None] - h * (r ** 3 * dot / mdl.d)[:, None]
    pairs = [None] * mdl.n_blocks
    for kind, l, cache in reversed(caches):
        if kind == "attn":
            dh = dh + S.attention_backward(sw, l, cache, dh)
            continue
        mats = mdl.static[l] if kind == "static" else W0[l]
        dx, pr = O.mlp_backward(mdl.mlp, mats, cache, dh)
        if kind == "dynamic":
            pairs[l] = pr
            if l == 0:
                break
        dh = dh + dx
    return O.chunk_update_closed(W0, M0, pairs, s["eta"][:b], s["beta"][:b], s["gamma"][:b], 1.0 / b)


# ---------------------------------------------------------------------------
# Final prediction with the attention blocks
# ---------------------------------------------------------------------------

def test_final_prediction_is_one_pass_over_the_sequence():
    """At fixed weights every key and value comes from the same W, so the
    grouped pass equals one pass of the independent restatement over the whole
    sequence (torch), for any group size."""
    s = setup(kind="swiglu", T=12, window=5)
    W = s["W0"]
    T_ = lambda a: torch.tensor(a, dtype=torch.float64)
    H, dh = s["H"], s["d"] // s["H"]
    kv0 = [(torch.zeros(H, 0, dh, dtype=torch.float64), torch.zeros(H, 0, dh, dtype=torch.float64),
            torch.zeros(0, dtype=torch.long)) for _ in range(s["L"])]
    ref, _ = AM.swa_losses(s["kind"], s["d"], s["h"], s["L"], 1e-6, T_(s["E"]), T_(s["g"]), T_(s["static_w"]),
                           T_(W), T_(s["X"]), torch.tensor(s["y"]), 0, torch_swa(s), kv0)
    for b in (3, 4, 12):
        tok, grp = S.final_prediction(s["model"], s["swa"], W, s["X"][None], s["y"][None], b)
        np.testing.assert_allclose(tok[0], ref.numpy(), rtol=1e-11)
        np.testing.assert_allclose(grp[0], ref.numpy().reshape(-1, b).mean(axis=1), rtol=1e-11)


def test_final_prediction_zero_output_projection_is_the_plain_prediction():
    s = setup(kind="gelu", T=8, window=3)
    s["attn_w"][:, 3] = 0.0
    sw = S.make_swa(s["d"], s["L"], s["H"], s["window"], s["attn_w"], s["ln_gain"], s["ln_bias"])
    tok, grp = S.final_prediction(s["model"], sw, s["W0"], s["X"][None], s["y"][None], 4)
    tok_p, grp_p = O.final_prediction(s["model"], s["W0"], s["X"][None], s["y"][None], 4)
    np.testing.assert_allclose(tok, tok_p, rtol=1e-12)
    np.testing.assert_allclose(grp, grp_p, rtol=1e-12)


def test_final_prediction_first_group_is_the_first_chunk_loss():
    s = setup(kind="swiglu", T=8, window=6)
    _, _, Ls = run_oracle(s, 4)
    _, grp = S.final_prediction(s["model"], s["swa"], s["W0"], s["X"][None], s["y"][None], 4)
    assert grp[0, 0] == pytest.approx(Ls[0], rel=1e-13)


# ---------------------------------------------------------------------------
# Planted mistakes
# ---------------------------------------------------------------------------

def _must_fail(fn, *a, **k):
    with pytest.raises(AssertionError):
        fn(*a, **k)


def test_planted_mistakes_are_caught(monkeypatch):
    # (a) window one key too wide
    monkeypatch.setattr(S, "window_mask", lambda q, k, w: ((np.asarray(q)[:, None] - np.asarray(k)[None, :] >= 0)
                                                          & (np.asarray(q)[:, None] - np.asarray(k)[None, :] <= w)))
    _must_fail(test_prefill_matches_per_token_recursion, "gelu", "e2ttt")
    monkeypatch.undo()

    # (b) rotary backward with the forward rotation
    monkeypatch.setattr(S, "rope_backward", S.rope)
    _must_fail(test_prefill_matches_per_token_recursion, "swiglu", "e2ttt")
    monkeypatch.undo()

    # (c) softmax backward without the row term D
    orig = S.attention_backward

    def no_D(sw, l, cache, g_out):
        lnc, qr, Ka, Va, p, o, cos, sin, mprev = cache
        return orig(sw, l, (lnc, qr, Ka, Va, p, np.zeros_like(o), cos, sin, mprev), g_out)
    monkeypatch.setattr(S, "attention_backward", no_D)
    _must_fail(test_prefill_matches_per_token_recursion, "gelu", "lact")
    monkeypatch.undo()

    # (d) the row-local shortcut in place of the weighted backward
    def row_local(s, b, rule="e2ttt", reduction="mean", **over):
        W, M = _row_local_update(s, b)
        return O.pack_blocks(W), O.pack_blocks(M), np.zeros(1)
    _check_one_chunk_against_recursion(run_oracle)
    _must_fail(_check_one_chunk_against_recursion, row_local)


def _check_one_chunk_against_recursion(runner):
    s = setup(kind="gelu", T=4, window=4)
    W, M, _ = runner(s, 4)
    Wr, Mr, _ = recursion_reference(s, 4)
    assert rel(W, Wr) < 1e-10 and rel(M, Mr) < 1e-10
