"""An independent restatement of the per-token loss in torch (float64, CPU), used
only to pin the numpy oracle: gradients come from torch autograd, not from the
oracle's hand-written backward.

Model ("TTT-E2E：端到端测试时训练的长上下文语言建模", 核心方法; dynamic MLP forms
from "Rethinking Expressivity and Efficiency in Test-Time Training",
快速权重网络实例化): per block, optional frozen static MLP then the dynamic MLP,
each with a residual; frozen RMSNorm; frozen LM head; next-token cross-entropy
per token.
"""
import torch
import torch.nn.functional as F


def _mlp(kind, mats, x):
    if kind == "gelu":
        w1, w2 = mats
        return F.gelu(x @ w1.T, approximate="none") @ w2.T
    w1, w2, w3 = mats
    return (F.silu(x @ w1.T) * (x @ w2.T)) @ w3.T


def split_blocks(flat, n_blocks, shapes):
    out, off = [], 0
    for _ in range(n_blocks):
        blk = []
        for r, c in shapes:
            blk.append(flat[off:off + r * c].reshape(r, c))
            off += r * c
        out.append(blk)
    return out


def shapes_of(kind, d, h):
    return [(h, d), (d, h)] if kind == "gelu" else [(h, d), (h, d), (d, h)]


def losses(kind, d, h, n_blocks, eps, E, g, static_flat, W_flat, X, y):
    """Per-token losses (torch tensors, float64)."""
    shapes = shapes_of(kind, d, h)
    Wb = split_blocks(W_flat, n_blocks, shapes)
    Sb = split_blocks(static_flat, n_blocks, shapes) if static_flat is not None else None
    hcur = X
    for l in range(n_blocks):
        if Sb is not None:
            hcur = hcur + _mlp(kind, Sb[l], hcur)
        hcur = hcur + _mlp(kind, Wb[l], hcur)
    z = hcur * torch.rsqrt(hcur.pow(2).mean(dim=1, keepdim=True) + eps) * g
    logits = z @ E.T
    return F.cross_entropy(logits, y, reduction="none")


def per_token_grads(kind, d, h, n_blocks, eps, E, g, static_flat, W_flat, X, y):
    """[n, n_params] per-token gradients by autograd."""
    W = W_flat.clone().requires_grad_(True)
    L = losses(kind, d, h, n_blocks, eps, E, g, static_flat, W, X, y)
    rows = []
    for t in range(L.shape[0]):
        (gt,) = torch.autograd.grad(L[t], W, retain_graph=True)
        rows.append(gt.clone())
    return torch.stack(rows), L.detach()


def recon_losses(kind, d, h, eps, W_flat, K, V):
    """Per-token reconstruction losses of E2-TTT's layer ("Rethinking
    Expressivity and Efficiency in Test-Time Training", 快速权重网络实例化 and
    the TTT modelling background): f(k) = k + LayerNorm(MLP(k)) without affine
    parameters, loss = mean squared error against v (torch tensors, float64)."""
    (mats,) = split_blocks(W_flat, 1, shapes_of(kind, d, h))
    f = K + F.layer_norm(_mlp(kind, mats, K), (d,), eps=eps)
    return F.mse_loss(f, V, reduction="none").mean(dim=1)


def recon_outputs(kind, d, h, eps, W_flat, Q):
    (mats,) = split_blocks(W_flat, 1, shapes_of(kind, d, h))
    return Q + F.layer_norm(_mlp(kind, mats, Q), (d,), eps=eps)


# ---------------------------------------------------------------------------
# Blocks with frozen sliding-window attention in front of the MLPs
# ("TTT-E2E：端到端测试时训练的长上下文语言建模", the sketch's TTTE2EBlock,
# TTTSelfAttention and RotaryEmbedding; causal window, no biases).  Written with
# library routines where one exists: F.layer_norm, F.scaled_dot_product_attention
# with a boolean mask, and the rotary embedding as a complex multiplication.
# ---------------------------------------------------------------------------

def rope_complex(x, pos, base=10000.0):
    """Rotary embedding as (x_first_half + i x_second_half) * exp(i pos theta_j)."""
    dh = x.shape[-1]
    half = dh // 2
    theta = torch.pow(torch.tensor(base, dtype=torch.float64),
                      -2.0 * torch.arange(half, dtype=torch.float64) / dh)
    ang = pos.to(torch.float64)[:, None] * theta[None, :]
    z = torch.complex(x[..., :half], x[..., half:]) * torch.polar(torch.ones_like(ang), ang)
    return torch.cat([z.real, z.imag], dim=-1)


def swa_losses(kind, d, h, n_blocks, eps, E, g, static_flat, W_flat, X, y, pos0, swa, kv):
    """Per-token losses of one chunk (rows X at positions pos0..) and the
    chunk's rotated keys and values per block (detached).

    swa: dict with n_heads, window, ln_eps and per-block lists Wq, Wk, Wv, Wo,
    ln_gain, ln_bias; kv: per block (K [H, m, dh], V [H, m, dh], positions [m])."""
    n = X.shape[0]
    H = swa["n_heads"]
    dh = d // H
    shapes = shapes_of(kind, d, h)
    Wb = split_blocks(W_flat, n_blocks, shapes)
    Sb = split_blocks(static_flat, n_blocks, shapes) if static_flat is not None else None
    pos = torch.arange(pos0, pos0 + n)
    hcur = X
    new_kv = []
    for l in range(n_blocks):
        a = F.layer_norm(hcur, (d,), swa["ln_gain"][l], swa["ln_bias"][l], swa["ln_eps"])
        split = lambda m: (a @ m.T).reshape(n, H, dh).transpose(0, 1)
        q = rope_complex(split(swa["Wq"][l]), pos)
        k = rope_complex(split(swa["Wk"][l]), pos)
        v = split(swa["Wv"][l])
        Kp, Vp, pp = kv[l]
        Ka, Va, kp = torch.cat([Kp, k], 1), torch.cat([Vp, v], 1), torch.cat([pp, pos])
        delta = pos[:, None] - kp[None, :]
        mask = (delta >= 0) & (delta < swa["window"])
        o = F.scaled_dot_product_attention(q, Ka, Va, attn_mask=mask)
        hcur = hcur + o.transpose(0, 1).reshape(n, d) @ swa["Wo"][l].T
        new_kv.append((k.detach(), v.detach(), pos))
        if Sb is not None:
            hcur = hcur + _mlp(kind, Sb[l], hcur)
        hcur = hcur + _mlp(kind, Wb[l], hcur)
    z = hcur * torch.rsqrt(hcur.pow(2).mean(dim=1, keepdim=True) + eps) * g
    return F.cross_entropy(z @ E.T, y, reduction="none"), new_kv
