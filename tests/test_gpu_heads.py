"""Input-dependent update scalars on the GPU ("Rethinking Expressivity and
Efficiency in Test-Time Training", 依赖于输入的动态参数化) against the oracle,
alone and feeding the inner loop."""
import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from weight_long_context_b200 import inputs as I

pytestmark = pytest.mark.gpu

# Readings: eta_base 0.01, alpha_base 1, tau 16 (the ranges of the workloads'
# scalar draws: eta ~ 0.01 sigmoid(N(0,1)), beta near 0.96, gamma in (0.99, 1)).
ETA_BASE, ALPHA_BASE, TAU = 0.01, 1.0, 16.0


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _heads(d, seed):
    rng = np.random.default_rng(seed)
    return rng.normal(0, 1.0 / np.sqrt(d), (3, d)), rng.normal(0, 1.0, 3)


@pytest.mark.parametrize("B,T,d", [(2, 300, 80), (1, 1024, 2048), (3, 7, 4)])
def test_scalar_heads_match_oracle(dev, B, T, d):
    from weight_long_context_b200 import ttt
    rng = np.random.default_rng(d)
    X = rng.normal(size=(B, T, d)).astype(np.float32)
    Wh, bh = _heads(d, d + 1)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
    e, b, g = ttt.ttt_scalar_heads(t(X), t(Wh), bh, ETA_BASE, ALPHA_BASE, TAU)
    e2, b2, g2 = ttt.ttt_scalar_heads(t(X), t(Wh), bh, ETA_BASE, ALPHA_BASE, TAU)
    assert torch.equal(e, e2) and torch.equal(b, b2) and torch.equal(g, g2)
    re, rb, rg = oracle.scalar_heads(X, Wh.astype(np.float32), bh.astype(np.float32), ETA_BASE, ALPHA_BASE, TAU)
    np.testing.assert_allclose(e.cpu().numpy(), re, rtol=2e-5, atol=1e-9)
    np.testing.assert_allclose(b.cpu().numpy(), rb, rtol=2e-5, atol=1e-9)
    np.testing.assert_allclose(g.cpu().numpy(), rg, rtol=1e-6, atol=1e-9)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_heads_feed_the_inner_loop(dev, precision):
    """Scalars from the heads kernel drive the prefill; the oracle computes its
    own scalars from the same hidden rows and runs its own prefill."""
    from weight_long_context_b200 import ttt
    w = I.Workload("heads", 48, 80, 272, 2, "swiglu", True, precision, 60, 20, 2, "e2ttt")
    x = I.make_inputs(w, seed=9, m0_scale=0.01, w0_per_sequence=True)
    Wh, bh = _heads(w.d, 3)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
    e, b, g = ttt.ttt_scalar_heads(t(x["hidden"]), t(Wh), bh, ETA_BASE, ALPHA_BASE, TAU)
    xg = dict(x, eta=e.cpu().numpy(), beta=b.cpu().numpy(), gamma=g.cpu().numpy())
    re, rb, rg = oracle.scalar_heads(x["hidden"], Wh.astype(np.float32), bh.astype(np.float32),
                                     ETA_BASE, ALPHA_BASE, TAU)
    xr = dict(x, eta=re, beta=rb, gamma=rg)
    e_ = H.compare(w, xr, H.run_gpu(w, xg, dev), H.run_oracle(w, xr))
    print("heads", precision, e_)
