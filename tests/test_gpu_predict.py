"""Final prediction at fixed fast weights on the GPU ("TTT-E2E：端到端测试时训练的
长上下文语言建模", 持续学习框架: the 预测 step, and the final-prediction part of
its inner-loop sketch): the whole sequence scored again at W, forward only,
against the oracle's final_prediction.

Tolerances: the group losses (means of b consecutive positions) use the
chunk-loss bound of the inner loop (1e-2 absolute).  The vector of token
losses uses the inner loop's bound on its state vectors, relative Frobenius
1e-4 (fp32 operands) and 3e-2 (bf16 operands).  A max-abs bound per token
does not hold for bf16: where the residual stream grows through stacked
SwiGLU blocks (the 128K stack's synthetic W0 drives row norms far past unit
scale by the last block), the 2^-9 rounding of each block's bf16 input
compounds through the blocks and single tokens move by ~0.1 while the group
means stay within 1e-3.  Rounding the same operands to bf16 in a float32
numpy forward gives max 0.128, mean 0.030, relative Frobenius 3.5e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from weight_long_context_b200 import inputs as I

pytestmark = pytest.mark.gpu



@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def t(a, dev, dt=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)


def gpu_predict(w, x, W, dev, b, handle=None):
    h = handle or H.make_handle(w, x, dev)
    grp, tok = h.predict(t(x["hidden"], dev), t(x["tokens"], dev, torch.int32), t(W, dev), b, token_loss=True)
    torch.cuda.synchronize()
    st = h.device_status()
    out = grp.cpu().numpy(), tok.cpu().numpy(), st
    if handle is None:
        h.close()
    return out


def oracle_predict(w, x, W, b, dtype=np.float64):
    return oracle.final_prediction(H.oracle_model(w, x), W, x["hidden"], x["tokens"], b, dtype=dtype)


def check(w, gpu, ref):
    grp, tok, st = gpu
    tok_r, grp_r = ref
    assert st == 0, f"device status {st}"
    assert np.all(np.isfinite(tok)) and np.all(np.isfinite(grp))
    e = dict(group=float(np.max(np.abs(grp - grp_r))), token=H.rel_fro(tok, tok_r),
             token_max=float(np.max(np.abs(tok - tok_r))))
    assert e["group"] <= H.TOL_LOSS, e
    assert e["token"] <= H.TOL_STATE[w.precision], e
    return e


RAGGED = [
    # name, d, h, V, L, mlp, static, T, b, batch
    ("gelu_1blk", 80, 208, 528, 1, "gelu", False, 72, 24, 2),
    ("swiglu_2blk_static", 48, 80, 272, 2, "swiglu", True, 60, 20, 2),
    ("swiglu_tile_tail", 208, 336, 1040, 1, "swiglu", False, 272, 136, 2),
]


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("case", RAGGED, ids=[c[0] for c in RAGGED])
def test_predict_ragged_parity(dev, case, precision):
    """Per-sequence weights, several tiles and a ragged tail in every dimension."""
    name, d, h, V, L, mlp, st, T, b, B = case
    w = I.Workload(name, d, h, V, L, mlp, st, precision, T, b, B, "e2ttt")
    x = I.make_inputs(w, seed=9, w0_per_sequence=True)
    e = check(w, gpu_predict(w, x, x["W0"], dev, b), oracle_predict(w, x, x["W0"], b))
    print(name, precision, e)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_predict_after_the_inner_loop(dev, precision):
    """The sketch's order: the inner loop gives W_T, then the forward-only pass
    at W_T; each side feeds its own W_T into its own prediction."""
    name, d, h, V, L, mlp, st, T, b, B = RAGGED[1]
    w = I.Workload(name, d, h, V, L, mlp, st, precision, T, b, B, "e2ttt")
    x = I.make_inputs(w, seed=4, m0_scale=0.01, w0_per_sequence=True)
    Wg, _, _, s = H.run_gpu(w, x, dev)
    assert s == 0
    Wr, _, _ = H.run_oracle(w, x)
    e = check(w, gpu_predict(w, x, Wg, dev, b), oracle_predict(w, x, Wr, b))
    print("after inner loop", precision, e)


@pytest.mark.parametrize("b", [4, 12, 60])
def test_predict_pass_size_only_groups(dev, b):
    """The rows per pass change only the grouping: every token's loss matches
    the oracle for any divisor of T, down to one pass over the whole sequence."""
    name, d, h, V, L, mlp, st, T, _, B = RAGGED[1]
    w = I.Workload(name, d, h, V, L, mlp, st, "fp32", T, b, B, "e2ttt")
    x = I.make_inputs(w, seed=6, w0_per_sequence=True)
    check(w, gpu_predict(w, x, x["W0"], dev, b), oracle_predict(w, x, x["W0"], b))


def test_first_group_is_the_first_chunk_loss(dev):
    """At W_0 the first group of the prediction is the loss the inner loop
    reports for its first chunk (the same forward, at the chunk-start weights)."""
    name, d, h, V, L, mlp, st, T, b, B = RAGGED[0]
    w = I.Workload(name, d, h, V, L, mlp, st, "bf16", T, b, B, "e2ttt")
    x = I.make_inputs(w, seed=8, w0_per_sequence=True)
    _, _, loss, s = H.run_gpu(w, x, dev)
    grp, _, s2 = gpu_predict(w, x, x["W0"], dev, b)
    assert s == 0 and s2 == 0
    np.testing.assert_allclose(grp[:, 0], loss[:, 0], rtol=1e-6, atol=0)


def test_predict_full_dims_two_passes(dev):
    """The 128K stack's model (4 blocks, SwiGLU with static MLPs, V = 32000),
    two passes of 1024 rows, every token against the oracle in float32."""
    w = I.WORKLOADS["stack_128k"]
    w = w.with_(T=2 * 1024, b=1024)
    x = I.make_inputs(w, seed=0)
    e = check(w, gpu_predict(w, x, x["W0"], dev, w.b), oracle_predict(w, x, x["W0"], w.b, dtype=np.float32))
    print("stack_128k predict", e)


def test_predict_full_length_sampled(dev):
    """The benchmark's launch configuration: the full 131072-token sequence in
    passes of 8192 rows.  Sampled tokens against the oracle row by row; every
    group loss equals the mean of its own token losses (a property at any
    size)."""
    w = I.WORKLOADS["stack_128k"].with_(b=8192)
    x = I.make_inputs(w, seed=0)
    grp, tok, st = gpu_predict(w, x, x["W0"], dev, w.b)
    assert st == 0
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(w.T, 48, replace=False))
    ref = oracle.token_losses(H.oracle_model(w, x), x["W0"], x["hidden"][0, rows], x["tokens"][0, rows],
                              dtype=np.float32)
    err = H.rel_fro(tok[0, rows], ref)
    assert err <= H.TOL_STATE[w.precision], err
    means = tok[0].astype(np.float64).reshape(-1, w.b).mean(axis=1)
    np.testing.assert_allclose(grp[0], means, rtol=1e-5, atol=0)
    print("stack_128k full length", err)


def test_predict_bad_token_and_wrong_head(dev):
    from weight_long_context_b200 import ttt
    w = I.Workload("tok", 32, 32, 64, 1, "gelu", False, "bf16", 32, 16, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    x["tokens"][0, 7] = -1
    *_, st = gpu_predict(w, x, x["W0"], dev, 16)
    assert st == 5
    h = ttt.Handle(32, 32, 0, 1, "gelu", False, "bf16", None, None, None, head="recon", device=dev)
    with pytest.raises(ttt.TTTError) as ei:
        h.predict(t(x["hidden"], dev), t(x["tokens"], dev, torch.int32), t(x["W0"], dev), 16)
    assert ei.value.code == 3
    h.close()


def test_predict_empty_is_noop(dev):
    name, d, h, V, L, mlp, st, T, b, B = RAGGED[0]
    w = I.Workload(name, d, h, V, L, mlp, st, "bf16", T, b, B, "e2ttt")
    x = I.make_inputs(w, seed=1)
    hd = H.make_handle(w, x, dev)
    empty = torch.empty((0, T, d), dtype=torch.float32, device=dev)
    grp, tok = hd.predict(empty, torch.empty((0, T), dtype=torch.int32, device=dev),
                          torch.empty(0, dtype=torch.float32, device=dev), b, token_loss=True)
    assert grp.shape == (0, T // b) and tok.shape == (0, T)
    hd.close()
