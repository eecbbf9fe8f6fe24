"""Blocks with frozen sliding-window attention on the GPU ("TTT-E2E：端到端测试时
训练的长上下文语言建模": the sketch's TTTE2EBlock and TTTSelfAttention;
滑动窗口注意力), against the oracle's restatement (oracle/swa_oracle.py), whose
update takes sum_t K_t G_t as the gradient of the K-weighted chunk loss.

The attention weights are drawn with standard deviation 1/sqrt(d), so that the
scores are O(1) and the attention sub-layers carry as much of the gradient as
the MLPs (a small draw would leave the cross-token terms untested).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import swa_oracle as S
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


def run_both(w, x, a, dev, dtype=np.float64, n_chunks=None):
    h = H.make_handle(w, x, dev)
    h.set_attention(w.attn_heads, w.attn_window, t(a["attn_w"], dev), t(a["ln_gain"], dev), t(a["ln_bias"], dev))
    gpu = H.run_gpu(w, x, dev, handle=h)
    h.close()
    sw = S.make_swa(w.d, w.n_blocks, w.attn_heads, w.attn_window, a["attn_w"], a["ln_gain"], a["ln_bias"])
    ref = S.prefill(H.oracle_model(w, x), sw, x["W0"], x["M0"], x["hidden"], x["tokens"], x["eta"], x["beta"],
                    x["gamma"], w.b, dtype=dtype, rule=w.update_rule, reduction=w.reduction, n_chunks=n_chunks)
    return gpu, ref


CASES = [
    # name, d, h, V, L, mlp, static, T, b, batch, heads, window
    ("gelu_2blk", 64, 96, 272, 2, "gelu", False, 48, 16, 2, 4, 24),
    ("swiglu_3blk_static", 128, 80, 400, 3, "swiglu", True, 64, 16, 1, 4, 40),
    ("swiglu_dh64", 256, 176, 528, 2, "swiglu", False, 96, 32, 2, 4, 48),
]


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_swa_parity(dev, case, precision):
    name, d, hh, V, L, mlp, st, T, b, B, nh, win = case
    w = I.Workload(name, d, hh, V, L, mlp, st, precision, T, b, B, "e2ttt", attn_heads=nh, attn_window=win)
    x = I.make_inputs(w, seed=7, m0_scale=0.01, w0_per_sequence=True)
    a = I.make_swa_inputs(w, seed=7, scale=1.0 / np.sqrt(d))
    gpu, ref = run_both(w, x, a, dev)
    e = H.compare(w, x, gpu, ref)
    print(name, precision, e)


def test_swa_lact(dev):
    name, d, hh, V, L, mlp, st, T, b, B, nh, win = CASES[1]
    w = I.Workload(name, d, hh, V, L, mlp, st, "fp32", T, b, B, "e2ttt", update_rule="lact", attn_heads=nh,
                   attn_window=win)
    x = I.make_inputs(w, seed=3, m0_scale=0.01)
    a = I.make_swa_inputs(w, seed=3, scale=1.0 / np.sqrt(d))
    gpu, ref = run_both(w, x, a, dev)
    print("lact", H.compare(w, x, gpu, ref))


def test_swa_window_shorter_than_chunk(dev):
    """k < b: the window binds inside the chunk too."""
    w = I.Workload("short", 64, 96, 272, 2, "gelu", True, "fp32", 48, 16, 1, "e2ttt", attn_heads=2, attn_window=5)
    x = I.make_inputs(w, seed=2, m0_scale=0.01)
    a = I.make_swa_inputs(w, seed=2, scale=1.0 / np.sqrt(64))
    gpu, ref = run_both(w, x, a, dev)
    print("short window", H.compare(w, x, gpu, ref))


def test_zero_output_projection_matches_plain_gpu_path(dev):
    """Wo = 0: the attention path (with its two weighted streams below the top
    block) gives the plain GPU inner loop's result."""
    name, d, hh, V, L, mlp, st, T, b, B, nh, win = CASES[1]
    w = I.Workload(name, d, hh, V, L, mlp, st, "fp32", T, b, B, "e2ttt", attn_heads=nh, attn_window=win)
    x = I.make_inputs(w, seed=5, m0_scale=0.01)
    a = I.make_swa_inputs(w, seed=5, scale=1.0 / np.sqrt(d))
    a["attn_w"][:, 3] = 0.0
    h = H.make_handle(w, x, dev)
    h.set_attention(nh, win, t(a["attn_w"], dev), t(a["ln_gain"], dev), t(a["ln_bias"], dev))
    Wa, Ma, La, sa = H.run_gpu(w, x, dev, handle=h)
    h.set_attention(0, 0, None, None, None)
    Wp, Mp, Lp, sp = H.run_gpu(w, x, dev, handle=h)
    h.close()
    assert sa == 0 and sp == 0
    assert H.rel_fro(Wa, Wp) < 1e-5 and H.rel_fro(Ma, Mp) < 1e-5
    np.testing.assert_allclose(La, Lp, rtol=1e-5)


def test_swa_full_dims_first_chunks(dev):
    """The 128K stack with attention (32 heads of 64, window 8192): the
    benchmark's model and chunk size and its launch shapes, first two chunks,
    float32 oracle.  The MLP weights are drawn at a quarter of the workload's
    scale: at the workload's own draw the residual stream grows without bound
    through the eight SwiGLU MLPs, and two float32 programs (this GPU path in
    fp32 and the oracle) already disagree by 1.6 % on W there, as the plain
    path's bf16 run does by 2.5 %; at the smaller draw the stream stays O(1),
    the attention weights (std 0.02, O(1) scores) still carry the gradient
    between tokens, and the bound tests the kernels rather than the conditioning."""
    w = I.WORKLOADS["stack_128k_swa"].with_(T=2 * 1024)
    x = I.make_inputs(w, seed=0, m0_scale=1e-3)
    x["W0"] = x["W0"] * np.float32(0.25)
    x["static_w"] = x["static_w"] * np.float32(0.25)
    a = I.make_swa_inputs(w, seed=0)
    gpu, ref = run_both(w, x, a, dev, dtype=np.float32)
    print("stack_128k_swa", H.compare(w, x, gpu, ref))


def test_attention_argument_errors(dev):
    from weight_long_context_b200 import ttt
    w = I.Workload("err", 64, 96, 272, 2, "gelu", False, "bf16", 48, 16, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    a = I.make_swa_inputs(w, seed=0)
    args = (t(a["attn_w"], dev), t(a["ln_gain"], dev), t(a["ln_bias"], dev))
    with pytest.raises(ttt.TTTError) as ei:
        h.set_attention(3, 8, *args)            # d % heads
    assert ei.value.code == 2
    with pytest.raises(ttt.TTTError) as ei:
        h.set_attention(8, 8, *args)            # head size 8 is not a multiple of 16
    assert ei.value.code == 2
    h.set_attention(4, 8, *args)
    x2 = I.make_inputs(w.with_(T=48, b=12), seed=0)
    with pytest.raises(ttt.TTTError) as ei:     # b % 8
        H.run_gpu(w.with_(b=12), x2, dev, handle=h)
    assert ei.value.code == 2
    with pytest.raises(ttt.TTTError) as ei:
        h.predict(t(x["hidden"], dev), t(x["tokens"], dev, torch.int32), t(x["W0"], dev), 16)
    assert ei.value.code == 3
    h.close()
