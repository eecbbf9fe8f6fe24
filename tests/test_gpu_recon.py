"""E2-TTT's own layer on the GPU ("Rethinking Expressivity and Efficiency in
Test-Time Training": TTT modelling background, 快速权重网络实例化, Algorithm 1):
key/value reconstruction through f_W(x) = x + LN(MLP_W(x)), outputs
f_{W_0}(q_t), the chunk update; against the oracle element by element."""
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


def handle(w, dev):
    from weight_long_context_b200 import ttt
    return ttt.Handle(w.d, w.hidden, 16, 1, w.mlp, False, w.precision, None, None, None, w.rms_eps,
                      w.reduction, w.update_rule, head="recon", device=dev)


def run_gpu(w, x, dev):
    h = handle(w, dev)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    W, M = T(x["W0"]), T(x["M0"])
    loss, O = h.prefill_recon(T(x["K"]), T(x["V"]), T(x["Q"]), W, M, T(x["eta"]), T(x["beta"]), T(x["gamma"]), w.b)
    torch.cuda.synchronize()
    st = h.device_status()
    h.close()
    return W.cpu().numpy(), M.cpu().numpy(), loss.cpu().numpy(), st, O.cpu().numpy()


def run_oracle(w, x, dtype=np.float64, n_chunks=None):
    return oracle.prefill_recon(w.mlp, w.d, w.hidden, x["W0"], x["M0"], x["K"], x["V"], x["Q"], x["eta"],
                                x["beta"], x["gamma"], w.b, w.rms_eps, dtype=dtype,
                                update="lact" if w.update_rule == "lact" else "closed", reduction=w.reduction,
                                n_chunks=n_chunks)


def compare(w, x, gpu, ref):
    Wg, Mg, Lg, st, Og = gpu
    Wr, Mr, Lr, Or = ref
    e = H.compare(w, x, (Wg, Mg, Lg, st), (Wr, Mr, Lr))
    e["O"] = H.rel_fro(Og[:, :Or.shape[1]], Or)
    assert np.all(np.isfinite(Og)) and e["O"] <= H.TOL_STATE[w.precision], e
    return e


CASES = [
    # name, d, h, mlp, T, b, batch
    ("gelu", 48, 80, "gelu", 60, 20, 2),
    ("swiglu", 80, 208, "swiglu", 72, 24, 2),
    ("swiglu_tile_tail", 208, 336, "swiglu", 272, 136, 2),
]


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_recon_parity(dev, case, precision):
    name, d, h, mlp, T, b, B = case
    w = I.Workload(name, d, h, 16, 1, mlp, False, precision, T, b, B, "e2ttt", head="recon")
    x = I.make_recon_inputs(w, seed=4, m0_scale=0.001, w0_per_sequence=True)
    e = compare(w, x, run_gpu(w, x, dev), run_oracle(w, x))
    print(name, precision, e)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_recon_lact_rule(dev, precision):
    w = I.Workload("lact", 48, 80, 16, 1, "swiglu", False, precision, 60, 20, 2, "e2ttt", update_rule="lact",
                   head="recon")
    x = I.make_recon_inputs(w, seed=5, m0_scale=0.001)
    print(compare(w, x, run_gpu(w, x, dev), run_oracle(w, x)))


def test_recon_layer_dims_first_chunks(dev):
    """The 128K stack's layer dimensions (d 2048, SwiGLU h 5632, b 1024), first
    two chunks, element by element."""
    w = I.Workload("layer", 2048, 5632, 16, 1, "swiglu", False, "bf16", 2048, 1024, 1, "e2ttt", head="recon")
    x = I.make_recon_inputs(w, seed=0, m0_scale=1e-3)
    print(compare(w, x, run_gpu(w, x, dev), run_oracle(w, x, dtype=np.float32)))


def test_head_mismatch_is_rejected(dev):
    from weight_long_context_b200 import ttt
    w = I.Workload("g", 48, 80, 16, 1, "gelu", False, "fp32", 40, 20, 1, "e2ttt", head="recon")
    x = I.make_recon_inputs(w, seed=1)
    h = handle(w, dev)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    with pytest.raises(ttt.TTTError) as ei:
        h.prefill(T(x["K"]), T(x["tokens"]), T(x["W0"]), T(x["M0"]), T(x["eta"]), T(x["beta"]), T(x["gamma"]), 20)
    assert ei.value.code == 3
    h.close()
    wl = w.with_(head="lm", vocab=32)
    xl = I.make_inputs(wl, seed=1)
    hl = H.make_handle(wl, xl, dev)
    with pytest.raises(ttt.TTTError) as ei:
        hl.prefill_recon(T(x["K"]), T(x["V"]), T(x["Q"]), T(x["W0"]), T(x["M0"]), T(x["eta"]), T(x["beta"]),
                         T(x["gamma"]), 20)
    assert ei.value.code == 3
    hl.close()
