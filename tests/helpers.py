"""Shared helpers of the parity tests: run the CUDA path (through the C ABI
binding) and the oracle on the same seeded inputs and compare."""
import numpy as np

import oracle
from weight_long_context_b200 import inputs as I

# Tolerances fixed by the method statement: relative Frobenius error on the
# final W and M; absolute error on the per-chunk mean loss.
TOL_STATE = {"fp32": 1e-4, "bf16": 3e-2}
TOL_LOSS = 1e-2


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def oracle_model(w, x):
    return oracle.make_model(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.rms_eps, x["lm_head"],
                             x["rms_gain"], x["static_w"])


def run_oracle(w, x, dtype=np.float64, n_chunks=None):
    model = oracle_model(w, x)
    return oracle.prefill(model, x["W0"], x["M0"], x["hidden"], x["tokens"], x["eta"], x["beta"],
                          x["gamma"], w.b, dtype=dtype, n_chunks=n_chunks, reduction=w.reduction,
                          update="lact" if w.update_rule == "lact" else "closed")


def make_handle(w, x, dev):
    import torch
    from weight_long_context_b200 import ttt
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return ttt.Handle(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.has_static, w.precision,
                      T(x["lm_head"]), T(x["rms_gain"]),
                      T(x["static_w"]) if x["static_w"] is not None else None, w.rms_eps,
                      w.reduction, w.update_rule)


def run_gpu(w, x, dev, handle=None, return_handle=False):
    import torch
    h = handle or make_handle(w, x, dev)
    T = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    W, M = T(x["W0"]), T(x["M0"])
    loss = h.prefill(T(x["hidden"]), T(x["tokens"], torch.int32), W, M, T(x["eta"]), T(x["beta"]),
                     T(x["gamma"]), w.b)
    torch.cuda.synchronize()
    st = h.device_status()
    out = (W.cpu().numpy(), M.cpu().numpy(), loss.cpu().numpy(), st)
    if return_handle:
        return out + (h,)
    if handle is None:
        h.close()
    return out


def compare(w, x, gpu, ref, tol=None, tol_loss=TOL_LOSS):
    """Returns a dict of errors and asserts the tolerances."""
    tol = TOL_STATE[w.precision] if tol is None else tol
    Wg, Mg, Lg, st = gpu
    Wr, Mr, Lr = ref
    assert st == 0, f"device status {st}"
    e = dict(W=rel_fro(Wg, Wr), M=rel_fro(Mg, Mr) if np.any(Mr) else float(np.abs(Mg).max()),
             loss=float(np.max(np.abs(Lg - Lr))) if Lr.size else 0.0)
    # The change of W over the run: the stricter diagnostic (W is dominated by W0).
    e["dW"] = rel_fro(Wg - x["W0"], Wr - x["W0"]) if np.any(Wr - x["W0"]) else 0.0
    assert np.all(np.isfinite(Wg)) and np.all(np.isfinite(Mg)) and np.all(np.isfinite(Lg))
    assert e["W"] <= tol, e
    assert e["M"] <= tol, e
    assert e["loss"] <= tol_loss, e
    return e
