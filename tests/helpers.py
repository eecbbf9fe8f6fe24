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
    """||a - b|| / ||b|| (Frobenius).  A zero reference has no relative error:
    that is a test-design mistake, so it raises instead of quietly turning
    into an absolute norm."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    if not nb > 0:
        raise AssertionError("relative error against an all-zero reference")
    return float(np.linalg.norm(a - b) / nb)


def no_grad_state(w, x, n_chunks=None):
    """(W, M) the run would end with if every gradient were zero (fp64)."""
    B = x["eta"].shape[0]
    return oracle.state_without_gradients(
        np.asarray(x["W0"]).reshape(B, -1), np.asarray(x["M0"]).reshape(B, -1), x["eta"], x["beta"], x["gamma"],
        w.b, n_chunks=n_chunks, update="lact" if w.update_rule == "lact" else "closed")


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


# The state is stored in float32 after every chunk, so even exact update
# arithmetic leaves a rounding error of up to half an ulp of W (and M) per
# chunk; over C chunks STATE_ROUNDING * sqrt(C) * ||W|| bounds it.
STATE_ROUNDING = 4.0 * 2.0 ** -24


def grad_part_bound(tol, ref, ref_nograd, n_chunks):
    """Allowed relative error of the gradient-driven part ref - ref_nograd:
    the mode's bound plus the float32 state rounding, expressed relative to
    that part (it only matters where the part is a tiny share of the state)."""
    part = np.linalg.norm(np.asarray(ref, np.float64) - ref_nograd)
    return tol + STATE_ROUNDING * np.sqrt(max(n_chunks, 1)) * np.linalg.norm(np.asarray(ref, np.float64)) / part


def compare(w, x, gpu, ref, tol=None, tol_loss=TOL_LOSS, n_chunks=None):
    """Returns a dict of errors and asserts the tolerances.

    Besides the final W and M, the part of each that the gradients produced
    (final state minus the gradient-free state of the same scalars, see
    oracle.state_without_gradients) must meet the same relative bound, plus
    the rounding floor of a float32 state (grad_part_bound): the decayed W0
    and M0 can dominate W, and then a wrong or missing update term would hide
    inside the W bound.  ``n_chunks``: the run covered only the first chunks."""
    tol = TOL_STATE[w.precision] if tol is None else tol
    Wg, Mg, Lg, st = gpu
    Wr, Mr, Lr = ref
    assert st == 0, f"device status {st}"
    assert np.all(np.isfinite(Wg)) and np.all(np.isfinite(Mg)) and np.all(np.isfinite(Lg))
    Wn, Mn = no_grad_state(w, x, n_chunks)
    Wn, Mn = Wn.reshape(-1), Mn.reshape(-1)
    C = w.T // w.b if n_chunks is None else n_chunks
    e = dict(W=rel_fro(Wg, Wr), M=rel_fro(Mg, Mr), loss=float(np.max(np.abs(Lg - Lr))) if Lr.size else 0.0,
             dW=rel_fro(Wg - Wn, Wr - Wn), dM=rel_fro(Mg - Mn, Mr - Mn),
             dW_bound=grad_part_bound(tol, Wr, Wn, C), dM_bound=grad_part_bound(tol, Mr, Mn, C),
             grad_share_W=float(np.linalg.norm(Wr - Wn) / np.linalg.norm(Wr)))
    assert e["W"] <= tol, e
    assert e["M"] <= tol, e
    assert e["dW"] <= e["dW_bound"], e
    assert e["dM"] <= e["dM_bound"], e
    assert e["loss"] <= tol_loss, e
    return e
