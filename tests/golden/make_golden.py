"""Write the stored expected values of the full-length parity tests.

Calls only the CPU oracle (oracle/) and the seeded input generator.  For each
large workload it runs the whole inner loop in float32 on the host and stores,
as JSON: every per-chunk loss, and W_final / M_final at 2048 positions drawn
with a fixed seed, plus W_0, M_0 and the gradient-free final state
(oracle.state_without_gradients, elementwise) at the same positions, so a test
can check the part of the state the gradients produced.  The CUDA path's
full-length run is compared with these samples.

A name with the suffix ":live" runs the workload with its E2-TTT scalar draw
but gamma = 1 (inputs scalars "e2ttt_live"): under the plain draw the state of
the 128K stack and of the batched workload decays to zero over the sequence,
so only the losses would be checked; this added case keeps W and M live.  A
further ":q" scales W0 and the static MLPs to a quarter of the workload's draw
(QUARTER below): at the full draw the residual stream of the 4-block stack
grows through its eight SwiGLU MLPs until float32 and float64 runs of the
oracle itself differ by 2.4 % on the gradient-driven part of W after two
chunks, so a parity bound there would measure the draw, not the kernels.

    python tests/golden/make_golden.py sgd_3b stack_128k batched_16 stack_128k:live:q batched_16:live
"""
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from weight_long_context_b200 import inputs as I  # noqa: E402

N_SAMPLES = 2048
QUARTER = 0.25


def scale_mlp_weights(x, s):
    """W0 and the static MLP weights of an input draw, scaled by s (in place)."""
    x["W0"] = x["W0"] * np.float32(s)
    if x["static_w"] is not None:
        x["static_w"] = x["static_w"] * np.float32(s)
    return x


def sample_positions(n_params: int, seed: int = 1234) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n_params, size=min(N_SAMPLES, n_params), replace=False))


def make(spec: str, seed: int = 0):
    name, *opts = spec.split(":")
    live, quarter = "live" in opts, "q" in opts
    w = I.WORKLOADS[name]
    if live:
        w = w.with_(scalars="e2ttt_live")
    t0 = time.time()
    x = I.make_inputs(w, seed=seed)
    if quarter:
        scale_mlp_weights(x, QUARTER)
    model = oracle.make_model(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.rms_eps, x["lm_head"],
                              x["rms_gain"], x["static_w"], dtype=np.float32)
    W, M, L = oracle.prefill(model, x["W0"], x["M0"], x["hidden"], x["tokens"], x["eta"], x["beta"],
                             x["gamma"], w.b, dtype=np.float32)
    idx = sample_positions(W.size)
    B = w.batch
    per = W.size // B
    seq = idx // per
    # gradient-free final state at the sampled positions (elementwise in the
    # state, with each position's own sequence scalars)
    Wn = np.empty(idx.size)
    Mn = np.empty(idx.size)
    for s in range(B):
        sel = seq == s
        if np.any(sel):
            Wn[sel], Mn[sel] = oracle.state_without_gradients(
                x["W0"][idx[sel]], x["M0"][idx[sel]], x["eta"][s:s + 1], x["beta"][s:s + 1], x["gamma"][s:s + 1],
                w.b)
    Wd = W.astype(np.float64)
    out = dict(workload=name, scalars=w.scalars, mlp_weight_scale=QUARTER if quarter else 1.0, seed=seed, dtype="float32", oracle="oracle.prefill (closed form)",
               seconds=round(time.time() - t0, 1), chunk_loss=L.tolist(), sample_index=idx.tolist(),
               W=W[idx].tolist(), M=M[idx].tolist(), W0=x["W0"][idx].tolist(), M0=x["M0"][idx].tolist(),
               W_nograd=Wn.tolist(), M_nograd=Mn.tolist(),
               W_norm=float(np.linalg.norm(Wd)),
               M_norm=float(np.linalg.norm(M.astype(np.float64))),
               dW_norm=float(np.linalg.norm(Wd - x["W0"])))
    path = os.path.join(HERE, f"{name}{'_live' if live else ''}{'_q' if quarter else ''}_seed{seed}.json")
    with open(path + ".tmp", "w") as f:
        json.dump(out, f)
    os.replace(path + ".tmp", path)
    print(f"{name}: {out['seconds']} s -> {path}", flush=True)


if __name__ == "__main__":
    for nm in sys.argv[1:]:
        make(nm)
