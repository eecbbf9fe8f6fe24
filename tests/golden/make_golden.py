"""Write the stored expected values of the full-length parity tests.

Calls only the CPU oracle (oracle/) and the seeded input generator.  For each
large workload it runs the whole inner loop in float32 on the host and stores,
as JSON: every per-chunk loss, and W_final / M_final at 2048 positions drawn
with a fixed seed (plus W_0 there, for the delta diagnostic).  The CUDA path's
full-length run is compared with these samples.

    python tests/golden/make_golden.py sgd_3b stack_128k batched_16
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


def sample_positions(n_params: int, seed: int = 1234) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(n_params, size=min(N_SAMPLES, n_params), replace=False))


def make(name: str, seed: int = 0):
    w = I.WORKLOADS[name]
    t0 = time.time()
    x = I.make_inputs(w, seed=seed)
    model = oracle.make_model(w.d, w.hidden, w.vocab, w.n_blocks, w.mlp, w.rms_eps, x["lm_head"],
                              x["rms_gain"], x["static_w"], dtype=np.float32)
    W, M, L = oracle.prefill(model, x["W0"], x["M0"], x["hidden"], x["tokens"], x["eta"], x["beta"],
                             x["gamma"], w.b, dtype=np.float32)
    idx = sample_positions(W.size)
    out = dict(workload=name, seed=seed, dtype="float32", oracle="oracle.prefill (closed form)",
               seconds=round(time.time() - t0, 1), chunk_loss=L.tolist(), sample_index=idx.tolist(),
               W=W[idx].tolist(), M=M[idx].tolist(), W0=x["W0"][idx].tolist(),
               W_norm=float(np.linalg.norm(W.astype(np.float64))),
               M_norm=float(np.linalg.norm(M.astype(np.float64))),
               dW_norm=float(np.linalg.norm(W.astype(np.float64) - x["W0"])))
    path = os.path.join(HERE, f"{name}_seed{seed}.json")
    with open(path + ".tmp", "w") as f:
        json.dump(out, f)
    os.replace(path + ".tmp", path)
    print(f"{name}: {out['seconds']} s -> {path}", flush=True)


if __name__ == "__main__":
    for nm in sys.argv[1:]:
        make(nm)
