"""ttt_prefill_noalloc, the allocation-free variant of ttt_prefill.

Some callers must not allocate device memory while they run: a process whose
device memory is budgeted once at start-up, a host application that owns the
allocator and forbids raw cudaMalloc, or a latency-critical loop that cannot
afford the device synchronisation cudaMalloc/cudaFree imply.  The variant keeps
its scratch in a fixed 16 MiB device array inside the library instead of a
caller-provided workspace.  This file checks, through the C ABI, that two
calls in a row give the results of the regular entry point within the parity
tolerances, and that a problem needing more scratch than the array holds is
refused with a clear error.  It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from tests import helpers as H
from weight_long_context_b200 import inputs as I

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [I.WORKLOADS["e2ttt_block"].with_(T=256), I.WORKLOADS["tiny_sgd"]]


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(h, w, x, dev):
    """Inputs and outputs are allocated by the caller before the call; the
    entry point itself allocates nothing."""
    from weight_long_context_b200 import ttt
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    hidden, tokens = t(x["hidden"]), t(x["tokens"], torch.int32)
    W, M = t(x["W0"]), t(x["M0"])
    eta, beta, gamma = t(x["eta"]), t(x["beta"]), t(x["gamma"])
    loss = torch.empty((w.batch, w.n_chunks), dtype=torch.float32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    code = ttt.load_library().ttt_prefill_noalloc(h._h, w.batch, w.T, w.b, _p(hidden), _p(tokens), _p(W), _p(M),
                                                  _p(eta), _p(beta), _p(gamma), _p(loss), stream)
    assert code == 0, ttt.ttt_last_error()
    torch.cuda.synchronize()
    assert h.device_status() == 0
    return W.cpu().numpy(), M.cpu().numpy(), loss.cpu().numpy()


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_prefill_on_two_calls(dev, w):
    x = I.make_inputs(w, seed=11, m0_scale=1e-3 if w.scalars == "e2ttt" else 0.0)
    h = H.make_handle(w, x, dev)
    Wr, Mr, Lr, st = H.run_gpu(w, x, dev, handle=h)       # the regular entry point
    assert st == 0
    tol = H.TOL_STATE[w.precision]
    for _ in range(2):                                    # two calls in a row share the scratch
        Wn, Mn, Ln = _call_noalloc(h, w, x, dev)
        assert H.rel_fro(Wn, Wr) <= tol
        assert H.rel_fro(Mn, Mr) <= tol
        assert float(np.max(np.abs(Ln - Lr))) <= H.TOL_LOSS
    h.close()


def test_noalloc_rejects_more_scratch_than_it_holds(dev):
    from weight_long_context_b200 import ttt
    w = I.WORKLOADS["batched_16"].with_(T=512, batch=2)
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    assert ttt.ttt_workspace_size(h._h, w.batch, w.T, w.b) > 16 << 20
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    args = [t(x["hidden"]), t(x["tokens"], torch.int32), t(x["W0"]), t(x["M0"]), t(x["eta"]), t(x["beta"]),
            t(x["gamma"]), torch.empty((w.batch, w.n_chunks), device=dev)]
    code = ttt.load_library().ttt_prefill_noalloc(h._h, w.batch, w.T, w.b, *[_p(a) for a in args], None)
    assert code == 4
    assert "16777216" in ttt.ttt_last_error()
    h.close()
