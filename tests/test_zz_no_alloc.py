"""ttt_prefill_noalloc, the allocation-free variant of ttt_prefill.

Some callers must not allocate device memory while they run: a process whose
device memory is budgeted once at start-up, a host application that owns the
allocator and forbids raw cudaMalloc, or a latency-critical loop that cannot
afford the device synchronisation cudaMalloc/cudaFree imply.  The variant keeps
its scratch in a fixed 16 MiB device array inside the library instead of a
caller-provided workspace.  This file checks, through the C ABI, that two
calls in a row give the results of the regular entry point bit for bit (and
so the oracle's within the parity tolerances), that the calls leave the device
memory in use unchanged, that the attention blocks run on it too, and that a
problem needing more scratch than the array holds is refused with a clear
error.  It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from tests import helpers as H
from weight_long_context_b200 import inputs as I

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [I.WORKLOADS["e2ttt_block"].with_(T=256), I.WORKLOADS["tiny_sgd"]]
# frozen sliding-window attention in the blocks: the same entry point serves it
SWA_CASE = I.Workload("noalloc_swa", 64, 96, 272, 2, "gelu", False, "bf16", 48, 16, 2, "e2ttt", attn_heads=4,
                      attn_window=24)


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(w, x, dev):
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    return dict(hidden=t(x["hidden"]), tokens=t(x["tokens"], torch.int32), W=t(x["W0"]), M=t(x["M0"]),
                eta=t(x["eta"]), beta=t(x["beta"]), gamma=t(x["gamma"]),
                loss=torch.empty((w.batch, w.n_chunks), dtype=torch.float32, device=dev))


def _call_noalloc(h, w, a, dev):
    """Inputs and outputs (a, from _inputs) are allocated by the caller before
    the call; the entry point itself allocates nothing."""
    from weight_long_context_b200 import ttt
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    code = ttt.load_library().ttt_prefill_noalloc(h._h, w.batch, w.T, w.b, _p(a["hidden"]), _p(a["tokens"]),
                                                  _p(a["W"]), _p(a["M"]), _p(a["eta"]), _p(a["beta"]),
                                                  _p(a["gamma"]), _p(a["loss"]), stream)
    assert code == 0, ttt.ttt_last_error()


def _two_calls_match_prefill(h, w, x, dev):
    """The regular entry point first, then two allocation-free calls in a row
    on fresh copies of the inputs: both must give its results bit for bit
    (the same kernels on the same inputs, eager instead of from a graph) and
    neither may change the device memory in use."""
    Wr, Mr, Lr, st = H.run_gpu(w, x, dev, handle=h)
    assert st == 0
    runs = [_inputs(w, x, dev), _inputs(w, x, dev)]
    torch.cuda.synchronize()
    used_torch = torch.cuda.memory_allocated(dev)
    free0 = torch.cuda.mem_get_info(dev)[0]
    for a in runs:
        _call_noalloc(h, w, a, dev)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0, "device memory changed across the allocation-free calls"
    assert torch.cuda.memory_allocated(dev) == used_torch
    assert h.device_status() == 0
    for a in runs:
        assert np.array_equal(a["W"].cpu().numpy(), Wr)
        assert np.array_equal(a["M"].cpu().numpy(), Mr)
        assert np.array_equal(a["loss"].cpu().numpy(), Lr)
    return Wr, Mr, Lr


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_prefill_on_two_calls(dev, w):
    x = I.make_inputs(w, seed=11, m0_scale=1e-3 if w.scalars == "e2ttt" else 0.0)
    h = H.make_handle(w, x, dev)
    Wn, Mn, Ln = _two_calls_match_prefill(h, w, x, dev)
    h.close()
    # and the shared result against the oracle, at the parity bounds
    print(w.name, H.compare(w, x, (Wn, Mn, Ln, 0), H.run_oracle(w, x)))


def test_noalloc_with_attention_blocks(dev):
    from oracle import swa_oracle
    w = SWA_CASE
    x = I.make_inputs(w, seed=7, m0_scale=0.01, w0_per_sequence=True)
    sa = I.make_swa_inputs(w, seed=7, scale=1.0 / np.sqrt(w.d))
    h = H.make_handle(w, x, dev)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    h.set_attention(w.attn_heads, w.attn_window, t(sa["attn_w"]), t(sa["ln_gain"]), t(sa["ln_bias"]))
    from weight_long_context_b200 import ttt
    assert ttt.ttt_workspace_size(h._h, w.batch, w.T, w.b) <= 16 << 20
    Wn, Mn, Ln = _two_calls_match_prefill(h, w, x, dev)
    h.close()
    sw = swa_oracle.make_swa(w.d, w.n_blocks, w.attn_heads, w.attn_window, sa["attn_w"], sa["ln_gain"],
                             sa["ln_bias"])
    ref = swa_oracle.prefill(H.oracle_model(w, x), sw, x["W0"], x["M0"], x["hidden"], x["tokens"], x["eta"],
                             x["beta"], x["gamma"], w.b)
    print(w.name, H.compare(w, x, (Wn, Mn, Ln, 0), ref))


def test_noalloc_rejects_more_scratch_than_it_holds(dev):
    from weight_long_context_b200 import ttt
    w = I.WORKLOADS["batched_16"].with_(T=512, batch=2)
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    assert ttt.ttt_workspace_size(h._h, w.batch, w.T, w.b) > 16 << 20
    a = _inputs(w, x, dev)
    args = [a[k] for k in ("hidden", "tokens", "W", "M", "eta", "beta", "gamma", "loss")]
    code = ttt.load_library().ttt_prefill_noalloc(h._h, w.batch, w.T, w.b, *[_p(v) for v in args], None)
    assert code == 4
    assert "16777216" in ttt.ttt_last_error()
    h.close()
