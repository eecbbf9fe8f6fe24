"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same
seeded inputs.  Tolerances: relative Frobenius error on final W and M <= 1e-4
(fp32 mode) or 3e-2 (bf16 mode); per-chunk mean loss within 1e-2 absolute."""
import json
import os

import numpy as np
import pytest

from tests import helpers as H
from weight_long_context_b200 import inputs as I

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def W(name, **kw):
    return I.WORKLOADS[name].with_(**kw)


# ---------------------------------------------------------------------------
# K1 scalar scan alone
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("b,kind", [(1, "e2ttt"), (16, "sgd"), (64, "e2ttt"), (100, "mixed"),
                                    (1024, "e2ttt"), (1024, "sgd"), (4096, "e2ttt")])
def test_scalar_scan_matches_oracle(dev, b, kind):
    import oracle
    from weight_long_context_b200 import ttt
    rng = np.random.default_rng(b)
    B, nc = 3, 4
    T = b * nc
    eta = (0.01 / (1 + np.exp(-rng.normal(size=(B, T))))).astype(np.float32)
    if kind == "sgd":
        beta = np.zeros((B, T), np.float32)
        gamma = np.ones((B, T), np.float32)
    else:
        beta = rng.uniform(0.8, 0.99, (B, T)).astype(np.float32)
        gamma = rng.uniform(0.99, 1.0, (B, T)).astype(np.float32)
        if kind == "mixed":
            beta[:, ::7] = 0.0
            gamma[:, ::11] = 1.0
    t = lambda a: torch.from_numpy(a).to(dev)
    KW, KM, consts = ttt.ttt_scalar_kernels(t(eta), t(beta), t(gamma), b)
    KW, KM, consts = KW.cpu().numpy(), KM.cpu().numpy(), consts.cpu().numpy()
    for s in range(B):
        for c in range(nc):
            sl = slice(c * b, (c + 1) * b)
            kw, km, g0, b0, cM = oracle.scalar_kernels(eta[s, sl], beta[s, sl], gamma[s, sl])
            np.testing.assert_allclose(KW[s, sl], kw, rtol=2e-6, atol=1e-30)
            np.testing.assert_allclose(KM[s, sl], km, rtol=2e-6, atol=1e-30)
            np.testing.assert_allclose(consts[s, c, :3], [g0, b0, cM], rtol=2e-6, atol=1e-30)


# ---------------------------------------------------------------------------
# Small ragged shapes: several tiles and a ragged tail in every dimension
# ---------------------------------------------------------------------------

RAGGED = [
    # name, d, h, V, L, mlp, static, T, b, batch
    ("gelu_1blk", 80, 208, 528, 1, "gelu", False, 72, 24, 2),
    ("swiglu_2blk_static", 48, 80, 272, 2, "swiglu", True, 60, 20, 2),
    ("gelu_3blk_static", 64, 96, 400, 3, "gelu", True, 48, 16, 1),
    ("swiglu_tile_tail", 208, 336, 1040, 1, "swiglu", False, 272, 136, 2),
]


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("case", RAGGED, ids=[c[0] for c in RAGGED])
def test_ragged_parity(dev, case, precision):
    name, d, h, V, L, mlp, st, T, b, B = case
    w = I.Workload(name, d, h, V, L, mlp, st, precision, T, b, B, "e2ttt")
    x = I.make_inputs(w, seed=5, m0_scale=0.01, w0_per_sequence=True)
    gpu = H.run_gpu(w, x, dev)
    ref = H.run_oracle(w, x)
    e = H.compare(w, x, gpu, ref)
    print(name, precision, e)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("case", RAGGED[:2] + RAGGED[3:], ids=[c[0] for c in RAGGED[:2] + RAGGED[3:]])
def test_sum_reduction_parity(dev, case, precision):
    """The chunk objective as the plain sum of the token losses (the literal
    per-token loss of the E2-TTT recursion, loss_reduction = SUM): every
    gradient is b times the mean reduction's."""
    name, d, h, V, L, mlp, st, T, b, B = case
    w = I.Workload(name, d, h, V, L, mlp, st, precision, T, b, B, "e2ttt", reduction="sum")
    x = I.make_inputs(w, seed=6, m0_scale=0.01, w0_per_sequence=True)
    e = H.compare(w, x, H.run_gpu(w, x, dev), H.run_oracle(w, x))
    print(name, precision, "sum", e)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_online_sgd_b1(dev, precision):
    """b = 1, beta = 0, gamma = 1: online SGD, one token per chunk."""
    w = I.Workload("b1", 32, 48, 64, 2, "gelu", True, precision, 12, 1, 2, "sgd", 0.05, "uniform")
    x = I.make_inputs(w, seed=3)
    H.compare(w, x, H.run_gpu(w, x, dev), H.run_oracle(w, x))


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def test_tiny_sgd_full(dev):
    w = W("tiny_sgd")
    x = I.make_inputs(w, seed=0)
    e = H.compare(w, x, H.run_gpu(w, x, dev), H.run_oracle(w, x))
    print("tiny_sgd", e)


def test_e2ttt_block_full(dev):
    w = W("e2ttt_block")
    x = I.make_inputs(w, seed=0)
    e = H.compare(w, x, H.run_gpu(w, x, dev), H.run_oracle(w, x, dtype=np.float32))
    print("e2ttt_block", e)


@pytest.mark.parametrize("name", ["sgd_3b", "batched_16"])
def test_full_dims_first_chunks(dev, name):
    """Full model sizes and chunk size (the launch configuration the benchmark
    times), first two chunks, element by element against the oracle."""
    w = W(name)
    w = w.with_(T=2 * w.b, batch=min(w.batch, 4))
    x = I.make_inputs(w, seed=0, m0_scale=1e-3 if w.scalars == "e2ttt" else 0.0)
    e = H.compare(w, x, H.run_gpu(w, x, dev), H.run_oracle(w, x, dtype=np.float32))
    print(name, e)


def _stack_case(scale, precision):
    w = W("stack_128k", precision=precision).with_(T=2 * 1024)
    x = I.make_inputs(w, seed=0, m0_scale=1e-3)
    if scale != 1.0:
        x["W0"] = x["W0"] * np.float32(scale)
        x["static_w"] = x["static_w"] * np.float32(scale)
    return w, x


def test_stack_128k_first_chunks_against_fp64(dev):
    """The 128K stack at full dimensions and chunk size (the benchmark's launch
    shapes), first two chunks, against the oracle in float64, at the
    workload's draw and with W0 and the static MLPs at a quarter of it.

    The float32 oracle run beside it measures the conditioning: at the
    workload's draw the residual stream grows through the eight SwiGLU MLPs
    (no norm inside the blocks), and the float32 oracle itself is 0.45 % off
    on W and 2.4 % off on the gradient-driven part of W.  There the GPU's fp32
    mode must land where the float32 oracle lands (within twice its distance
    to float64), and the bf16 mode's W and M within the bf16 bound or ten
    times the float32 oracle's distance, whichever is larger (bf16 rounding
    is amplified by the same draw; measured 2.6 % on W and 3.0 % on M), with
    the chunk losses within 1e-2.  At the quarter draw float32 agrees with
    float64 to about 1e-5 and every quantity, the gradient-driven parts
    included, is held to the bound of its mode."""
    rows = {}
    for scale in (1.0, 0.25):
        w, x = _stack_case(scale, "bf16")
        ref = H.run_oracle(w, x, dtype=np.float64)
        gpu = {p: H.run_gpu(w.with_(precision=p), x, dev) for p in ("bf16", "fp32")}
        o32 = H.run_oracle(w, x, dtype=np.float32)
        Wn, Mn = (a.reshape(-1) for a in H.no_grad_state(w, x))

        def errs(Wa, Ma, La):
            return dict(W=H.rel_fro(Wa, ref[0]), M=H.rel_fro(Ma, ref[1]), dW=H.rel_fro(Wa - Wn, ref[0] - Wn),
                        dM=H.rel_fro(Ma - Mn, ref[1] - Mn), loss=float(np.max(np.abs(La - ref[2]))))
        for p, g in gpu.items():
            assert g[3] == 0
            rows[(scale, "gpu_" + p)] = errs(*g[:3])
        rows[(scale, "oracle_fp32")] = errs(*o32)
    for k, e in rows.items():
        print("stack_128k 2 chunks vs fp64", k, {a: f"{v:.2e}" for a, v in e.items()})
    f16, f32, o32 = rows[(1.0, "gpu_bf16")], rows[(1.0, "gpu_fp32")], rows[(1.0, "oracle_fp32")]
    for k in ("W", "M"):
        assert f16[k] <= max(H.TOL_STATE["bf16"], 10 * o32[k]), (k, f16, o32)
    for k in ("W", "M", "dW", "dM"):
        assert f32[k] <= 2 * o32[k] + H.TOL_STATE["fp32"], (k, f32, o32)
    assert f16["loss"] <= H.TOL_LOSS and f32["loss"] <= H.TOL_LOSS
    q16, q32 = rows[(0.25, "gpu_bf16")], rows[(0.25, "gpu_fp32")]
    assert q16["loss"] <= H.TOL_LOSS
    assert max(q16[k] for k in ("W", "M", "dW", "dM")) <= H.TOL_STATE["bf16"], q16
    assert max(q32[k] for k in ("W", "M", "dW", "dM")) <= H.TOL_STATE["fp32"] and q32["loss"] <= H.TOL_LOSS, q32


def _golden(stem):
    path = os.path.join(GOLDEN, f"{stem}_seed0.json")
    assert os.path.exists(path), f"{path} missing: run tests/golden/make_golden.py"
    return json.load(open(path))


def _check_sampled(w, gpu, g):
    """Sampled final state (W, M and their gradient-driven parts) and every
    chunk loss against a stored oracle run."""
    Wg, Mg, Lg, st = gpu
    assert st == 0
    idx = np.asarray(g["sample_index"])
    tol = H.TOL_STATE[w.precision]
    Wr, Mr = np.asarray(g["W"]), np.asarray(g["M"])
    Wn, Mn = np.asarray(g["W_nograd"]), np.asarray(g["M_nograd"])
    e = dict(W=H.rel_fro(Wg[idx], Wr), M=H.rel_fro(Mg[idx], Mr), dW=H.rel_fro(Wg[idx] - Wn, Wr - Wn),
             dM=H.rel_fro(Mg[idx] - Mn, Mr - Mn), loss=float(np.max(np.abs(Lg - np.asarray(g["chunk_loss"])))),
             grad_share_W=float(np.linalg.norm(Wr - Wn) / np.linalg.norm(Wr)))
    C = w.T // w.b
    e["dW_bound"] = H.grad_part_bound(tol, Wr, Wn, C)
    e["dM_bound"] = H.grad_part_bound(tol, Mr, Mn, C)
    assert e["W"] <= tol and e["M"] <= tol and e["dW"] <= e["dW_bound"] and e["dM"] <= e["dM_bound"], e
    assert e["loss"] <= H.TOL_LOSS, e
    return e


def test_full_length_sampled_sgd_3b(dev):
    """Full-length run of the 3B-class SGD layer at the benchmark's sizes vs
    stored oracle samples (tests/golden/sgd_3b_seed0.json, written by
    tests/golden/make_golden.py): W, M, the part of W the updates added, and
    all 32 chunk losses."""
    w = W("sgd_3b")
    x = I.make_inputs(w, seed=0)
    print("sgd_3b", _check_sampled(w, H.run_gpu(w, x, dev), _golden("sgd_3b")))


@pytest.mark.parametrize("name,stem", [("stack_128k", "stack_128k_live_q"), ("batched_16", "batched_16_live")])
def test_full_length_live_state(dev, name, stem):
    """Added case: the 128K stack and the batched workload at full length with
    the E2-TTT draw of eta and beta but gamma = 1, so the fast weights stay
    live to the end (under the workloads' own draw they decay to zero, see
    the next test).  Sampled W, M, their gradient-driven parts and every chunk
    loss against tests/golden/<stem>_seed0.json.  The stack's W0 and static
    MLPs are drawn at a quarter of the workload's scale, where float32 and
    float64 agree (see test_stack_128k_first_chunks_against_fp64)."""
    g = _golden(stem)
    w = W(name).with_(scalars="e2ttt_live")
    x = I.make_inputs(w, seed=0)
    s = g.get("mlp_weight_scale", 1.0)
    if s != 1.0:
        x["W0"] = x["W0"] * np.float32(s)
        if x["static_w"] is not None:
            x["static_w"] = x["static_w"] * np.float32(s)
    print(name, "live", _check_sampled(w, H.run_gpu(w, x, dev), g))


@pytest.mark.parametrize("name", ["stack_128k", "batched_16"])
def test_full_length_decayed_state(dev, name):
    """The workloads' own draw at full length.  gamma ~ U(0.99, 1) multiplies
    the state by about 0.006 per chunk of 1024 tokens (0.28 per 256), and with
    zero weights every gradient of the MLP vanishes, so the oracle's final W and
    M are zero (or below 1e-15): there is no relative error to take.  What is
    checked: every chunk loss (they depend on the state while it lives) and
    that the GPU state decayed as well."""
    g = _golden(name)
    w = W(name)
    x = I.make_inputs(w, seed=0)
    Wg, Mg, Lg, st = H.run_gpu(w, x, dev)
    assert st == 0
    assert g["W_norm"] < 1e-12 * np.linalg.norm(x["W0"])
    assert np.linalg.norm(Wg) < 1e-6 * np.linalg.norm(x["W0"]) and np.linalg.norm(Mg) < 1e-6 * np.linalg.norm(x["W0"])
    eL = float(np.max(np.abs(Lg - np.asarray(g["chunk_loss"]))))
    assert eL <= H.TOL_LOSS, eL
    print(name, "loss", eL, "W norm", float(np.linalg.norm(Wg)))


# ---------------------------------------------------------------------------
# Properties that hold at any size
# ---------------------------------------------------------------------------

def test_resume_and_determinism_bitwise(dev):
    """Chunk-end state is the only carried state: prefill(T) equals
    prefill(T1) then prefill(T - T1) bit for bit, and reruns are identical."""
    w = W("e2ttt_block", T=1024)
    x = I.make_inputs(w, seed=2, m0_scale=1e-3)
    Wa, Ma, La, _ = H.run_gpu(w, x, dev)
    Wb, Mb, Lb, _ = H.run_gpu(w, x, dev)
    assert np.array_equal(Wa, Wb) and np.array_equal(Ma, Mb) and np.array_equal(La, Lb)
    T1 = 512
    x1 = dict(x, hidden=x["hidden"][:, :T1], tokens=x["tokens"][:, :T1], eta=x["eta"][:, :T1],
              beta=x["beta"][:, :T1], gamma=x["gamma"][:, :T1])
    W1, M1, L1, _ = H.run_gpu(w.with_(T=T1), x1, dev)
    x2 = dict(x, hidden=x["hidden"][:, T1:], tokens=x["tokens"][:, T1:], eta=x["eta"][:, T1:],
              beta=x["beta"][:, T1:], gamma=x["gamma"][:, T1:], W0=W1, M0=M1)
    W2, M2, L2, _ = H.run_gpu(w.with_(T=T1), x2, dev)
    assert np.array_equal(W2, Wa) and np.array_equal(M2, Ma)
    assert np.array_equal(np.concatenate([L1, L2], axis=1), La)


@pytest.mark.parametrize("seg", [0, 1, 3])
def test_host_prefill_matches_device_prefill_bitwise(dev, seg):
    """ttt_prefill_host streams the sequence in segments of seg chunks with
    the copies overlapping the compute; chunk-end state is the only carried
    state, so it must give ttt_prefill's results bit for bit (two sequences:
    strided segment copies; seg = 3 of 4 chunks leaves a ragged last segment)."""
    w = W("batched_16", T=1024, batch=2)
    x = I.make_inputs(w, seed=2, m0_scale=1e-3, w0_per_sequence=True)
    Wa, Ma, La, st, h = H.run_gpu(w, x, dev, return_handle=True)
    pin = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a if dt is None else a.astype(dt))).pin_memory()
    Wh, Mh, Lh = h.prefill_host(pin(x["hidden"]), pin(x["tokens"], np.int32), pin(x["W0"]), pin(x["M0"]),
                                pin(x["eta"]), pin(x["beta"]), pin(x["gamma"]), w.b, seg_chunks=seg)
    assert h.device_status() == 0
    assert np.array_equal(Wh.numpy(), Wa) and np.array_equal(Mh.numpy(), Ma) and np.array_equal(Lh.numpy(), La)
    h.close()


def test_zero_head_gives_log_v(dev):
    w = I.Workload("zh", 64, 96, 160, 1, "swiglu", False, "bf16", 64, 32, 1, "e2ttt")
    x = I.make_inputs(w, seed=1, m0_scale=0.01)
    x["lm_head"] = np.zeros_like(x["lm_head"])
    Wg, Mg, Lg, st = H.run_gpu(w, x, dev)
    np.testing.assert_allclose(Lg, np.log(160.0), rtol=1e-6)
    Wr, Mr, _ = H.run_oracle(w, x)
    assert H.rel_fro(Wg, Wr) < 1e-6 and H.rel_fro(Mg, Mr) < 1e-6


# ---------------------------------------------------------------------------
# Edge cases and errors
# ---------------------------------------------------------------------------

def test_empty_calls_are_noops(dev):
    from weight_long_context_b200 import ttt
    w = I.Workload("e", 32, 32, 32, 1, "gelu", False, "fp32", 16, 8, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    W0 = t(x["W0"])
    Wc = W0.clone()
    empty = torch.empty((1, 0, 32), device=dev)
    e2 = torch.empty((1, 0), device=dev)
    h.prefill(empty, e2.to(torch.int32), Wc, t(x["M0"]), e2, e2, e2, 8)
    torch.cuda.synchronize()
    assert torch.equal(Wc, W0)
    assert h.device_status() == 0
    h.close()


def test_shape_and_argument_errors(dev):
    from weight_long_context_b200 import ttt
    w = I.Workload("e", 32, 32, 32, 1, "gelu", False, "fp32", 16, 8, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    args = [t(x["hidden"]), t(x["tokens"], torch.int32), t(x["W0"]), t(x["M0"]), t(x["eta"]),
            t(x["beta"]), t(x["gamma"])]
    with pytest.raises(ttt.TTTError) as ei:
        h.prefill(*args, b=5)           # T % b != 0
    assert ei.value.code == 2
    with pytest.raises(ttt.TTTError) as ei:
        h.prefill(*args, b=0)
    assert ei.value.code == 2
    assert ttt.ttt_workspace_size(h._h, 1, 16, 8) > 0
    # unsupported model shape
    cfg = ttt.ttt_config(30, 32, 32, 1, 0, 0, 0, 0, 1e-6)
    with pytest.raises(ttt.TTTError) as ei:
        ttt.ttt_create(cfg, args[0], args[0], None)
    assert ei.value.code == 3
    h.close()


def test_workspace_too_small(dev):
    import ctypes
    from weight_long_context_b200 import ttt
    w = I.Workload("e", 32, 32, 32, 1, "gelu", False, "fp32", 16, 8, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    loss = torch.empty((1, 2), device=dev)
    p = lambda a: ctypes.c_void_p(a.data_ptr())
    args = [t(x["hidden"]), t(x["tokens"], torch.int32), t(x["W0"]), t(x["M0"]), t(x["eta"]),
            t(x["beta"]), t(x["gamma"])]
    code = ttt.load_library().ttt_prefill(h._h, 1, 16, 8, *[p(a) for a in args], p(loss), p(ws), 256,
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 4
    h.close()


def test_bad_token_sets_device_status(dev):
    w = I.Workload("tok", 32, 32, 64, 1, "gelu", False, "bf16", 32, 16, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    x["tokens"][0, 5] = 64            # == V: outside [0, V)
    *_, st = H.run_gpu(w, x, dev)
    assert st == 5


def test_nonfinite_hidden_sets_device_status(dev):
    w = I.Workload("nan", 32, 32, 64, 1, "gelu", False, "fp32", 32, 16, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    x["hidden"][0, 3, :] = np.nan
    *_, st = H.run_gpu(w, x, dev)
    assert st == 6


def test_bounded_wait_times_out_cleanly(dev):
    """A wait on a flag nothing sets gives up after its limit and reports
    TTT_ERR_TIMEOUT; the context stays usable afterwards."""
    w = I.Workload("e", 32, 32, 32, 1, "gelu", False, "fp32", 16, 8, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    h.selftest_bounded_wait(1000)
    assert h.device_status() == 7
    assert h.device_status() == 0
    # still usable
    Wg, Mg, Lg, st = H.run_gpu(w, x, dev, handle=h)
    assert st == 0 and np.all(np.isfinite(Wg))
    h.close()


PROF_CASES = [
    I.Workload("prof", 128, 256, 544, 2, "swiglu", True, "bf16", 256, 64, 2, "e2ttt"),
    # eight MLP levels: the backward reuses each of the three rotating dU and
    # output-gradient buffers while the aggregation stream may still read it
    I.Workload("prof_deep", 128, 256, 544, 4, "swiglu", True, "bf16", 256, 64, 2, "e2ttt"),
    I.Workload("prof_deep_gelu", 96, 224, 416, 5, "gelu", False, "bf16", 192, 64, 1, "e2ttt"),
]


@pytest.mark.parametrize("w", PROF_CASES, ids=[c.name for c in PROF_CASES])
def test_profiled_path_matches_graph_path(dev, w):
    """ttt_prefill_profiled runs the same kernels eagerly and serially, with
    events: results are bit-identical to the graph path, whose aggregations
    run on a second stream beside the backward, and every launch is
    accounted for."""
    x = I.make_inputs(w, seed=4, m0_scale=1e-3)
    Wa, Ma, La, st, h = H.run_gpu(w, x, dev, return_handle=True)
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    W, M = t(x["W0"]), t(x["M0"])
    loss, stats = h.prefill_profiled(t(x["hidden"]), t(x["tokens"], torch.int32), W, M, t(x["eta"]),
                                     t(x["beta"]), t(x["gamma"]), w.b)
    assert np.array_equal(W.cpu().numpy(), Wa) and np.array_equal(M.cpu().numpy(), Ma)
    assert np.array_equal(loss.cpu().numpy(), La)
    names = {s["name"] for s in stats}
    assert {"agg_update", "mlp_up", "mlp_down", "ce_logits_lse", "ce_dz", "mlp_bwd_dA"} <= names
    assert all(s["ms"] > 0 and s["launches"] > 0 for s in stats)
    upd = next(s for s in stats if s["name"] == "agg_update")
    # two aggregation GEMMs per dynamic MLP per chunk, 2 x 2 x rows x cols x b x batch FLOPs
    assert upd["launches"] == 2 * w.n_blocks * w.n_chunks
    m = 3 if w.mlp == "swiglu" else 2
    assert upd["flops"] == pytest.approx(4.0 * m * w.hidden * w.d * w.b * w.batch * w.n_blocks * w.n_chunks)
    h.close()


def test_misaligned_state_rejected(dev):
    """W and M must be 16-byte aligned: a 4-byte offset is rejected before any launch."""
    import ctypes
    from weight_long_context_b200 import ttt
    w = I.Workload("e", 32, 32, 32, 1, "gelu", False, "bf16", 16, 8, 1, "e2ttt")
    x = I.make_inputs(w, seed=0)
    h = H.make_handle(w, x, dev)
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    n = ttt.ttt_workspace_size(h._h, 1, 16, 8)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=dev)
    loss = torch.empty((1, 2), device=dev)
    Wbig = torch.zeros(x["W0"].size + 4, device=dev)
    p = lambda a: ctypes.c_void_p(a.data_ptr())
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    hid, tok, M0 = t(x["hidden"]), t(x["tokens"], torch.int32), t(x["M0"])
    sc = [t(x["eta"]), t(x["beta"]), t(x["gamma"])]
    for Wp, Mp in ((Wbig[1:], M0), (t(x["W0"]), Wbig[1:])):
        code = ttt.load_library().ttt_prefill(h._h, 1, 16, 8, p(hid), p(tok), p(Wp), p(Mp), *[p(a) for a in sc],
                                              p(loss), p(ws), n, st)
        assert code == 1
    assert h.device_status() == 0
    h.close()
