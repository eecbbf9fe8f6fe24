"""Host-side logic of bench.py on CPU: the algorithmic FLOP count per token,
the JSON of the reference arm's helpers, and the multi-rank timing reduction
with world-size-2 gloo process groups (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from weight_long_context_b200 import inputs as I


@pytest.mark.parametrize("name,expect", [("tiny_sgd", 0.295e6), ("e2ttt_block", 31.5e6), ("sgd_3b", 745.5e6),
                                         ("stack_128k", 1807.8e6), ("batched_16", 125.8e6)])
def test_flops_per_token(name, expect):
    assert bench.flops_per_token(I.WORKLOADS[name]) == pytest.approx(expect, rel=2e-3)


def test_stack_breakdown():
    w = I.WORKLOADS["stack_128k"]
    d, h = w.d, w.hidden
    # MLP fwd 553.6M, head 262.1M, bwd 438.3M, aggregation 553.6M per token
    assert 8 * 6 * d * h == pytest.approx(553.6e6, rel=1e-3)
    assert 4 * d * w.vocab == pytest.approx(262.1e6, rel=1e-3)


def test_workload_config_keys():
    c = bench.workload_config(I.WORKLOADS["stack_128k"])
    assert c["workload"] == "stack_128k" and "model" not in c
    assert c["l2"].startswith("inputs larger than L2")
    assert bench.workload_config(I.WORKLOADS["tiny_sgd"])["l2"].startswith("L2 flushed")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    bench.init_dist("gloo", timeout_s=60)
    import torch.distributed as dist
    ms = 10.0 + 5.0 * rank                 # rank 1 is the slowest
    mx = bench.reduce_max(ms)
    rate = bench.whole_job_rate(1000.0, world, mx / 1e3)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, rate))


def test_multirank_max_and_whole_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the max over ranks; whole-job rate = units of all ranks / that time
    assert all(mx == 15.0 for _, mx, _ in res)
    assert all(rate == pytest.approx(2 * 1000.0 / 0.015) for _, _, rate in res)


def test_predict_flops_per_token():
    """Forward only: 8 MLPs (4 static + 4 dynamic) of 2 m d h and the logits 2 d V."""
    w = I.WORKLOADS["stack_128k"]
    assert bench.predict_flops_per_token(w) == 8 * 2 * 3 * w.d * w.hidden + 2 * w.d * w.vocab
    assert bench.predict_flops_per_token(w) == pytest.approx(684.72e6, rel=1e-4)


def test_attention_flops_per_token():
    """No attention adds nothing; with window >= T every query sees t + 1 keys
    (mean (T + 1) / 2), and the lower blocks' MLP backward runs a second time."""
    w = I.WORKLOADS["stack_128k"]
    assert bench.attention_flops_per_token(w) == 0.0
    small = w.with_(T=64, b=16, attn_heads=2, attn_window=1 << 20, n_blocks=2, has_static=False)
    d, h, m = small.d, small.hidden, small.n_mats
    kbar, bbar = (64 + 1) / 2, (16 + 1) / 2
    expect = (2 * (8 * d * d + 4 * d * kbar) + 1 * 2 * (8 * d * d + 4 * d * kbar + 4 * d * bbar)
              + 2 * d * h)                 # block 0's dynamic MLP: B1 only (nothing dynamic below it)
    assert bench.attention_flops_per_token(small) == pytest.approx(expect, rel=1e-12)
    # a window of one key: each query sees only itself
    one = small.with_(attn_window=1)
    expect1 = 2 * (8 * d * d + 4 * d) + 2 * (8 * d * d + 4 * d + 4 * d) + 2 * d * h
    assert bench.attention_flops_per_token(one) == pytest.approx(expect1, rel=1e-12)
    assert bench.flops_per_token(I.WORKLOADS["stack_128k_swa"]) == pytest.approx(
        bench.flops_per_token(w) + bench.attention_flops_per_token(I.WORKLOADS["stack_128k_swa"]))
