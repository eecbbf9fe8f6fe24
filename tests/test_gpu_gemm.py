"""The tcgen05 GEMM engine alone (through ttt_gemm_bf16) against a plain
PyTorch fp32 matmul of the same bf16 operands: every operand layout, batching,
ragged tails in M, N and K, and sizes spanning many tiles."""
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


SHAPES = [(128, 256, 64, 1), (24, 200, 80, 3), (296, 520, 136, 2), (1024, 2304, 1024, 1), (136, 96, 24, 4),
          (64, 48, 16, 1)]


@pytest.mark.parametrize("a_k", [True, False])
@pytest.mark.parametrize("b_k", [True, False])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"{m}x{n}x{k}b{z}" for m, n, k, z in SHAPES])
def test_gemm_layouts(dev, shape, a_k, b_k):
    from weight_long_context_b200 import ttt
    M, N, K, Z = shape
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn(Z, M, K, generator=g).to(dev, torch.bfloat16)
    B = torch.randn(Z, N, K, generator=g).to(dev, torch.bfloat16)
    ref = torch.matmul(A.float(), B.float().transpose(1, 2))
    Ain = A if a_k else A.transpose(1, 2).contiguous()
    Bin = B if b_k else B.transpose(1, 2).contiguous()
    D = ttt.ttt_gemm_bf16(Ain, Bin, a_k, b_k)
    torch.cuda.synchronize()
    err = (D - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, err


def test_gemm_rejects_unaligned_strides(dev):
    from weight_long_context_b200 import ttt
    A = torch.zeros(1, 136, 300, device=dev, dtype=torch.bfloat16)   # MN-major, pitch 600 bytes
    B = torch.zeros(1, 64, 136, device=dev, dtype=torch.bfloat16)
    with pytest.raises(ttt.TTTError) as ei:
        ttt.ttt_gemm_bf16(A, B, False, True)
    assert ei.value.code == 3


SPLITK = [(1024, 2048, 5632, 1), (1024, 2048, 11264, 1), (512, 520, 4096, 2), (296, 264, 1000, 1),
          # whole waves of tiles plus a last wave finished as paired halves
          (1024, 11264, 2048, 1), (1024, 5632, 2048, 1), (1000, 5600, 1000, 1)]


@pytest.mark.parametrize("b_k", [True, False])
@pytest.mark.parametrize("shape", SPLITK, ids=[f"{m}x{n}x{k}b{z}" for m, n, k, z in SPLITK])
def test_gemm_split_k(dev, shape, b_k):
    """With a workspace the engine may split K across CTA pairs (every tile, or
    only the tiles of the last wave) and add the fp32 partials in a fixed
    order: accurate, and the same bits on every run."""
    from weight_long_context_b200 import ttt
    M, N, K, Z = shape
    g = torch.Generator(device="cpu").manual_seed(M + N + K)
    A = torch.randn(Z, M, K, generator=g).to(dev, torch.bfloat16)
    B = torch.randn(Z, N, K, generator=g).to(dev, torch.bfloat16)
    Bin = B if b_k else B.transpose(1, 2).contiguous()
    ws = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    D = ttt.ttt_gemm_bf16(A, Bin, True, b_k, workspace=ws)
    D2 = ttt.ttt_gemm_bf16(A, Bin, True, b_k, workspace=ws)
    torch.cuda.synchronize()
    ref = torch.matmul(A.float(), B.float().transpose(1, 2))
    err = (D - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, err
    assert torch.equal(D, D2)
