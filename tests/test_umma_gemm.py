"""Kernel-level numerics of the bf16 tensor-core contraction (tcgen05 / TMEM / TMA) against a
plain PyTorch fp32 matmul of the same bf16 operands, for every operand layout the layer uses,
ragged M and K, and split-K partial sums."""
import pytest
import torch

from tests.gpu_util import poetx

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _operands(M, N, K, a_mn, b_mn, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    a_store = A.t().contiguous() if a_mn else A          # MN-major: [K][M]
    b_store = B.contiguous() if b_mn else B.t().contiguous()  # MN-major: [K][N]; K-major: [N][K]
    ref = A.float() @ B.float()
    return a_store.cuda(), b_store.cuda(), ref


LAYOUTS = [(False, False, False), (False, True, False), (True, True, True), (False, False, True),
           (False, True, True)]


@pytest.mark.parametrize("a_mn,b_mn,f32", LAYOUTS)
@pytest.mark.parametrize("M,N,K", [(128, 64, 64), (200, 128, 192), (384, 256, 320),
                                   (1000, 512, 256), (136, 768, 1024)])
def test_umma_gemm_matches_fp32_matmul(a_mn, b_mn, f32, M, N, K):
    a, b, ref = _operands(M, N, K, a_mn, b_mn, seed=M * 7 + N + K)
    c = torch.empty(M, N, device="cuda", dtype=torch.float32 if f32 else torch.bfloat16)
    poetx.testing_gemm_bf16(a, a_mn, b, b_mn, M, N, K, c)
    torch.cuda.synchronize()
    poetx.device_status()
    err = (c.float().cpu() - ref).abs().max().item() / ref.abs().max().item()
    assert err < (2e-6 * K ** 0.5 if f32 else 6e-3), err


@pytest.mark.parametrize("splits", [2, 3, 4, 8])
def test_umma_gemm_split_k_partials(splits):
    M, N, K = 256, 256, 1000   # ragged K: the last split reads zero-filled rows
    a, b, ref = _operands(M, N, K, True, True, seed=splits)
    c = torch.full((splits, M, N), float("nan"), device="cuda")
    poetx.testing_gemm_bf16(a, True, b, True, M, N, K, c, splits=splits)
    torch.cuda.synchronize()
    total = c.sum(0).cpu()
    assert (total - ref).abs().max().item() / ref.abs().max().item() < 1e-5


def test_umma_gemm_identity_is_exact():
    """A I == A exactly: every product is by 1.0 or 0.0 and fp32 sums of them are exact."""
    M, K = 300, 256
    A = torch.randn(M, K).to(torch.bfloat16).cuda()
    eye = torch.eye(K, dtype=torch.bfloat16, device="cuda")
    for b_mn in (False, True):
        c = torch.empty(M, K, device="cuda", dtype=torch.bfloat16)
        poetx.testing_gemm_bf16(A, False, eye, b_mn, M, K, K, c)
        torch.cuda.synchronize()
        assert torch.equal(c, A)


def test_umma_gemm_rejects_uncovered_shapes():
    a = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(48, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(128, 48, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(poetx.PoetxError) as e:
        poetx.testing_gemm_bf16(a, False, b, False, 128, 48, 64, c)
    assert e.value.status == 7


# ------------------------------------------------------------------ CTA-pair kernel
@pytest.mark.parametrize("a_mn,b_mn,f32", LAYOUTS)
@pytest.mark.parametrize("M,N,K", [(256, 256, 64), (304, 512, 192), (1000, 256, 1024),
                                   (512, 768, 320)])
def test_umma_pair_gemm_matches_fp32_matmul(a_mn, b_mn, f32, M, N, K):
    a, b, ref = _operands(M, N, K, a_mn, b_mn, seed=M * 3 + N + K)
    c = torch.empty(M, N, device="cuda", dtype=torch.float32 if f32 else torch.bfloat16)
    poetx.testing_gemm_bf16(a, a_mn, b, b_mn, M, N, K, c, variant=1)
    torch.cuda.synchronize()
    poetx.device_status()
    err = (c.float().cpu() - ref).abs().max().item() / ref.abs().max().item()
    assert err < (2e-6 * K ** 0.5 if f32 else 6e-3), err


def test_umma_pair_gemm_split_k_and_identity():
    M, N, K = 512, 256, 1000
    a, b, ref = _operands(M, N, K, True, True, seed=7)
    c = torch.full((4, M, N), float("nan"), device="cuda")
    poetx.testing_gemm_bf16(a, True, b, True, M, N, K, c, splits=4, variant=1)
    torch.cuda.synchronize()
    total = c.sum(0).cpu()
    assert (total - ref).abs().max().item() / ref.abs().max().item() < 1e-5
    A = torch.randn(384, 256).to(torch.bfloat16).cuda()
    eye = torch.eye(256, dtype=torch.bfloat16, device="cuda")
    for b_mn in (False, True):
        out = torch.empty(384, 256, device="cuda", dtype=torch.bfloat16)
        poetx.testing_gemm_bf16(A, False, eye, b_mn, 384, 256, 256, out, variant=1)
        torch.cuda.synchronize()
        assert torch.equal(out, A)
