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


# ------------------------------------------------------------------ bounded waits
@pytest.mark.parametrize("variant,M,N", [(0, 128, 256), (1, 256, 256), (2, 256, 512)])
def test_bounded_wait_runs_out_reports_timeout_and_recovers(variant, M, N):
    """The error path of the bounded waits, made to run out without any fault: one output tile
    (one CTA, or one CTA pair) with K = 131072, whose main loop runs for a fraction of a
    millisecond, and the epilogue's wait for the finished accumulator limited to 1 us. The wait
    expires; the epilogue records its code in the device error word and leaves, the producer
    and the MMA issuer finish their copies and MMAs (one tile: neither waits for an accumulator
    the epilogue would hand back), TMEM is freed and the kernel returns. poetx_device_status
    then reports POETX_ERR_TIMEOUT once and clears the word, and the next product on the same
    context is correct."""
    poetx.device_status()
    K = 131072
    g = torch.Generator(device="cpu").manual_seed(variant)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    b = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()   # K-major B
    c = torch.zeros(M, N, device="cuda", dtype=torch.bfloat16)
    poetx.testing_gemm_bf16(a, False, b, False, M, N, K, c, variant=variant, epi_wait_ns=1000)
    torch.cuda.synchronize()    # the kernel returned
    with pytest.raises(poetx.PoetxError) as e:
        poetx.device_status()
    assert e.value.status == 9 and "259" in str(e.value), str(e.value)   # 0x103: epilogue wait
    poetx.device_status()       # cleared
    # a normal product afterwards: same kernel, default wait limit
    Ks = 1024
    a2, b2, ref = _operands(M, N, Ks, False, False, seed=11 + variant)
    f32 = variant != 2   # the 256 x 512 kernel writes bf16 only
    c2 = torch.empty(M, N, device="cuda", dtype=torch.float32 if f32 else torch.bfloat16)
    poetx.testing_gemm_bf16(a2, False, b2, False, M, N, Ks, c2, variant=variant)
    torch.cuda.synchronize()
    poetx.device_status()
    err = (c2.float().cpu() - ref).abs().max().item() / ref.abs().max().item()
    assert err < (2e-6 * Ks ** 0.5 if f32 else 6e-3), err


# ------------------------------------------------------------------ 256 x 512 pair tiles
@pytest.mark.parametrize("variant", [2, 3])
@pytest.mark.parametrize("b_mn", [False, True])
@pytest.mark.parametrize("M,N,K", [(256, 512, 64), (300, 1024, 192), (1000, 512, 1024),
                                   (4096, 5120, 128), (4000, 5120, 2048)])
def test_umma_wide_gemm_matches_fp32_matmul_and_pair_kernel(variant, b_mn, M, N, K):
    """The dense kernel on 256 x 512 pair tiles (with and without the shared A collector)
    against an fp32 matmul, and bit for bit against the 256 x 256 pair kernel: both issue the
    same 256 x 256 x 16 MMAs in the same K order per output element. The 4096 / 4000-row cases
    give each cluster several tiles, so the accumulator halves are handed back and reused while
    the next tile starts; K = 128 is shorter than the stage ring; M = 300, 1000, 4000 are ragged."""
    a, b, ref = _operands(M, N, K, False, b_mn, seed=M + N + K + variant)
    c = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    poetx.testing_gemm_bf16(a, False, b, b_mn, M, N, K, c, variant=variant)
    c1 = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    poetx.testing_gemm_bf16(a, False, b, b_mn, M, N, K, c1, variant=1)
    torch.cuda.synchronize()
    poetx.device_status()
    err = (c.float().cpu() - ref).abs().max().item() / ref.abs().max().item()
    assert err < 6e-3, err
    assert torch.equal(c, c1)


def test_umma_wide_rejects_narrow_n():
    a = torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(768, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(256, 768, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(poetx.PoetxError) as e:
        poetx.testing_gemm_bf16(a, False, b, False, 256, 768, 64, c, variant=2)
    assert e.value.status == 7


@pytest.mark.parametrize("splits", [1, 3])
@pytest.mark.parametrize("M,N,K", [(512, 512, 4096), (256, 1024, 1000)])
def test_umma_wide_gemm_m_major_fp32_split_k(splits, M, N, K):
    """The per-block-gradient layout (A and B M/N-major, contraction over the rows, fp32 out,
    split K into partial products) on 256 x 512 pair tiles, against an fp32 matmul and bit for
    bit against the 256 x 256 pair kernel's partials."""
    a, b, ref = _operands(M, N, K, True, True, seed=splits * 13 + M)
    c = torch.full((splits, M, N), float("nan"), device="cuda")
    poetx.testing_gemm_bf16(a, True, b, True, M, N, K, c, splits=splits, variant=2)
    c1 = torch.full((splits, M, N), float("nan"), device="cuda")
    poetx.testing_gemm_bf16(a, True, b, True, M, N, K, c1, splits=splits, variant=1)
    torch.cuda.synchronize()
    poetx.device_status()
    total = c.sum(0).cpu()
    assert (total - ref).abs().max().item() / ref.abs().max().item() < 1e-5
    assert torch.equal(c, c1)
