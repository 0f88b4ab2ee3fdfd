"""The measurement kernels behind the roofline denominators: the 128-bit copy
and the tcgen05 FP8 GEMM give correct results (a GEMM that skipped work would
report a false peak)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def test_copy_kernel(csa):
    g = torch.Generator(device="cuda").manual_seed(1)
    for n in (16, 4096 * 16 + 48, (64 << 20) + 16 * 7):
        src = torch.randint(0, 256, (n,), dtype=torch.uint8, device="cuda", generator=g)
        dst = torch.zeros(n, dtype=torch.uint8, device="cuda")
        csa.csa_bench_copy(src, dst)
        torch.cuda.synchronize()
        assert torch.equal(src, dst)


def _e4m3_values(codes):
    return codes.view(torch.float8_e4m3fn).to(torch.float64)


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (256, 512, 384), (2560, 2560, 256)])
def test_fp8_gemm_kernel(csa, M, N, K):
    # (2560, 2560, 256): 20 x 10 = 200 output tiles over 148 CTAs, so some
    # CTAs take a second tile in the other TMEM accumulator
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    A = torch.randint(0, 256, (M, K), dtype=torch.uint8, device="cuda", generator=g)
    B = torch.randint(0, 256, (N, K), dtype=torch.uint8, device="cuda", generator=g)
    A[(A & 0x7F) == 0x7F] = 0          # no NaN codes
    B[(B & 0x7F) == 0x7F] = 0
    D = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    csa.csa_bench_fp8_gemm(A, B, D)
    torch.cuda.synchronize()
    a, b = _e4m3_values(A), _e4m3_values(B)
    ref = a @ b.t()
    bound = 1e-5 * (a.abs() @ b.abs().t()) + 1e-30
    err = (D.to(torch.float64) - ref).abs()
    assert bool(torch.isfinite(D).all())
    assert bool((err <= bound).all()), float((err / bound).max())


def test_fp8_gemm_rejects_shapes(csa):
    A = torch.zeros((100, 128), dtype=torch.uint8, device="cuda")
    B = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    D = torch.zeros((100, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(csa.CsaError):
        csa.csa_bench_fp8_gemm(A, B, D)
