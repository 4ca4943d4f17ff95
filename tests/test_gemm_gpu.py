"""tcgen05 bf16 GEMM against torch's fp32 product of the same bf16 operands."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tpc():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tree_packed_chunkwise_b200 as t
    t.lib()
    return t


def padded(x):
    """Same values with the leading dimension rounded up to a multiple of 8 (TMA stride rule)."""
    import torch
    r, c = x.shape
    buf = torch.zeros(r, (c + 7) // 8 * 8, dtype=x.dtype, device=x.device)
    buf[:, :c] = x
    return buf[:, :c]


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 500, 200), (1, 8, 8), (700, 1030, 2048),
                                   (300, 520, 4100), (520, 300, 4620)])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_gemm_matches_torch(tpc, M, N, K, a_mn, b_mn):
    import torch
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N + K)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    a = padded(A.t()) if a_mn else padded(A)
    b = padded(B.t()) if b_mn else padded(B)
    ref = A.float() @ B.float().t()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    C = tpc.tpc_gemm_bf16(a, b, a_mn=bool(a_mn), b_mn=bool(b_mn), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    err = (C - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, err
    # bf16 output and fp32 accumulation into an existing C
    Cb = tpc.tpc_gemm_bf16(a, b, a_mn=bool(a_mn), b_mn=bool(b_mn), out_dtype=torch.bfloat16)
    assert ((Cb.float() - ref).abs() <= 1e-2 * ref.abs() + 1e-2).all()
    C2 = torch.ones(M, N, device="cuda")
    tpc.tpc_gemm_bf16(a, b, c=C2, a_mn=bool(a_mn), b_mn=bool(b_mn), alpha=2.0, beta=0.5)
    assert (C2 - (2 * ref + 0.5)).abs().max().item() <= 1e-5 * (2 * ref.abs().max().item() + 1)


def test_gemm_rejects_bad_arguments(tpc):
    import torch
    a = torch.zeros(16, 12, dtype=torch.bfloat16, device="cuda")  # lda = 12, not a multiple of 8
    b = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tpc.TpcError) as e:
        tpc.tpc_gemm_bf16(a, b)
    assert e.value.code == 2


@pytest.mark.parametrize("M,N,K,passes", [(300, 500, 200, 2), (700, 1030, 2048, 2), (2048, 512, 454, 3)])
def test_split_gemm_is_fp32_accurate(tpc, M, N, K, passes):
    """fp32 operands as bf16 hi/lo pairs: the product matches fp64 to fp32 accumulation accuracy
    (a bf16 operand rounding alone would leave errors near 2^-9 relative)."""
    import torch
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    A = torch.randn(M, K, device="cuda", generator=g)
    if passes == 2:
        W = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
        ah, al = tpc.split_bf16(A)
        C = tpc.tpc_gemm_split(ah, al, W, None)
        ref = A.double() @ W.double().t()
    else:  # weight-gradient form: both operands fp32 and stored MN-major ([K][M], [K][N])
        Bt = torch.randn(K, N, device="cuda", generator=g)
        At = A.t().contiguous()
        ah, al = tpc.split_bf16(At)
        bh, bl = tpc.split_bf16(Bt)
        C = tpc.tpc_gemm_split(ah, al, bh, bl, a_mn=True, b_mn=True)
        ref = A.double() @ Bt.double()
    torch.cuda.synchronize()
    err = ((C.double() - ref).abs().max() / ref.pow(2).mean().sqrt()).item()
    assert err < 1e-4, err
