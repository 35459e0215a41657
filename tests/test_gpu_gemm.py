"""The tensor-core GEMM core (tcgen05 + TMEM + TMA) against an fp32 torch
reference of the same product, through the C ABI."""
import pytest
import torch

pytestmark = pytest.mark.gpu

CASES = [
    # M, N, K, batch, b_kmajor, tile (128/256: one CTA; 512: CTA pair)
    (128, 256, 64, 1, True, 256),       # one tile, one k-block
    (128, 256, 64, 1, False, 256),
    (256, 512, 1024, 1, True, 256),     # several tiles, 16 k-blocks
    (256, 512, 1024, 1, False, 256),
    (1024, 1024, 1024, 3, True, 256),   # batched
    (1024, 1024, 1024, 3, False, 256),
    (1024, 1024, 1024, 2, True, 128),
    (1024, 1024, 1024, 2, False, 128),
    (200, 72, 136, 2, True, 256),       # ragged M, N, K (partial tiles, OOB zero fill)
    (200, 72, 136, 2, False, 256),
    (64, 64, 256, 5, True, 256),        # M smaller than the 128-row tile
    (300, 1000, 520, 1, False, 128),
    (8, 8, 8, 1, True, 256),            # tiny
    (8, 8, 8, 1, False, 128),
    # CTA-pair kernel (tcgen05 cta_group::2, 256 x 256 tiles)
    (256, 256, 64, 1, True, 512),
    (256, 256, 64, 1, False, 512),
    (1024, 1024, 1024, 3, True, 512),
    (1024, 1024, 1024, 3, False, 512),
    (512, 768, 4096, 2, False, 512),
    (300, 1000, 520, 2, True, 512),     # ragged: partial pair tiles, OOB zero fill
    (300, 1000, 520, 2, False, 512),
    (64, 64, 256, 3, True, 512),        # M smaller than one CTA's half
    (2048, 2048, 256, 1, True, 512),
]


@pytest.mark.parametrize("M,N,K,batch,kmajor,tile", CASES)
def test_gemm_matches_fp32_reference(dmuon_lib, M, N, K, batch, kmajor, tile):
    g = torch.Generator(device="cuda").manual_seed(M * 131 + N * 7 + K + batch)
    A = torch.randn(batch, M, K, device="cuda", generator=g).bfloat16()
    B = (torch.randn(batch, N, K, device="cuda", generator=g) if kmajor
         else torch.randn(batch, K, N, device="cuda", generator=g)).bfloat16()
    C = torch.randn(batch, M, N, device="cuda", generator=g).bfloat16()
    D = torch.full((batch, M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    alpha, beta = 0.75, -1.5
    dmuon_lib.dmuon_gemm_bf16(A, B, D, alpha=alpha, beta=beta, C=C, b_kmajor=kmajor, tile=tile)
    torch.cuda.synchronize()
    Bf = B.float().transpose(-1, -2) if kmajor else B.float()
    ref = alpha * torch.bmm(A.float(), Bf) + beta * C.float()
    err = (D.float() - ref).abs()
    # bf16 output rounding (2^-9 relative) plus fp32 accumulation-order noise
    tol = ref.abs() * 2.0 ** -8 + 1e-5 * K ** 0.5 * 4
    assert torch.isfinite(D.float()).all()
    bad = (err > tol).sum().item()
    assert bad == 0, f"{bad} elements off; max err {err.max().item():.3e}"


def test_gemm_without_addend_and_alpha(dmuon_lib):
    A = torch.randn(2, 256, 512, device="cuda").bfloat16()
    D = torch.empty(2, 256, 256, device="cuda", dtype=torch.bfloat16)
    dmuon_lib.dmuon_gemm_bf16(A, A, D, alpha=2.0, beta=0.0, C=None, b_kmajor=True)
    torch.cuda.synchronize()
    ref = 2.0 * torch.bmm(A.float(), A.float().transpose(1, 2))
    assert torch.allclose(D.float(), ref, rtol=2 ** -7, atol=1e-3)
    # X X^T is symmetric up to bf16 rounding
    assert torch.allclose(D.float(), D.float().transpose(1, 2), rtol=2 ** -7, atol=1e-3)


@pytest.mark.parametrize("tile", [256, 512])
def test_gemm_deterministic(dmuon_lib, tile):
    A = torch.randn(4, 512, 1024, device="cuda").bfloat16()
    B = torch.randn(4, 1024, 768, device="cuda").bfloat16()
    D1 = torch.empty(4, 512, 768, device="cuda", dtype=torch.bfloat16)
    D2 = torch.empty_like(D1)
    dmuon_lib.dmuon_gemm_bf16(A, B, D1, b_kmajor=False, tile=tile)
    dmuon_lib.dmuon_gemm_bf16(A, B, D2, b_kmajor=False, tile=tile)
    torch.cuda.synchronize()
    assert torch.equal(D1, D2)


SYM_CASES = [(1024, 1024, 2, 256), (1024, 512, 2, 512), (1000, 520, 1, 128), (1000, 520, 1, 512),
             (200, 136, 3, 256), (128, 64, 1, 512), (2048, 256, 1, 512), (776, 96, 2, 256)]


@pytest.mark.parametrize("M,K,batch,tile", SYM_CASES)
@pytest.mark.parametrize("form", ["gram", "square"])
def test_gemm_symmetric_output(dmuon_lib, M, K, batch, tile, form):
    """sym = 1: only blocks on or above the block diagonal run; blocks above
    it are also stored mirrored.  Checked on X X^T (K-major) and on S S for a symmetric S
    (MN-major right operand) with a symmetric addend, against fp32 torch."""
    g = torch.Generator(device="cuda").manual_seed(M + K * 3 + batch + tile)
    D = torch.full((batch, M, M), float("nan"), device="cuda", dtype=torch.bfloat16)
    if form == "gram":
        X = torch.randn(batch, M, K, device="cuda", generator=g).bfloat16()
        dmuon_lib.dmuon_gemm_bf16(X, X, D, alpha=0.5, b_kmajor=True, tile=tile, sym=True)
        ref = 0.5 * torch.bmm(X.float(), X.float().transpose(1, 2))
    else:
        R = torch.randn(batch, M, M, device="cuda", generator=g)
        S = (R + R.transpose(1, 2)).bfloat16()
        dmuon_lib.dmuon_gemm_bf16(S, S, D, alpha=-2.0, beta=1.5, C=S, b_kmajor=False, tile=tile, sym=True)
        ref = -2.0 * torch.bmm(S.float(), S.float()) + 1.5 * S.float()
    torch.cuda.synchronize()
    Df = D.float()
    assert torch.isfinite(Df).all(), "unwritten elements"
    # blocks off the block diagonal are mirrored (exactly symmetric); diagonal
    # blocks are computed in full, symmetric up to rounding
    assert torch.allclose(Df, Df.transpose(1, 2), rtol=2 ** -7, atol=1e-3 * Df.abs().max().item())
    Kk = K if form == "gram" else M
    tol = ref.abs() * 2.0 ** -8 + 1e-5 * Kk ** 0.5 * 8
    bad = ((Df - ref).abs() > tol).sum().item()
    assert bad == 0, f"{bad} elements off; max err {(Df - ref).abs().max().item():.3e}"
