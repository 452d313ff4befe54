"""The tcgen05 GEMM core against a float64 matmul of the same bf16 operands, for every
operand layout the block uses (K-major and MN-major A and B), on sizes that span
several 128 x 256 x 64 tiles and leave ragged tails in M, N and K."""
import numpy as np
import pytest
import torch

from _helpers import dev, rms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from capacity_limited_routed_b200 import moe
    return moe


def _operands(m, n, k, seed):
    rng = np.random.default_rng(seed)
    a = torch.from_numpy(rng.standard_normal((m, k), dtype=np.float32)).to(torch.bfloat16)
    b = torch.from_numpy(rng.standard_normal((n, k), dtype=np.float32)).to(torch.bfloat16)
    return a, b


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("mnk", [(128, 256, 64), (296, 264, 200), (1000, 776, 1048)])
def test_gemm_layouts_f32(M, a_mn, b_mn, mnk):
    m, n, k = mnk
    a, b = _operands(m, n, k, seed=m + n + k + 2 * a_mn + b_mn)
    ref = a.double() @ b.double().T
    A = (a.T.contiguous() if a_mn else a).to(dev())
    B = (b.T.contiguous() if b_mn else b).to(dev())
    D = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    M.moe_gemm_bf16(m, n, k, A, a_mn, B, b_mn, D, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = D.double().cpu()
    err = (got - ref).abs().max().item()
    assert err <= 1e-4 * rms(ref.numpy()) * np.sqrt(k / 64), err


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1), (1, 0)])
def test_gemm_bf16_output(M, a_mn, b_mn):
    m, n, k = 520, 392, 320
    a, b = _operands(m, n, k, seed=5)
    ref = (a.double() @ b.double().T)
    A = (a.T.contiguous() if a_mn else a).to(dev())
    B = (b.T.contiguous() if b_mn else b).to(dev())
    D = torch.zeros((m, n), dtype=torch.bfloat16, device=dev())
    M.moe_gemm_bf16(m, n, k, A, a_mn, B, b_mn, D)
    got = D.double().cpu()
    # one bf16 rounding of a float32 sum
    assert ((got - ref).abs() <= 2.0 ** -8 * ref.abs() + 1e-3 * rms(ref.numpy())).all()


def test_gemm_single_tile_exact_small_integers(M):
    """Small integers multiply and add exactly in float32: the result must be exact."""
    m, n, k = 128, 256, 192
    rng = np.random.default_rng(1)
    a = torch.from_numpy(rng.integers(-3, 4, size=(m, k)).astype(np.float32)).to(torch.bfloat16)
    b = torch.from_numpy(rng.integers(-3, 4, size=(n, k)).astype(np.float32)).to(torch.bfloat16)
    ref = a.double() @ b.double().T
    D = torch.zeros((m, n), dtype=torch.float32, device=dev())
    M.moe_gemm_bf16(m, n, k, a.to(dev()), 0, b.to(dev()), 0, D)
    assert torch.equal(D.double().cpu(), ref)


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1), (1, 0)])
@pytest.mark.parametrize("n", [96, 160])
def test_gemm_partial_tiles_many(M, a_mn, b_mn, n):
    """Output widths that leave most of each 256-wide tile empty, over many tiles and a
    short contraction: the epilogue's staging buffers must never be rewritten while a
    store still reads them."""
    m, k = 4096, 64
    a, b = _operands(m, n, k, seed=n + 2 * a_mn + b_mn)
    ref = a.double() @ b.double().T
    A = (a.T.contiguous() if a_mn else a).to(dev())
    B = (b.T.contiguous() if b_mn else b).to(dev())
    for _ in range(3):
        D = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev())
        M.moe_gemm_bf16(m, n, k, A, a_mn, B, b_mn, D)
        torch.cuda.synchronize()
        err = (D.double().cpu() - ref).abs().max().item()
        assert err <= 1e-4 * rms(ref.numpy()), err


@pytest.mark.parametrize("k", [64, 130, 384, 448, 449])
def test_gemm_weight_gradient_short_contractions(M, k):
    """Both operands MN-major with a float32 result (the weight-gradient form) at the
    contraction lengths of an expert's rows (a few 64-deep blocks, ragged tails), over
    several 256-row slabs and n-tiles with ragged edges, twice in a row."""
    m, n = 776, 520
    a, b = _operands(m, n, k, seed=k)
    ref = a.double() @ b.double().T
    A, B = a.T.contiguous().to(dev()), b.T.contiguous().to(dev())
    for _ in range(2):
        D = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev())
        M.moe_gemm_bf16(m, n, k, A, 1, B, 1, D)
        torch.cuda.synchronize()
        err = (D.double().cpu() - ref).abs().max().item()
        assert err <= 1e-4 * rms(ref.numpy()) * max(1.0, np.sqrt(k / 64)), err


def test_gemm_weight_gradient_full_token_contraction(M):
    """The dense weight-gradient form at the block's full size: both operands MN-major,
    K = 16,384 tokens, a [6144][3072] float32 result (the latent-projection and shared
    weight gradients of the training step), checked on sampled output rows against a
    float64 contraction of the same bf16 operands."""
    m, n, k = 6144, 3072, 16384
    gen = torch.Generator(device=dev()).manual_seed(77)
    A = torch.randn((k, m), generator=gen, device=dev()).to(torch.bfloat16)   # [K][M]
    B = torch.randn((k, n), generator=gen, device=dev()).to(torch.bfloat16)   # [K][N]
    D = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    M.moe_gemm_bf16(m, n, k, A, 1, B, 1, D, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert bool(torch.isfinite(D).all().item())
    rows = np.sort(np.random.default_rng(3).choice(m, size=24, replace=False))
    rows = np.unique(np.concatenate([rows, [0, 255, 256, m - 1]]))
    a_h = A[:, torch.from_numpy(rows).to(dev())].double().cpu().numpy()        # [K][rows]
    b_h = B.double().cpu().numpy()                                            # [K][N]
    ref = a_h.T @ b_h
    got = D[torch.from_numpy(rows).to(dev())].double().cpu().numpy()
    err = np.abs(got - ref).max()
    # float32 accumulation of 16,384 products of unit-variance terms
    assert err <= 1e-4 * rms(ref) * np.sqrt(k / 64), err
