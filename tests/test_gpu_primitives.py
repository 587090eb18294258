"""tcgen05 / TMA building blocks: one 128x128x128 bf16 product per operand form,
checked against a float64 matmul of the same bf16 values."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


@pytest.mark.parametrize("variant", [0, 1, 2, 3])
def test_mma_selftest(nl, variant):
    import torch
    g = torch.Generator().manual_seed(variant)
    a = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    b = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    c = nl.selftest_mma(variant, a.cuda(), b.cuda()).cpu().numpy().astype(np.float64)
    A = a.double().numpy()
    Bm = b.double().numpy()
    want = A @ Bm.T if variant == 0 else A @ Bm
    np.testing.assert_allclose(c, want, rtol=0, atol=2e-3)


@pytest.mark.parametrize("variant", [0, 1])
def test_mma_pair_selftest(nl, variant):
    """A product over a pair of CTAs (M = 256): each CTA holds half of A and of
    B, the even CTA issues the product, each CTA reads its 128 rows of D."""
    import torch
    g = torch.Generator().manual_seed(10 + variant)
    if variant == 0:
        a = torch.randn(256, 128, generator=g).to(torch.bfloat16)
        b = torch.randn(256, 128, generator=g).to(torch.bfloat16)
        want = a.double().numpy() @ b.double().numpy().T
    else:
        a = torch.randn(256, 256, generator=g).to(torch.bfloat16)
        b = torch.randn(256, 128, generator=g).to(torch.bfloat16)
        want = a.double().numpy() @ b.double().numpy()
    c = nl.selftest_mma_pair(variant, a.cuda(), b.cuda()).cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(c, want, rtol=0, atol=4e-3)


def test_arithmetic_rate_selftests(nl):
    """The measured fp64 FMA, fp64 exp and fp32 ex2 rates that serve as roofline
    denominators are finite and within what one GPU can do (fp64 FMA: between 1
    and 200 TFLOP/s; an fp64 exponential costs many FMAs, so its rate in Gexp/s
    stays below the FMA rate in G-FMA/s)."""
    tf = nl.selftest_fp64_tflops()
    gexp = nl.selftest_fp64_exp_rate()
    assert 1.0 < tf < 200.0
    assert 1.0 < gexp < tf * 1e3 / 2
    # the exponential unit: 16 per clock per SM at most, so below 16 * 148 SMs * 2.1 GHz
    ex2 = nl.selftest_ex2_rate()
    assert 100.0 < ex2 < 16 * 148 * 2.1
