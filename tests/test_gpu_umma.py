"""One-tile checks of the tcgen05 building blocks (K-major S = A B^T and
MN-major O = P V from TMA-loaded, 128B-swizzled shared memory, and P V with
P as a tensor-memory A operand) against a float64 product on the CPU."""
import pytest
import torch

from sparse_attention_context_b200 import api

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,bn", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_umma_tile(cuda_ok, d, bn):
    g = torch.Generator().manual_seed(d * 1000 + bn)
    A = torch.randn(128, d, generator=g).bfloat16()
    B = torch.randn(bn, d, generator=g).bfloat16()
    P = torch.rand(128, bn, generator=g).bfloat16()
    V = torch.randn(bn, d, generator=g).bfloat16()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    S, O, O2 = api.isa_selftest_umma(A.cuda(), B.cuda(), P.cuda(), V.cuda(), ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    S_ref = A.double() @ B.double().T
    O_ref = P.double() @ V.double()
    assert torch.allclose(S.cpu().double(), S_ref, rtol=1e-5, atol=1e-4), (S.cpu().double() - S_ref).abs().max()
    assert torch.allclose(O.cpu().double(), O_ref, rtol=1e-5, atol=1e-4), (O.cpu().double() - O_ref).abs().max()
    assert torch.allclose(O2.cpu().double(), O_ref, rtol=1e-5, atol=1e-4), (O2.cpu().double() - O_ref).abs().max()


def test_umma_pair_tile(cuda_ok):
    """One M = 256 tile on a CTA pair (cta_group::2): each CTA holds 128 rows
    of A, half the keys of B and half the columns of V; both products must
    equal the float64 ones row for row."""
    g = torch.Generator().manual_seed(2561)
    A = torch.randn(256, 128, generator=g).bfloat16()
    B = torch.randn(128, 128, generator=g).bfloat16()
    P = torch.rand(256, 128, generator=g).bfloat16()
    V = torch.randn(128, 128, generator=g).bfloat16()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    S, O = api.isa_selftest_umma_pair(A.cuda(), B.cuda(), P.cuda(), V.cuda(), ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    S_ref = A.double() @ B.double().T
    O_ref = P.double() @ V.double()
    assert torch.allclose(S.cpu().double(), S_ref, rtol=1e-5, atol=1e-4), (S.cpu().double() - S_ref).abs().max()
    assert torch.allclose(O.cpu().double(), O_ref, rtol=1e-5, atol=1e-4), (O.cpu().double() - O_ref).abs().max()
