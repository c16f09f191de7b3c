"""The final division of a folded row (out = A / L) as every attention call
computes it -- the row's reciprocal once, then two residual corrections --
against the IEEE quotient (torch's float32 division on the GPU), bit for bit,
over random and edge-case operands."""
import pytest
import torch

import paged_kv_decode_31_b200 as pkv

pytestmark = pytest.mark.gpu


def _expected(A, L):
    return torch.where(L > 0, A / L, torch.zeros_like(A))


def _same_bits(got, ref):
    nan = torch.isnan(ref)
    assert torch.equal(torch.isnan(got), nan)
    g = got.view(torch.int32)[~nan]
    r = ref.view(torch.int32)[~nan]
    bad = (g != r).nonzero()
    assert bad.numel() == 0, f"{bad.numel()} quotients differ, first at {int(bad[0])}"


def test_matches_ieee_division_on_random_operands():
    gen = torch.Generator(device="cuda").manual_seed(5)
    n = 1 << 24
    # |A| log-uniform over 2^[-140, 140] (past both fast-path bounds), random
    # signs; L as a row sum: log-uniform over [1, 2^31]
    e = torch.rand(n, generator=gen, device="cuda") * 280.0 - 140.0
    sgn = torch.where(torch.rand(n, generator=gen, device="cuda") < 0.5, -1.0, 1.0)
    A = (sgn * torch.exp2(e.double())).float()
    L = torch.exp2(torch.rand(n, generator=gen, device="cuda").double() * 31.0).float()
    _same_bits(pkv.binding.debug_final_out(A, L), _expected(A, L))
    # dense mantissas in one binade: every rounding position of the quotient
    A2 = 1.0 + torch.rand(n, generator=gen, device="cuda")
    L2 = 1.0 + torch.rand(n, generator=gen, device="cuda")
    _same_bits(pkv.binding.debug_final_out(A2, L2), _expected(A2, L2))
    _same_bits(pkv.binding.debug_final_out(-A2 * 3.0e-20, L2 * 7.0e5),
               _expected(-A2 * 3.0e-20, L2 * 7.0e5))


def test_matches_ieee_division_on_edge_operands():
    f = torch.finfo(torch.float32)
    specials = [0.0, -0.0, float("inf"), float("-inf"), float("nan"), f.tiny, -f.tiny,
                f.tiny / 8, f.max, -f.max, 1.0, -1.0, 3.0, 0.1, 2.0 ** -90, 2.0 ** 96,
                2.0 ** -90 * (1 - 2 ** -24), 2.0 ** 96 * (1 + 2 ** -23), 2.0 ** -100, 2.0 ** 100,
                1.0 - 2 ** -24, 1.0 + 2 ** -23]
    Ls = [1.0, 2.0, 3.0, 0.5, 2.0 ** 31, 2.0 ** 40, 2.0 ** 41, 2.0 ** -20, 2.0 ** -21, f.tiny,
          0.0, -0.0, -1.0, float("inf"), float("nan"), 1.0 + 2 ** -23, 1.9999999, 7.0, 1e-30]
    A = torch.tensor(specials, dtype=torch.float32).repeat_interleave(len(Ls)).cuda()
    L = torch.tensor(Ls, dtype=torch.float32).repeat(len(specials)).cuda()
    _same_bits(pkv.binding.debug_final_out(A, L), _expected(A, L))
