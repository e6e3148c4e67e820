"""The tensor-core operand layouts (128B-swizzled K-major and MN-major, M = 128; bf16 and tf32) give A @ B."""
import pytest
import torch

pytestmark = pytest.mark.gpu

SHAPES = {0: (128, 64, 128), 1: (128, 64, 64), 2: (128, 128, 64), 3: (128, 64, 128), 4: (128, 64, 64),
          5: (128, 64, 32)}


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4, 5])
def test_umma_layout_selftest(mode):
    from gated_delta_rule_105_b200.binding import check_error, umma_selftest
    M, N, K = SHAPES[mode]
    g = torch.Generator().manual_seed(mode)
    A = torch.randn(M, K, generator=g).bfloat16().float()
    B = torch.randn(K, N, generator=g).bfloat16().float()
    D = umma_selftest(A.cuda(), B.cuda(), mode)
    check_error()
    ref = (A.double() @ B.double()).float()
    err = (D.cpu() - ref).abs().max().item()
    assert err < 1e-3 * ref.abs().max().item(), f"mode {mode}: max err {err}"
