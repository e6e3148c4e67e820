"""CPU tests of the synthetic input generator (shapes, value ranges, determinism, packed lengths)."""
import numpy as np
import torch

from gated_delta_rule_105_b200.inputs import WORKLOADS, draw_lengths, generate


def test_shapes_ranges_and_determinism():
    a = generate(2, 70, 3, 64, 128, "bf16", seed=5, h0_std=0.02)
    b = generate(2, 70, 3, 64, 128, "bf16", seed=5, h0_std=0.02)
    for key in ("q", "k", "v", "g", "beta", "h0"):
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (2, 70, 3, 64) and a["v"].shape == (2, 70, 3, 128)
    assert a["q"].dtype == torch.bfloat16 and a["g"].dtype == torch.float32
    assert (a["g"] < 0).all() and ((a["beta"] > 0) & (a["beta"] < 1)).all()
    norms = a["k"].float().norm(dim=-1)
    assert torch.allclose(norms, torch.ones_like(norms), atol=1e-2)
    assert a["h0"].shape == (2, 3, 64, 128) and abs(a["h0"].std().item() - 0.02) < 2e-3
    assert a["scale"] == 64 ** -0.5


def test_gdn2_gates():
    a = generate(1, 33, 2, 64, 64, "f32", seed=1, variant="gdn2")
    assert a["g"].shape == (1, 33, 2, 64) and a["b"].shape == (1, 33, 2, 64) and a["w"].shape == (1, 33, 2, 64)
    assert (a["g"] < 0).all() and ((a["b"] > 0) & (a["b"] < 1)).all() and ((a["w"] > 0) & (a["w"] < 1)).all()
    assert a["q"].dtype == torch.float32


def test_packed_lengths():
    rng = np.random.Generator(np.random.PCG64(3))
    for _ in range(20):
        lens = draw_lengths(rng, 16, 65536, 512, 8192)
        assert lens.sum() == 65536 and lens.min() >= 512 and lens.max() <= 8192


def test_workload_table():
    w = WORKLOADS["gdn_bf16_b4h16t4096_dk128_dv256_h0"]
    assert (w.B, w.T, w.H, w.dk, w.dv, w.dtype) == (4, 4096, 16, 128, 256, "bf16") and w.h0_std == 0.02
    assert WORKLOADS["gdn_bf16_varlen65536x16_h16_dk128_dv256"].n_seqs == 16
    assert WORKLOADS["gdn2_bf16_b4h16t4096_dk128_dv128"].variant == "gdn2"
