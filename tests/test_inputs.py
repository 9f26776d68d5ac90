"""Seeded generators and the host FP8 quantiser (input preparation shared by both sides)."""

import numpy as np
import torch

from oracle import fp_formats
from sparse_attention_token_indexer_b200 import inputs


def test_quantiser_round_trip_and_saturation():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(64, 3, 32, generator=g)
    codes, scale = inputs.quantize_e4m3_rows(x)
    back = fp_formats.dequantize(codes.numpy(), scale.numpy(), "e4m3")
    xf = x.double().numpy()
    amax = np.abs(xf).reshape(64, -1).max(axis=1)
    # the row maximum lands on +-448 exactly; e4m3 keeps 3 mantissa bits (half-ulp 2^-4)
    assert np.all(np.abs(fp_formats.e4m3_to_f64(codes.numpy())).reshape(64, -1).max(axis=1) == 448.0)
    err = np.abs(back - xf)
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, 2.0 ** -10 * scale.double().numpy()[:, None, None])
    assert np.all(err <= bound * (1 + 1e-6))
    assert np.allclose(scale.numpy(), amax / 448.0, rtol=1e-6)


def test_zero_row_gets_unit_scale():
    codes, scale = inputs.quantize_e4m3_rows(torch.zeros(2, 8))
    assert torch.all(codes == 0) and torch.all(scale == 1.0)


def test_generators_are_seeded_and_shaped():
    a = inputs.tiny_prefill(seed=0)
    b = inputs.tiny_prefill(seed=0)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["k"], b["k"]) and torch.equal(a["w"], b["w"])
    assert a["q"].shape == (1024, 4, 64) and a["k"].shape == (1024, 64) and a["w"].shape == (1024, 4)
    p = inputs.group_prefill(256, H=8, d=32, K=16, G=16, B=64, Hg=4)
    assert p["qbar"].shape == (16, 4, 32) and p["wbar"].shape == (16, 4)
    d = inputs.decode_problem(Bs=2, S=600, H=4, d=32, K=8, Hg=2, steps=3)
    assert d["k"].shape == (2, 602, 32) and d["q_steps"].shape == (3, 2, 4, 32)
    assert inputs.decode_seq_len(d, 2).tolist() == [602, 602]
