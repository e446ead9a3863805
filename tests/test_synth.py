"""The shared input generators: both evaluations of the counter-based weights agree."""
import numpy as np
import pytest

import synth


def test_weight_generators_agree_on_cpu():
    torch = pytest.importorskip("torch")
    case = synth.MoeCase("t", 8, 64, 96, 3, 2, 0, "none", seed=4)
    wg, wu, wd = synth.expert_weights_torch(case, "cpu")
    for e in range(case.E):
        for which, t in enumerate((wg, wu, wd)):
            ref = synth.expert_weight_bits(case, e, which)
            got = t[e].contiguous().view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(got, ref)
    up = synth.expert_weights_uploaded(case, "cpu")
    for a, b in zip(up, (wg, wu, wd)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_weight_statistics():
    case = synth.CONFIGS["mid"]
    wg = synth.bf16_bits_to_f32(synth.expert_weight_bits(case, 3, 0)).astype(np.float64)
    assert abs(wg.mean()) < 1e-3
    assert abs(wg.std() * np.sqrt(case.d) - 1.0) < 0.01


def test_bf16_rounding_ties_to_even():
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)
    assert synth.f32_to_bf16_bits(v).tolist() == [0x3F80, 0x3F82, 0xBF80]
