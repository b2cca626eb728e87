"""The seeded input generator: deterministic, standard normal, correct rounding."""
import numpy as np
import torch

import synth


def test_deterministic_and_counter_addressable():
    a = synth.normal(123, 4, (1000,), "f64")
    b = synth.normal(123, 4, (1000,), "f64")
    np.testing.assert_array_equal(a, b)
    tail = synth.normal(123, 4, (10,), "f64", offset=990)
    np.testing.assert_array_equal(a[990:], tail)
    assert not np.array_equal(a, synth.normal(123, 5, (1000,), "f64"))
    assert not np.array_equal(a, synth.normal(124, 4, (1000,), "f64"))


def test_moments_standard_normal():
    z = synth.normal(7, 1, (400_000,), "f64")
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    assert abs(((z > 1.96).mean()) - 0.025) < 0.002


def test_rounding_matches_torch():
    z = synth.normal(9, 2, (50_000,), "f64")
    np.testing.assert_array_equal(synth.normal(9, 2, (50_000,), "f32"), z.astype(np.float32))
    bf = torch.from_numpy(z.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.normal(9, 2, (50_000,), "bf16"), bf)
    np.testing.assert_array_equal(synth.round_to(z, "bf16"), bf)
    np.testing.assert_array_equal(synth.widen(bf, "bf16"),
                                  torch.from_numpy(bf.view(np.int16)).view(torch.bfloat16).double().numpy())
