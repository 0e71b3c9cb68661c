"""The seeded input generator: determinism, sub-range regeneration, bf16 rounding."""
import numpy as np

import synth


def test_counter_based_subranges_match_full():
    full = synth.normal(7, 3, 1000)
    assert np.array_equal(full[250:700], synth.normal(7, 3, 450, first=250))
    assert np.array_equal(full, synth.normal(7, 3, 1000))
    assert not np.array_equal(full, synth.normal(8, 3, 1000))
    assert not np.array_equal(full, synth.normal(7, 4, 1000))


def test_normal_moments():
    x = synth.normal(1, 1, 200000, mean=0.5, std=2.0).astype(np.float64)
    assert abs(x.mean() - 0.5) < 0.03 and abs(x.std() - 2.0) < 0.03


def test_logistic_rates_are_positive_and_scaled():
    lr = synth.logistic_normal(1, 4, 10000, denom=64.0)
    assert (lr > 0).all() and (lr < 1 / 64).all() and abs(lr.mean() - 0.5 / 64) < 1e-3


def test_bf16_round_to_nearest_even():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties go to the even one (1.0)
    vals = np.array([1.0, 1 + 2**-8, 1 + 3 * 2**-8, -2.5, 3.0e-3], np.float32)
    got = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(vals))
    assert got[0] == 1.0 and got[1] == 1.0 and got[2] == 1 + 2 * 2**-7 and got[3] == -2.5
    assert abs(got[4] - 3.0e-3) <= 3.0e-3 * 2**-8
    x = synth.normal(2, 2, 10000)
    r = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    assert np.all(np.abs(r - x) <= np.abs(x) * 2**-8)


def test_chain_slices_match_full_tensor():
    w = synth.workload(1, B=2, H=3, L=40)
    full = synth.linear_inputs(w)
    part = synth.linear_inputs(w, chains=[1, 5])
    for k in ("XQ", "XK", "XV", "lr"):
        assert np.array_equal(part[k][0], full[k][0, 1]) and np.array_equal(part[k][1], full[k][1, 2])
