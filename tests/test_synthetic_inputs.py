"""The seeded input module: determinism and one-step bf16 rounding."""
import numpy as np
import torch

from synthetic import bf16_bits_to_f64, normal, round_to_bf16, sample


def test_seeded_and_deterministic():
    a = normal(5, (3, 7))
    b = normal(5, (3, 7))
    c = normal(6, (3, 7))
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    s = sample(5, (3, 7), "f32")
    assert s.stored.dtype == np.float32
    assert np.array_equal(s.exact, a.astype(np.float32).astype(np.float64))


def test_bf16_matches_torch_on_float32_values():
    v = normal(7, (4096,)).astype(np.float32)
    ours = round_to_bf16(v.astype(np.float64))
    theirs = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_bf16_ties_to_even_and_roundtrip():
    # 1 + 2^-8 lies half way between bf16 neighbours 1 and 1 + 2^-7: ties to even -> 1
    assert bf16_bits_to_f64(round_to_bf16(np.array([1.0 + 2.0 ** -8])))[0] == 1.0
    # 1 + 3 * 2^-8 is half way between 1 + 2^-7 and 1 + 2^-6: ties to even -> 1 + 2^-6
    assert bf16_bits_to_f64(round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8])))[0] == 1.0 + 2.0 ** -6
    # no double rounding: just above the tie goes up even though float32 would tie
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert bf16_bits_to_f64(round_to_bf16(np.array([x])))[0] == 1.0 + 2.0 ** -7
    s = sample(8, (1000,), "bf16")
    assert np.array_equal(round_to_bf16(s.exact), s.stored)
    assert np.abs(s.exact - normal(8, (1000,))).max() <= 2.0 ** -8 * 4.5
