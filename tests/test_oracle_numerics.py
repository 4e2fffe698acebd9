"""Pins for oracle.numerics: single rounding fp64 -> bf16, nearest, ties to even."""
import numpy as np
import torch

from oracle.numerics import round_to_bf16, round_to_f32


def test_bf16_matches_torch_cast_on_fp32_values():
    # For values that are already fp32, RNE to bf16 is one rounding in both
    # torch (fp32 -> bf16 cast) and the oracle (fp64 -> bf16): they must agree.
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200_000),
        rng.standard_normal(20_000) * 1e-30,
        rng.standard_normal(20_000) * 1e30,
        rng.standard_normal(2_000) * 1e-39,   # bf16 subnormal range
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = round_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_ties_and_single_rounding():
    e = 2.0 ** -8
    cases = {
        1.0 + e: 1.0,                            # tie -> even mantissa (0)
        1.0 + 3 * e: 1.0 + 4 * e,                # tie -> even mantissa (2)
        1.0 + e + 2.0 ** -30: 1.0 + 2 * e,       # just above the tie: up
        1.0 + e - 2.0 ** -30: 1.0,               # just below the tie: down
        -(1.0 + 3 * e): -(1.0 + 4 * e),
        2.0 ** -133: 2.0 ** -133,                # smallest subnormal kept
        2.0 ** -134: 0.0,                        # tie with 0 -> even (0)
        3 * 2.0 ** -134: 2.0 ** -132,            # tie -> even
        0.0: 0.0,
    }
    xs = np.array(list(cases.keys()))
    want = np.array(list(cases.values()))
    assert np.array_equal(round_to_bf16(xs), want)
    # the same value through fp32 first would round twice and land elsewhere
    assert round_to_bf16(np.array([round_to_f32(1.0 + e + 2.0 ** -30)]))[0] == 1.0


def test_f32_rounding_is_nearest():
    x = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 1.0 + 2.0 ** -24 + 2.0 ** -40])
    assert np.array_equal(round_to_f32(x), [1.0, 1.0 + 2.0 ** -22, 1.0 + 2.0 ** -23])
