"""The error metrics of the parity tests (CPU): closed cases."""
import numpy as np
import torch

from tolerance import bf16_floor, bf16_halfulp, err_excess, err_out, err_state, out_report


def test_exact_result_rounded_to_bf16_has_no_excess():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(20000) * np.abs(rng.standard_normal(20000)) * 3
    x = torch.from_numpy(ref).float().bfloat16()
    plain, floor, relaxed, excess = out_report(x, ref)
    assert excess == 0.0
    assert plain == floor > 0.0
    assert relaxed <= 2.0 ** -8 + 1e-12          # at most half an ulp relative


def test_halfulp_of_bf16_values():
    x = np.array([1.0, 1.5, 2.0, 3.0, -0.375, 0.0])
    assert np.allclose(bf16_halfulp(x), [2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 2.0 ** -7, 2.0 ** -10, 0.0])


def test_excess_measures_error_beyond_rounding():
    ref = np.ones(100)
    x = ref.copy()
    x[7] = 1.0 + 0.1                              # 0.1 absolute on one element, rms(ref) = 1
    assert abs(err_excess(x, ref) - (0.1 - 2.0 ** -8)) < 1e-12
    assert abs(err_state(x, ref) - 0.1) < 1e-12


def test_all_zero_reference_uses_absolute_error():
    ref = np.zeros(50)
    assert err_out(np.zeros(50), ref) == 0.0
    assert err_out(np.full(50, 1e-3), ref) == 1e-3
    assert bf16_floor(ref) == 0.0
