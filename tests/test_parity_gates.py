"""The two parity gates themselves, on hand-made arrays (no GPU): what each
one measures and the case the elementwise gate exists for."""
import numpy as np
import pytest

from parity_util import FLOOR_TOL, TOL, checked_err, rel_err_rms_floor, scaled_err


def test_scaled_error_is_max_error_over_max_reference():
    ref = np.array([4.0, -2.0, 0.5])
    got = np.array([4.0, -2.1, 0.5])
    assert scaled_err(got, ref) == pytest.approx(0.1 / 4.0)


def test_rms_floor_error_by_hand():
    ref = np.array([3.0, 0.0, -4.0, 0.0])          # rms = 2.5
    got = np.array([3.0, 0.05, -4.0, 0.0])
    assert rel_err_rms_floor(got, ref) == pytest.approx(0.05 / 2.5)
    got = np.array([3.3, 0.0, -4.0, 0.0])
    assert rel_err_rms_floor(got, ref) == pytest.approx(0.3 / 5.5)


def test_error_on_a_small_output_passes_scaled_gate_and_fails_elementwise_gate():
    # normal outputs (max ~4 rms): an error of 0.06 rms on the output nearest
    # zero is under 2 % of the largest output but 6 % of the rms floor
    rng = np.random.default_rng(1)
    ref = rng.standard_normal(4096)
    ref /= np.sqrt(np.mean(ref * ref))
    got = ref.copy()
    got[np.argmin(np.abs(ref))] += 0.06
    assert scaled_err(got, ref) <= TOL["bf16"]
    assert rel_err_rms_floor(got, ref) > FLOOR_TOL["bf16"]
    with pytest.raises(AssertionError, match="rms floor"):
        checked_err(got, ref, "bf16", "small output")


def test_bf16_rounding_passes_both_gates():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(4096)
    # round to an 8-bit mantissa, the output rounding of a bf16 kernel
    m, e = np.frexp(ref)
    got = np.ldexp(np.round(m * 256.0) / 256.0, e)
    assert checked_err(got, ref, "bf16") <= TOL["bf16"]
    assert rel_err_rms_floor(got, ref) <= 2.0 ** -8


def test_zero_reference():
    assert rel_err_rms_floor(np.zeros(3), np.zeros(3)) == 0.0
    assert rel_err_rms_floor(np.array([0.0, 1e-3, 0.0]), np.zeros(3)) == pytest.approx(1e-3)
