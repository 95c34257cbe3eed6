"""CPU checks of the parity-test comparison helper: the worst-row error
catches a wrong row of small values that the normwise error alone lets
through."""
import numpy as np

from tests._util import normwise_err, rel_err, row_err


def test_row_error_sees_a_bad_small_row():
    ref = np.ones((4, 8))
    ref[2] *= 1e-2                  # a row of small values
    got = ref.copy()
    got[2] *= 1.5                   # 50 % off on that row only
    assert normwise_err(got, ref) < 1e-2      # hidden by the large rows
    assert abs(row_err(got, ref) - 0.5) < 1e-12
    assert rel_err(got, ref) > 0.49


def test_row_error_floor_for_zero_rows():
    ref = np.ones((3, 4))
    ref[1] = 0.0
    got = ref.copy()
    got[1] = 1e-6                   # absolute error 1e-6 on a zero row
    # judged against 1e-3 of the tensor's max: 1e-3, not infinity
    assert abs(row_err(got, ref) - 1e-3) < 1e-12


def test_exact_and_one_dimensional():
    ref = np.linspace(-2, 3, 17)
    assert rel_err(ref.copy(), ref) == 0.0
    got = ref.copy()
    got[5] += 3e-3
    assert abs(rel_err(got, ref) - 1e-3) < 1e-12
