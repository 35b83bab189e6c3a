"""The parity checker's two error figures (host logic, no GPU)."""
import numpy as np
import pytest

from tests.gpu_helpers import REPORT, check_close, elem_err_per_head, rel_err_per_head


def test_per_head_and_per_element_figures():
    ref = np.array([[[1.0, 1e-4, -2.0]], [[0.5, 0.25, 0.0]]])
    got = ref.copy()
    got[0, 0, 1] = 2e-4            # 1e-4 off on an element below the floor (1e-3 * 2)
    got[1, 0, 2] = 1e-3            # 1e-3 off on a zero element (floor 1e-3 * 0.5)
    assert rel_err_per_head(got, ref) == pytest.approx(max(1e-4 / 2.0, 1e-3 / 0.5))
    assert elem_err_per_head(got, ref) == pytest.approx(max(1e-4 / 2e-3, 1e-3 / 5e-4))


def test_check_close_records_and_asserts():
    n = len(REPORT)
    ref = np.ones((1, 4, 4))
    check_close(ref * (1 + 1e-3), ref, label="ok")
    assert REPORT[-1]["label"] == "ok" and len(REPORT) == n + 1
    with pytest.raises(AssertionError):
        check_close(ref * 1.5, ref, label="off")
