"""The SFU exp2 rate the scan's roofline divides by, measured on the GPU
(ssm_measure_ex2_rate), against the rate derived from the SM count, 16 exp2
per clock per SM and the maximum SM clock."""
import pytest
import torch

import selective_state_space_51_b200 as S

pytestmark = pytest.mark.gpu


def test_ex2_rate_matches_the_derived_peak():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    derived = sms * 16 * 1965e6
    rate = S.ssm_measure_ex2_rate(0)
    # clocks below the maximum (power cap) lower the rate; more than the
    # derived peak would mean the kernel is not doing its work
    assert 0.5 * derived < rate < 1.1 * derived, (rate, derived)


def test_ex2_rate_rejects_bad_arguments():
    import ctypes
    lib = S.library()
    out = ctypes.c_double()
    assert lib.ssm_measure_ex2_rate(-1, ctypes.byref(out)) == S.SSM_ERR_INVALID
    assert lib.ssm_measure_ex2_rate(0, None) == S.SSM_ERR_INVALID
