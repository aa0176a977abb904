"""The pipe-rate probe (mss_probe_pipe_rates): per SM and clock, the fp32
fma pipe delivers at most its 128 lanes with scalar or packed fma, the
multi-function unit at most 16 ex2 results and shuffles at most 32 results;
a well-fed loop reaches most of each."""
import pytest
import torch

import selective_state_space_mss_b200 as mss

pytestmark = pytest.mark.gpu


def test_pipe_rates_within_unit_counts():
    torch.cuda.set_device(0)
    r = mss.probe_pipe_rates()
    assert set(r) == set(mss.PIPE_RATE_NAMES)
    # upper bounds: the unit counts per SM (a few percent of slack for the
    # cycle counter read outside the loops); lower bounds: half of them
    assert 64.0 < r["ffma"] <= 128.0 * 1.03
    assert 64.0 < r["ffma2"] <= 128.0 * 1.03
    assert 8.0 < r["mufu_ex2"] <= 16.0 * 1.03
    assert 16.0 < r["shfl"] <= 32.0 * 1.03
    assert mss.get_device_error() == 0
