"""The int8 tensor-core rate measurement (bitlinear_measure_i8_peak) runs,
reports no timeout, and gives a rate in the range a B200 can have: dense
int8 is nominally 4.5 POPS (8192 int8 MAC per clock per SM, 148 SMs, about
1.9 GHz); the measured figure must be positive and below 1.2 x that."""

import pytest
import torch

import bitlinear_fwd_b200 as bl

pytestmark = pytest.mark.gpu


def test_i8_peak_is_plausible():
    assert torch.cuda.is_available()
    r = bl.measure_i8_peak(iters=2000, reps=2)
    assert r["grid"] == torch.cuda.get_device_properties(0).multi_processor_count
    assert 500.0 < r["tops"] < 1.2 * 4500.0, r
