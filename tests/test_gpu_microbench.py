"""The exponential-unit rate bench.py divides the attention kernel's exponentials by: measured
with CUDA events, it must be a plausible number of ex2 per clock per SM (the nominal figure is 16;
a result far off means the microbenchmark is not measuring the unit)."""
import os
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_ex2_rate_is_plausible():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bench
    from ragged_varlen_attention_rra_b200 import build
    build.build_microbench()
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    rate = bench.measure_ex2_rate(torch.cuda.Stream(), n_sms)
    assert rate is not None
    per_clk = rate / (n_sms * 1965e6)  # at the B200's maximum SM clock
    assert 4 <= per_clk <= 64, per_clk
