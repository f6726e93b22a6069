"""The INT8 tensor-core peak probe (ck_test_i8_mma_peak), which gives the
GEMM's roofline a measured denominator: it must run clean on the device and
report a plausible rate."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_i8_mma_peak_probe_runs_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int8_quantized_linear_convrot256_b200 as ck

    ck.clear_device_error()
    stream = torch.cuda.current_stream()
    ck.test_i8_mma_peak(2000, stream=stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    ops = ck.test_i8_mma_peak(50000, stream=stream)
    e1.record(stream)
    e1.synchronize()
    tops = ops / (e0.elapsed_time(e1) / 1e3) / 1e12
    assert ck.device_error() == ck.CK_OK
    assert 1000.0 < tops < 6000.0, tops
