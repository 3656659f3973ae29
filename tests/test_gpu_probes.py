"""The library's tensor-core rate probe runs to completion on the GPU (no
timed-out wait, a plausible rate). Its figure is the measured denominator that
the benchmark reports beside the nominal FP4 peak."""

import pytest
import torch

import bit_w4a4_quantized_nvfp4_b200 as svdq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_w4a4_quantized_nvfp4_b200 import build

    build.build()
    svdq.load()


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
def test_mma_probe_runs(mode):
    svdq.probe_mma_peak(64, mode)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fl = svdq.probe_mma_peak(1024, mode)
    e1.record()
    torch.cuda.synchronize()
    assert svdq.device_error() == 0
    tflops = fl / (e0.elapsed_time(e1) * 1e-3) / 1e12
    # far below any tensor-core rate means it did not run as designed; above
    # the 18 PF sparse figure means it did not do the work
    assert 500.0 < tflops < 18000.0, tflops


def test_mma_probe_rejects_bad_arguments():
    with pytest.raises(svdq.SvdqError):
        svdq.probe_mma_peak(0)
    with pytest.raises(svdq.SvdqError):
        svdq.probe_mma_peak(16, mode=5)
