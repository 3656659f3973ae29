"""The device conversions the quantisers use (fp32 -> E2M1, fp32 -> E4M3, both
round-to-nearest-even and saturating, and fp32 -> bf16) agree with the CPU
oracle's on every one of the 2^32 fp32 bit patterns. This pins the oracle's
format code against hardware behaviour and the kernels' conversions against
the oracle."""

import numpy as np
import pytest
import torch

import oracle
import bit_w4a4_quantized_nvfp4_b200 as svdq

pytestmark = pytest.mark.gpu


def test_all_fp32_bit_patterns():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_w4a4_quantized_nvfp4_b200 import build

    build.build()
    chunk = 1 << 28
    total_bad = np.zeros(3, np.int64)
    firsts = []
    for start in range(0, 1 << 32, chunk):
        bits = torch.arange(start, start + chunk, dtype=torch.int64, device="cuda").to(torch.int32)
        v = bits.view(torch.float32)
        e2, e4, b16 = svdq.probe_convert(v)
        torch.cuda.synchronize()
        bad, first = oracle.check_cvt_range(start, chunk, e2.cpu().numpy(), e4.cpu().numpy(),
                                            b16.cpu().numpy().view(np.uint16))
        total_bad += bad
        firsts.append(first)
        del bits, v, e2, e4, b16
    assert total_bad.tolist() == [0, 0, 0], (total_bad, [hex(int(f.min())) for f in np.array(firsts).T])
