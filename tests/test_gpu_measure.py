"""The measurement helpers of the C ABI on a GPU: the SM clock trace
(flkl_clock_trace) gives increasing timestamps and a clock within the part's
range, and flkl_gemm_ctas reports an even number of SMs no larger than the
device's SM count."""

from __future__ import annotations

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_clock_trace_samples_a_plausible_sm_clock():
    import lm_head_projection_b200 as pkg

    n, iv = 200, 20_000
    buf = torch.zeros(2 * n, dtype=torch.int64, device="cuda")
    assert pkg.flkl_clock_trace(buf.data_ptr(), n, iv,
                                torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    t, c = buf[0::2].cpu(), buf[1::2].cpu()
    assert bool((t[1:] > t[:-1]).all()) and bool((c[1:] > c[:-1]).all())
    # sample i is taken once the timer passes start + i * interval (the first
    # one as soon as the kernel runs): about n * interval in all
    span = int(t[-1] - t[0])
    assert (n - 2) * iv <= span <= 20 * (n - 1) * iv
    mhz = float(c[-1] - c[0]) / span * 1e3
    props = torch.cuda.get_device_properties(0)
    assert 50.0 < mhz < 4000.0, mhz
    # argument checks
    assert pkg.flkl_clock_trace(buf.data_ptr(), 0, iv, None) == 1
    assert pkg.flkl_clock_trace(buf.data_ptr(), n, 10, None) == 1
    assert props.multi_processor_count > 0


def test_gemm_ctas_fit_the_device():
    import lm_head_projection_b200 as pkg

    n = pkg.flkl_gemm_ctas()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert n > 0 and n % 2 == 0 and n <= sms
