"""Failure detection on the GPU without provoking a fault.  A bounded mbarrier wait that
nothing satisfies gives up after its limit and records FP8Q_ERR_TIMEOUT in the device status
word (the mechanism every GEMM role uses); the kernel exits cleanly, the status read clears
the word, and the context keeps working for ordinary calls afterwards."""
import time

import numpy as np
import pytest

import workloads
from oracle import quant as Q

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_the_context_survives(cuda_lib):
    fq = cuda_lib
    assert fq.device_status() == fq.FP8Q_OK
    t0 = time.perf_counter()
    assert fq.fp8q_selftest_bounded_wait(10_000_000, fq._stream()) == fq.FP8Q_OK   # 10 ms limit
    assert fq.device_status() == fq.FP8Q_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert fq.device_status() == fq.FP8Q_OK          # the read cleared the word

    x = workloads.normal_bf16((256, 512), 1.0, 77)
    q = fq.quantize_1x128(x.cuda())
    assert fq.device_status() == fq.FP8Q_OK
    oq, os_ = Q.quantize_1x128_rowwise(workloads.bf16_bits(x))
    assert np.array_equal(q["q_row"].cpu().numpy(), oq)
    assert np.array_equal(q["s_row"].cpu().numpy().view(np.uint32), os_.astype(np.float32).view(np.uint32))
