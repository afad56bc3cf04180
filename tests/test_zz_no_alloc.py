"""fp8q_quantize_tensor_noalloc: per-tensor quantization for callers that cannot let a library
allocate device memory (an application whose own allocator owns all device memory, or one
under a fixed memory budget where a lazy allocation could fail mid-run).  Its scratch is the
library's fixed device array instead of the pool fp8q_quantize_tensor allocates.

Checked through the C ABI against the allocating entry point, bit for bit (the tolerance the
quantizer tests use), on two calls in a row.  The second input has a much smaller amax than
the first, so a scratch word left over from the first call would change its scale."""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _call(fn, x, q, s_dec):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.c_void_p(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0),
              ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(s_dec.data_ptr()), stream)


def test_noalloc_matches_allocating_entry_point_on_two_calls(cuda_lib):
    L = cuda_lib.lib()
    inputs = [workloads.normal_bf16((300, 648), 1.0, 901, 1e-3, 50.0),
              workloads.normal_bf16((256, 1024), 0.01, 902)]
    scales = []
    for x in inputs:
        x = x.cuda()
        q_ref = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
        s_ref = torch.empty((1,), dtype=torch.float32, device="cuda")
        assert _call(L.fp8q_quantize_tensor, x, q_ref, s_ref) == 0
        q = torch.full(x.shape, 0xAA, dtype=torch.uint8, device="cuda")
        s = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        assert _call(L.fp8q_quantize_tensor_noalloc, x, q, s) == 0
        torch.cuda.synchronize()
        assert torch.equal(q, q_ref)
        assert s.cpu().numpy().view(np.uint32)[0] == s_ref.cpu().numpy().view(np.uint32)[0]
        scales.append(float(s.item()))
    assert scales[1] < scales[0] / 10      # the second call did not reuse the first call's amax
