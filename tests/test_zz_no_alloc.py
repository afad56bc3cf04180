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


_FRESH = r'''
import ctypes, json, os, sys
import numpy as np
import torch
sys.path.insert(0, os.environ["FP8Q_ROOT"])
import fp4_precision_gemm_b200 as fq
import workloads
from oracle import quant as Q

torch.cuda.set_device(0)
L = fq.lib()
stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
P = lambda t: ctypes.c_void_p(t.data_ptr())
xs = [workloads.normal_bf16((300, 648), 1.0, 911, 1e-3, 50.0), workloads.normal_bf16((256, 1024), 0.01, 912)]
dev = [x.cuda() for x in xs]
qs = [torch.empty(x.shape, dtype=torch.uint8, device="cuda") for x in xs]
ss = [torch.empty((1,), dtype=torch.float32, device="cuda") for x in xs]
# an empty call first: loads the library's device code and looks up its fixed array, the
# one-time costs of any first call (module memory, not an allocation by the entry point)
assert L.fp8q_quantize_tensor_noalloc(P(dev[0]), 0, 648, 648, P(qs[0]), P(ss[0]), stream) == 0
torch.cuda.synchronize()
assert float(ss[0].item()) == 1.0
free0 = torch.cuda.mem_get_info()[0]
for x, q, s in zip(dev, qs, ss):
    assert L.fp8q_quantize_tensor_noalloc(P(x), x.shape[0], x.shape[1], x.stride(0), P(q), P(s), stream) == 0
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
same = []
for x, q, s in zip(xs, qs, ss):
    oq, os_ = Q.quantize_tensor(workloads.bf16_bits(x))
    same.append(bool(np.array_equal(q.cpu().numpy(), oq))
                and int(s.cpu().numpy().view(np.uint32)[0]) == int(np.float32(os_).view(np.uint32)))
# the allocating entry point, for contrast: its first call creates the library's scratch pool
q2 = torch.empty(dev[0].shape, dtype=torch.uint8, device="cuda")
s2 = torch.empty((1,), dtype=torch.float32, device="cuda")
assert L.fp8q_quantize_tensor(P(dev[0]), 300, 648, 648, P(q2), P(s2), stream) == 0
torch.cuda.synchronize()
free2 = torch.cuda.mem_get_info()[0]
print(json.dumps({"free0": free0, "free1": free1, "free2": free2, "oracle_equal": same}))
'''


def test_noalloc_first_calls_in_a_fresh_process_allocate_nothing_and_match_the_oracle(cuda_lib):
    """In a process where it is the only fp8q entry point called, two calls leave the
    device's free memory unchanged (the library's scratch pool is never created), and its
    codes and decode scales equal the oracle's.  The allocating entry point called
    afterwards in the same process shows that the measurement sees the pool's allocation."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, FP8Q_ROOT=root, CUDA_MODULE_LOADING="EAGER")
    r = subprocess.run([sys.executable, "-c", _FRESH], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["oracle_equal"] == [True, True]
    assert d["free1"] == d["free0"], d                 # nothing allocated by the two calls
    assert d["free2"] < d["free1"], d                  # the pool allocation is visible to the check
