"""Failure detection without a GPU fault: a bounded wait that nothing completes gives up after about a second,
reports itself through the device error word (timeout bit, site code), and leaves the context usable."""
import time

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports():
    from invariant_deterministic_full_b200 import ops
    assert torch.cuda.is_available()
    torch.cuda.synchronize()
    assert ops.device_error(reset=True) == 0
    t0 = time.monotonic()
    ops.selftest_wait_timeout()
    torch.cuda.synchronize()
    dt = time.monotonic() - t0
    v = ops.device_error(reset=True)
    assert v & 1, hex(v)              # wait timeout
    assert (v >> 8) == 0x31, hex(v)   # the self-test's site code
    assert 0.9 < dt < 30.0
    # the context is still usable: an invariant GEMM runs and matches a float64 product of the same bf16 values
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal((5, 128)).astype(np.float32)).cuda().to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((64, 128)).astype(np.float32)).cuda().to(torch.bfloat16)
    y = ops.gemm(x, w, out_dtype=torch.float32).cpu().double()
    ref = x.cpu().double() @ w.cpu().double().T
    assert torch.allclose(y, ref, rtol=1e-5, atol=1e-4)
    assert ops.device_error(reset=True) == 0
