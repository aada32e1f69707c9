"""Bounds and repeatability (GPU; compute-sanitizer is not available, so writes are checked with guard regions).

Outputs live inside larger buffers poisoned with NaN (or a byte pattern for integer outputs); after the call the
guard rows, columns and the bytes past the workspace size must be untouched and the written region finite.  The
tiny model's greedy decode is also run in two separate processes, which must agree bit for bit."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def api():
    assert torch.cuda.is_available()
    from invariant_deterministic_full_b200 import ops
    from invariant_deterministic_full_b200._lib import lib, check
    ops.device_error(reset=True)
    return ops, lib, check


def _nan(*shape, dtype=torch.float32):
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


@pytest.mark.parametrize("mode", [0, 1])
def test_gemm_writes_only_its_rows_columns_and_workspace(api, mode):
    ops, lib, check = api
    M, N, K, pad = 37, 192, 256, 64
    g = torch.Generator().manual_seed(5)
    x = torch.randn(M, K, generator=g)
    x = (x.to(torch.bfloat16) if mode == 0 else x).cuda()
    w = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16).cuda()
    ybuf = _nan(M + 2, N + pad)
    y = ybuf[1:M + 1]
    wsb = lib.bi_gemm_workspace_size(M, N, K, mode, 0)
    ws = torch.full((wsb + 4096,), 0xFF, dtype=torch.uint8, device="cuda")
    check(lib.bi_gemm(x.data_ptr(), K, w.data_ptr(), y.data_ptr(), N + pad, 1, M, N, K, 0, 0, None, mode, 0, ws.data_ptr(),
                      wsb, ops._stream()), "bi_gemm")
    torch.cuda.synchronize()
    assert torch.isnan(ybuf[0]).all() and torch.isnan(ybuf[M + 1]).all()
    assert torch.isnan(ybuf[1:M + 1, N:]).all()
    assert torch.isfinite(ybuf[1:M + 1, :N]).all()
    assert bool((ws[wsb:] == 0xFF).all())
    assert ops.device_error() == 0


def test_rmsnorm_writes_only_its_rows(api):
    ops, lib, check = api
    M, H = 5, 4096
    g = torch.Generator().manual_seed(6)
    x = torch.randn(M, H, generator=g).to(torch.bfloat16).cuda()
    r = torch.randn(M, H, generator=g).to(torch.bfloat16).cuda()
    gamma = torch.ones(H, dtype=torch.bfloat16, device="cuda")
    ybuf, rbuf, y32buf = _nan(M + 2, H, dtype=torch.bfloat16), _nan(M + 2, H, dtype=torch.bfloat16), _nan(M + 2, H)
    check(lib.bi_rmsnorm(x.data_ptr(), r.data_ptr(), rbuf[1].data_ptr(), gamma.data_ptr(), ybuf[1].data_ptr(),
                         y32buf[1].data_ptr(), M, H, 1e-5, 0, ops._stream()), "bi_rmsnorm")
    torch.cuda.synchronize()
    for buf in (ybuf, rbuf, y32buf):
        assert torch.isnan(buf[0].float()).all() and torch.isnan(buf[M + 1].float()).all()
        assert torch.isfinite(buf[1:M + 1].float()).all()
    assert ops.device_error() == 0


@pytest.mark.parametrize("B", [3, 12])
def test_lmhead_writes_only_its_rows_and_workspace(api, B):
    ops, lib, check = api
    H, V = 512, 4096
    g = torch.Generator().manual_seed(7)
    h = torch.randn(B, H, generator=g)
    h = (h / h.pow(2).mean(dim=1, keepdim=True).sqrt()).cuda()
    W = (0.02 * torch.randn(V, H, generator=g)).to(torch.bfloat16).cuda()
    extra = 8
    lp, lse, mg = _nan(B + extra), _nan(B + extra), _nan(B + extra)
    am = torch.full((B + extra,), -7, dtype=torch.int32, device="cuda")
    rc = torch.full((B + extra,), 0xEE, dtype=torch.uint8, device="cuda")
    logits = _nan(B + 1, V)
    wsb = lib.bi_lmhead_workspace_size(B, H, V, 0)
    ws = torch.full((wsb + 4096,), 0xFF, dtype=torch.uint8, device="cuda")
    check(lib.bi_lmhead_logprob(h.data_ptr(), W.data_ptr(), None, B, H, V, 0.1, 0, lp.data_ptr(), lse.data_ptr(),
                                am.data_ptr(), mg.data_ptr(), rc.data_ptr(), logits.data_ptr(), ws.data_ptr(), wsb,
                                ops._stream()), "bi_lmhead_logprob")
    torch.cuda.synchronize()
    for t in (lp, lse, mg):
        assert torch.isnan(t[B:]).all() and torch.isfinite(t[:B]).all()
    assert bool((am[B:] == -7).all()) and bool(((am[:B] >= 0) & (am[:B] < V)).all())
    assert bool((rc[B:] == 0xEE).all()) and bool((rc[:B] <= 1).all())
    assert torch.isnan(logits[B]).all() and torch.isfinite(logits[:B]).all()
    assert bool((ws[wsb:] == 0xFF).all())
    assert ops.device_error() == 0


_RUN = """
import sys
import numpy as np
import synth
from synth import configs
from invariant_deterministic_full_b200 import model
m = model.Model(configs.TINY, mode=0, n_slots=3, capacity=64, init="host")
prompts = [synth.prompt_tokens(r, 16, configs.TINY["vocab"]) for r in range(3)]
seqs, rec = model.greedy_generate(m, prompts, 8)
np.save(sys.argv[1], np.concatenate([np.ascontiguousarray(rec["logprob"]).ravel().view(np.uint32),
                                     np.ascontiguousarray(rec["argmax"]).ravel().astype(np.uint32)]))
"""


def test_tiny_decode_bit_identical_across_processes(tmp_path):
    outs = []
    for i in range(2):
        p = tmp_path / f"run{i}.npy"
        r = subprocess.run([sys.executable, "-c", _RUN, str(p)], cwd=ROOT, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(np.load(p))
    assert outs[0].size == 2 * 3 * 8
    assert np.array_equal(outs[0], outs[1])
