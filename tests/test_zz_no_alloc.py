"""bi_lmhead_logprob_noalloc: the LM-head logprob for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

It must give the same results as bi_lmhead_logprob called with a caller
workspace, on two calls in a row (the second call must not see anything left
over from the first), and reject row counts whose scratch would not fit.
This file is collected last so a stop-at-first-failure run has already run
every other test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _call_noalloc(L, h, W, target, thresh, mode, want_logits):
    B, H = h.shape
    V = W.shape[0]
    dev = h.device
    out = dict(logprob=torch.full((B,), float("nan"), device=dev), lse=torch.full((B,), float("nan"), device=dev),
               argmax=torch.full((B,), -7, dtype=torch.int32, device=dev),
               margin=torch.full((B,), float("nan"), device=dev),
               recomputed=torch.full((B,), 9, dtype=torch.uint8, device=dev))
    logits = torch.empty(B, V, dtype=torch.float32, device=dev) if want_logits else None
    p = lambda t: ctypes.c_void_p(0 if t is None else t.data_ptr())
    rc = L.lib.bi_lmhead_logprob_noalloc(p(h), p(W), p(target), B, H, V, thresh, mode, p(out["logprob"]),
                                         p(out["lse"]), p(out["argmax"]), p(out["margin"]), p(out["recomputed"]),
                                         p(logits), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if want_logits:
        out["logits"] = logits
    return rc, out


@pytest.mark.parametrize("mode", [0, 1])
def test_noalloc_matches_workspace_entry_point_twice(mode):
    from invariant_deterministic_full_b200 import _lib as L, ops
    assert torch.cuda.is_available()
    H, V = 4096, 128256
    W = torch.empty(V, H, dtype=torch.bfloat16, device="cuda")
    ops.synth_fill_bf16(W, V, H, synth.key(synth.WEIGHT_SEED, synth.S_LMHEAD), 0.02)
    rng = np.random.default_rng(mode)
    for call, (B, seed, want_logits) in enumerate([(24, 7, False), (9, 8, True)]):
        h = torch.from_numpy(synth.hidden_states(seed, B, H)).cuda()
        tgt = torch.from_numpy(rng.integers(-1, V, size=B).astype(np.int32)).cuda()
        ref = ops.lmhead_logprob(h, W, tgt, threshold=0.1, mode=mode, want_logits=want_logits)
        rc, got = _call_noalloc(L, h, W, tgt, 0.1, mode, want_logits)
        assert rc == L.BI_OK, L.lib.bi_last_error()
        torch.cuda.synchronize()
        for k in ref:
            assert torch.equal(got[k], ref[k]), (call, k)
        if mode == 0:
            assert 0 < int(got["recomputed"].sum()) < B  # the recompute path ran in the scratch too
    assert ops.device_error() == 0


def test_noalloc_rejects_rows_beyond_the_fixed_scratch():
    from invariant_deterministic_full_b200 import _lib as L
    H, V, B = 4096, 128256, 64
    need = L.lib.bi_lmhead_workspace_size(B, H, V, 0)
    assert need > (80 << 20)
    fake = ctypes.c_void_p(1 << 20)  # rejected before any pointer is used
    rc = L.lib.bi_lmhead_logprob_noalloc(fake, fake, None, B, H, V, 0.1, 0, fake, fake, fake, fake, fake, None, None)
    assert rc == L.BI_ERR_WORKSPACE
    assert b"scratch" in L.lib.bi_last_error()
