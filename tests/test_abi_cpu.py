"""The C-ABI library loads, exports every symbol include/bi.h declares, and
rejects invalid arguments on the host with status codes (no GPU needed: every
case here fails validation before any CUDA call).

The validation cases pass placeholder device addresses that are never meant to
be dereferenced.  They run only where the library's own CUDA runtime sees no
device (the `host_only` fixture asks the library, not torch), so a broken check
can never turn into a launch on a real GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__._lib_builder().build()
    from invariant_deterministic_full_b200 import _lib
    return _lib


@pytest.fixture
def host_only(L):
    if L.lib.bi_num_sms(0) > 0:
        pytest.skip("placeholder device addresses are only passed where the library sees no CUDA device")
    return L


def _declared():
    src = open(os.path.join(ROOT, "include", "bi.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bi_[a-z0-9_]+)\s*\(", src)))


def test_header_symbols_exported(L):
    names = _declared()
    assert len(names) >= 19
    so = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(so, n), f"{n} declared in bi.h but not exported"
    assert set(names) == set(L.SIGNATURES), "binding and header disagree"


def test_version_and_status_codes(L):
    assert L.lib.bi_version() == 1
    assert (L.BI_ERR_INVALID_ARG, L.BI_ERR_UNSUPPORTED, L.BI_ERR_WORKSPACE, L.BI_ERR_CAPACITY, L.BI_ERR_CUDA) == \
        (1, 2, 3, 4, 5)


def test_gemm_validation(host_only):
    L = host_only
    lib = L.lib
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    assert lib.bi_gemm(None, 64, fake, fake, 64, 0, 4, 64, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_gemm(fake, 96, fake, fake, 64, 0, 4, 64, 96, 0, 0, None, 0, 0, None, 0, None) == L.BI_ERR_UNSUPPORTED
    assert b"K % 64" in lib.bi_last_error()
    assert lib.bi_gemm(fake, 64, fake, fake, 64, 0, 4, 96, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_ERR_UNSUPPORTED
    assert lib.bi_gemm(fake, 60, fake, fake, 64, 0, 4, 64, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_ERR_UNSUPPORTED
    assert lib.bi_gemm(fake, 64, fake, fake, 16, 0, 4, 64, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_gemm(fake, 64, fake, fake, 64, 0, 4, 64, 64, 0, 7, None, 0, 0, None, 0, None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_gemm(fake, 64, ctypes.c_void_p((1 << 20) + 2), fake, 64, 0, 4, 64, 64, 0, 0, None, 0, 0, None, 0,
                       None) == L.BI_ERR_UNSUPPORTED
    assert lib.bi_gemm(fake, 64, fake, fake, 64, 0, 0, 64, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_OK  # M = 0: no work
    assert lib.bi_gemm(None, 64, fake, None, 64, 0, 0, 64, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_OK  # empty x, y
    assert lib.bi_gemm(None, 64, None, None, 64, 0, 0, 64, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_gemm(fake, 64, fake, None, 64, 0, 4, 64, 64, 0, 0, None, 0, 0, None, 0, None) == L.BI_ERR_INVALID_ARG
    # RoPE + KV-append epilogue: its arguments are required, checked against the cache, and bf16 invariant only
    kv = L.KvLayout(1 << 20, 1 << 20, 2, 1, 2, 64, 64, 0)
    ea = L.EpiArgs(1 << 20, 64, 1 << 20, ctypes.pointer(kv), 0, 1 << 20, 1 << 20, 4)  # N = (4 + 2*2) * 64 = 512
    R = L.EPI_ROPE_KV_APPEND
    assert lib.bi_gemm(fake, 64, fake, None, 0, 0, 4, 512, 64, 0, R, None, 0, 0, None, 0, None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_gemm(fake, 64, fake, fake, 512, 0, 4, 512, 64, 0, 0, ctypes.byref(ea), 0, 0, None, 0, None) == \
        L.BI_ERR_INVALID_ARG  # arguments given for an epilogue that takes none
    assert lib.bi_gemm(fake, 64, fake, None, 0, 0, 4, 512, 64, 0, R, ctypes.byref(ea), 1, 0, None, 0, None) == \
        L.BI_ERR_UNSUPPORTED  # LayerCast
    assert lib.bi_gemm(fake, 64, fake, None, 0, 0, 4, 512, 64, 0, R, ctypes.byref(ea), 0, 1, None, 0, None) == \
        L.BI_ERR_UNSUPPORTED  # FAST variant
    assert lib.bi_gemm(fake, 64, fake, None, 0, 0, 4, 576, 64, 0, R, ctypes.byref(ea), 0, 0, None, 0, None) == \
        L.BI_ERR_INVALID_ARG  # N is not (Hq + 2 Hkv) * head_dim
    ea.layer = 1
    assert lib.bi_gemm(fake, 64, fake, None, 0, 0, 4, 512, 64, 0, R, ctypes.byref(ea), 0, 0, None, 0, None) == \
        L.BI_ERR_INVALID_ARG  # layer beyond the cache
    ea.layer = 0
    assert lib.bi_gemm(fake, 64, fake, None, 0, 0, 0, 512, 64, 0, R, ctypes.byref(ea), 0, 0, None, 0, None) == L.BI_OK
    # n_full names the whole matrix a row shard belongs to: at least N rows, a multiple of 64
    assert lib.bi_gemm(fake, 64, fake, fake, 64, 0, 4, 128, 64, 64, 0, None, 0, 0, None, 0, None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_gemm(fake, 64, fake, fake, 64, 0, 4, 128, 64, 200, 0, None, 0, 0, None, 0, None) == \
        L.BI_ERR_INVALID_ARG
    assert lib.bi_gemm_workspace_size(4, 64, 64, 0, 0) == 0


def test_rmsnorm_lmhead_validation(host_only):
    L = host_only
    lib = L.lib
    fake = ctypes.c_void_p(1 << 20)
    assert lib.bi_rmsnorm(None, None, None, fake, fake, None, 2, 64, 1e-5, 0, None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_rmsnorm(fake, None, None, fake, fake, None, 2, 60, 1e-5, 0, None) == L.BI_ERR_UNSUPPORTED
    assert lib.bi_rmsnorm(fake, None, None, fake, fake, None, 2, 32768, 1e-5, 0, None) == L.BI_ERR_UNSUPPORTED
    args = [fake] * 6
    assert lib.bi_lmhead_logprob(None, fake, None, 2, 64, 128, 0.1, 0, *args[:5], None, fake, 1 << 30,
                                 None) == L.BI_ERR_INVALID_ARG
    assert lib.bi_lmhead_logprob(fake, fake, None, 2, 64, 100, 0.1, 0, *args[:5], None, fake, 1 << 30,
                                 None) == L.BI_ERR_UNSUPPORTED
    need = lib.bi_lmhead_workspace_size(2, 64, 128, 0)
    assert need > 0
    assert lib.bi_lmhead_logprob(fake, fake, None, 2, 64, 128, 0.1, 0, *args[:5], None, fake, need - 512,
                                 None) == L.BI_ERR_WORKSPACE


def _tiny_ctx(L, capacity=64, mode=0):
    fake = 1 << 20
    desc = L.ModelDesc(1, 256, 4, 4, 64, 1024, 4096, 1e-5, mode, 0, 0.1)
    w = L.Weights(*([fake] * 10), capacity)
    kv = L.KvLayout(fake, fake, 2, 1, 4, capacity, 64, 1 if mode else 0)
    ctx = ctypes.c_void_p()
    rc = L.lib.bi_ctx_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(ctx))
    return rc, ctx, kv


def test_ctx_validation(host_only):
    L = host_only
    lib = L.lib
    rc, ctx, kv = _tiny_ctx(L)
    assert rc == L.BI_OK and ctx.value
    assert lib.bi_decode_workspace_size(ctx, 8, 8, 63) > 0
    # KV dtype must follow the mode
    desc = L.ModelDesc(1, 256, 4, 4, 64, 1024, 4096, 1e-5, 1, 0, 0.1)
    w = L.Weights(*([1 << 20] * 10), 64)
    c2 = ctypes.c_void_p()
    assert lib.bi_ctx_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(c2)) == \
        L.BI_ERR_INVALID_ARG
    bad = L.ModelDesc(1, 250, 4, 4, 64, 1024, 4096, 1e-5, 0, 0, 0.1)
    assert lib.bi_ctx_create(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(c2)) == \
        L.BI_ERR_UNSUPPORTED
    bad = L.ModelDesc(1, 4096, 64, 1, 64, 1024, 4096, 1e-5, 0, 0, 0.1)  # 64 q heads on one kv head
    kv1 = L.KvLayout(1 << 20, 1 << 20, 2, 1, 1, 64, 64, 0)
    assert lib.bi_ctx_create(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(kv1), ctypes.byref(c2)) == \
        L.BI_ERR_UNSUPPORTED
    bad = L.ModelDesc(1, 256, 6, 4, 64, 1024, 4096, 1e-5, 0, 0, 0.1)
    assert lib.bi_ctx_create(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(c2)) == \
        L.BI_ERR_INVALID_ARG
    lib.bi_ctx_destroy(ctx)


def test_decode_step_capacity_and_workspace_rejected_on_host(host_only):
    L = host_only
    lib = L.lib
    rc, ctx, _ = _tiny_ctx(L, capacity=64)
    assert rc == L.BI_OK
    slot = np.zeros(3, dtype=np.int32)
    pos = np.array([10, 11, 64], dtype=np.int32)  # 64 == capacity
    fake = 1 << 20
    b = L.Batch(3, fake, fake, fake, slot.ctypes.data, pos.ctypes.data, fake, 3, 0)
    o = L.StepOut(fake, fake, fake, fake, fake, 0, 0)
    assert lib.bi_decode_step(ctx, ctypes.byref(b), ctypes.byref(o), ctypes.c_void_p(fake), 1 << 40, None) == \
        L.BI_ERR_CAPACITY
    assert b"capacity" in lib.bi_last_error()
    pos[2] = 12
    need = lib.bi_decode_workspace_size(ctx, 3, 3, 12)
    assert lib.bi_decode_step(ctx, ctypes.byref(b), ctypes.byref(o), ctypes.c_void_p(fake), need - 1024, None) == \
        L.BI_ERR_WORKSPACE
    b.n_lm = 4  # more output rows than tokens
    assert lib.bi_decode_step(ctx, ctypes.byref(b), ctypes.byref(o), ctypes.c_void_p(fake), need, None) == \
        L.BI_ERR_INVALID_ARG
    # a slot outside the cache is rejected before anything is launched (here a launch would fail with BI_ERR_CUDA)
    b.n_lm = 3
    slot[1] = 2  # the tiny context has 2 slots
    c0 = lib.bi_launch_count()
    assert lib.bi_decode_step(ctx, ctypes.byref(b), ctypes.byref(o), ctypes.c_void_p(fake), need, None) == \
        L.BI_ERR_INVALID_ARG
    assert b"slot" in lib.bi_last_error()
    assert lib.bi_launch_count() == c0
    lib.bi_ctx_destroy(ctx)


def test_attention_validation(host_only):
    L = host_only
    lib = L.lib
    fake = 1 << 20
    kv = L.KvLayout(fake, fake, 2, 1, 4, 64, 64, 0)
    slot = np.array([0, 2], dtype=np.int32)
    pos = np.array([0, 1], dtype=np.int32)
    args = lambda s, p: (ctypes.c_void_p(fake), ctypes.byref(kv), 0, ctypes.c_void_p(fake), ctypes.c_void_p(fake),
                         s.ctypes.data, p.ctypes.data, ctypes.c_void_p(fake), 2, 4, 0.125, 0, 0,
                         ctypes.c_void_p(fake), 1 << 30, None)
    assert lib.bi_attention(*args(slot, pos)) == L.BI_ERR_INVALID_ARG  # slot 2 of 2
    slot[1] = 1
    pos[1] = 70
    assert lib.bi_attention(*args(slot, pos)) == L.BI_ERR_CAPACITY
    kv.head_dim = 96
    pos[1] = 1
    assert lib.bi_attention(*args(slot, pos)) == L.BI_ERR_UNSUPPORTED


def test_failing_cuda_call_maps_to_bi_err_cuda(host_only):
    # With no device visible to the library's runtime, the launch fails on the host (no CUDA device), which must
    # come back as BI_ERR_CUDA with a message; nothing reaches a GPU.
    L = host_only
    fake = ctypes.c_void_p(1 << 20)
    assert L.lib.bi_rmsnorm(fake, None, None, fake, fake, None, 2, 64, 1e-5, 0, None) == L.BI_ERR_CUDA
    assert L.lib.bi_last_error()
