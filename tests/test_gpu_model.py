"""Whole-decoder GPU tests through bi_decode_step.

Bitwise (0 ULP) invariance of the GPU path with itself across batch size,
batch composition, prefill chunking and prefill vs decode; parity with the
fp64 oracle, teacher-forced on the GPU's own tokens: |logprob - oracle|
<= 2e-2 on the bf16 path (oracle in bf16-storage emulation), relative 1e-5 in
LayerCast mode and in the FP32-storage mode (mode 2; exact fp64 oracle);
greedy tokens equal the oracle's wherever the oracle's top-2 margin exceeds
0.05.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import configs

pytestmark = pytest.mark.gpu

N_STEPS = 16


@pytest.fixture(scope="module")
def pkg():
    from invariant_deterministic_full_b200 import model, ops
    assert torch.cuda.is_available()
    ops.device_error(reset=True)
    return model, ops


@pytest.fixture(scope="module")
def tiny_w():
    return synth.model_weights(configs.TINY)


def _prompts(n, length, vocab):
    return [synth.prompt_tokens(r, length, vocab) for r in range(n)]


def _run_bs(pkg, w, mode, bs, chunk=None, n_steps=N_STEPS):
    model, ops = pkg
    m = model.Model(configs.TINY, mode=mode, n_slots=8, capacity=256, host_weights=w)
    seqs, rec = model.greedy_generate(m, _prompts(bs, 64, configs.TINY["vocab"]), n_steps, chunk=chunk)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    m.close()
    return seqs, rec


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_tiny_bitwise_across_batch_sizes_and_chunking(pkg, tiny_w, mode):
    ref_seqs, ref = _run_bs(pkg, tiny_w, mode, 8)
    for bs, chunk in ((1, None), (3, 16), (8, 7)):
        seqs, rec = _run_bs(pkg, tiny_w, mode, bs, chunk=chunk)
        for b in range(bs):
            assert seqs[b] == ref_seqs[b]
            for k in ("logprob", "lse", "argmax", "margin", "recomputed"):
                assert np.array_equal(rec[k][b], ref[k][b]), (bs, b, k)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_tiny_decode_equals_teacher_forced_prefill(pkg, tiny_w, mode):
    model, ops = pkg
    seqs, rec = _run_bs(pkg, tiny_w, mode, 3)
    m = model.Model(configs.TINY, mode=mode, n_slots=8, capacity=256, host_weights=tiny_w)
    for b in range(3):
        s = np.array(seqs[b], dtype=np.int32)
        n = len(s) - 1
        for chunk in (None, 32, 5):
            o = model.prefill(m, 5, s[:n], chunk=chunk, targets=s[1:n + 1])
            # decode step j ran at position 64 + j with target = the token it chose
            dec = o["logprob"][64:64 + N_STEPS]
            assert np.array_equal(dec, rec["logprob"][b]), (b, chunk)
            assert np.array_equal(o["lse"][64:], rec["lse"][b])
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    m.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_tiny_oracle_parity_teacher_forced(pkg, tiny_w, mode):
    model, ops = pkg
    seqs, rec = _run_bs(pkg, tiny_w, mode, 3)
    m = model.Model(configs.TINY, mode=mode, n_slots=8, capacity=256, host_weights=tiny_w)
    omode = oracle.OR_BF16 if mode == 0 else oracle.OR_EXACT
    for b in range(3):
        s = np.array(seqs[b], dtype=np.int32)
        n = len(s) - 1
        o = model.prefill(m, 6, s[:n], targets=s[1:n + 1])
        res, _ = oracle.forward(configs.TINY, tiny_w, s[:n], s[1:n + 1], mode=omode)
        lp = o["logprob"].astype(np.float64)
        if mode == 0:
            assert np.abs(lp - res[:, 1]).max() <= 2e-2
        else:
            assert (np.abs(lp - res[:, 1]) <= 1e-5 * np.abs(res[:, 1])).all(), np.abs(lp - res[:, 1]).max()
        # greedy choices agree with the oracle wherever its margin is clear
        res_g, _ = oracle.forward(configs.TINY, tiny_w, s[:n], None, mode=omode)
        gen = np.arange(63, n)
        clear = res_g[gen, 3] > 0.05
        assert (s[gen + 1][clear] == res_g[gen, 2][clear].astype(np.int32)).all()
    m.close()


def test_tiny_recompute_flag_semantics(pkg, tiny_w):
    """bf16 path: recomputed == (own bf16 margin < 0.1); the margin matches the oracle's bf16-path margin."""
    model, ops = pkg
    seqs, rec = _run_bs(pkg, tiny_w, 0, 3)
    assert np.array_equal(rec["recomputed"], (rec["margin"] < 0.1).astype(np.uint8))
    m = model.Model(configs.TINY, mode=0, n_slots=8, capacity=256, host_weights=tiny_w)
    s = np.array(seqs[0], dtype=np.int32)
    n = len(s) - 1
    o = model.prefill(m, 6, s[:n], targets=s[1:n + 1])
    res, _ = oracle.forward(configs.TINY, tiny_w, s[:n], s[1:n + 1], mode=oracle.OR_BF16)
    assert np.abs(o["margin"] - res[:, 3]).max() <= 2e-2
    m.close()


@pytest.mark.parametrize("mode", [0, 1])
def test_llama8b_shape_batches_512_token_prompts_bitwise(pkg, mode):
    """The 8B-shaped random-init model, bf16 and LayerCast: 32 prompts of 512 random ids (attention spans three
    256-key chunks), 16 greedy decode steps.  Every sequence's tokens, logprobs, lse, margins and recompute flags
    are bitwise the same decoded at batch 32, 16, 8, 4 and 1 (prompts prefilled in different chunkings), and equal
    to a teacher-forced chunked prefill of the finished sequence."""
    model, ops = pkg
    cfg = configs.LLAMA8B
    V = cfg["vocab"]
    m = model.Model(cfg, mode=mode, n_slots=32, capacity=544, init="device")
    prompts = _prompts(32, 512, V)
    seqs32, rec32 = model.greedy_generate(m, prompts, N_STEPS)
    for B, off, chunk in ((16, 16, 300), (8, 3, None), (4, 27, 128), (1, 11, 97)):
        seqs, rec = model.greedy_generate(m, prompts[off:off + B], N_STEPS, chunk=chunk)
        for b in range(B):
            assert seqs[b] == seqs32[off + b], (B, b)
            for k in ("logprob", "lse", "argmax", "margin", "recomputed"):
                assert np.array_equal(rec[k][b], rec32[k][off + b]), (B, b, k)
    s = np.array(seqs32[9], dtype=np.int32)
    o = model.prefill(m, 0, s[:-1], chunk=200, targets=s[1:])
    # decode step j ran at position 512 + j; the prefill row for that position has the same target
    assert np.array_equal(o["logprob"][512:], rec32["logprob"][9])
    assert np.array_equal(o["lse"][512:], rec32["lse"][9])
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    m.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_llama8b_width_two_layers_oracle_parity(pkg, mode):
    """Every matrix at the 8B shape (hidden 4096, 32/8 heads x 128, FFN 14336, vocab 128256), 2 layers,
    so the fp64 oracle can run the whole forward: teacher-forced parity on the GPU's tokens."""
    model, ops = pkg
    cfg = configs.shrink(configs.LLAMA8B, n_layers=2)
    w = synth.model_weights(cfg)
    m = model.Model(cfg, mode=mode, n_slots=2, capacity=64, host_weights=w)
    seqs, rec = model.greedy_generate(m, _prompts(1, 5, cfg["vocab"]), 2)
    s = np.array(seqs[0], dtype=np.int32)
    n = len(s) - 1
    o = model.prefill(m, 1, s[:n], targets=s[1:n + 1])
    res, _ = oracle.forward(cfg, w, s[:n], s[1:n + 1], mode=oracle.OR_BF16 if mode == 0 else oracle.OR_EXACT)
    lp = o["logprob"].astype(np.float64)
    if mode == 0:
        assert np.abs(lp - res[:, 1]).max() <= 2e-2
    else:
        assert (np.abs(lp - res[:, 1]) <= 1e-5 * np.abs(res[:, 1])).all(), np.abs(lp - res[:, 1]).max()
    assert np.array_equal(o["logprob"][5:], rec["logprob"][0])
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    m.close()
