"""Invariant tensor parallelism on one GPU (the tp ranks run one after another; the all-gather is a
concatenation): every projection split by output rows over the full K, no reduce-scatter.  A token's logprob, lse,
argmax, margin and recompute flag, and every KV-cache row, must be bitwise those of bi_decode_step at tp = 1
("Meituan bitwise train/infer consistency", key practices, the TP item)."""
import numpy as np
import pytest
import torch

import synth
from synth import configs

pytestmark = pytest.mark.gpu

KEYS = ("logprob", "lse", "argmax", "margin", "recomputed")


def _check(o_ref, o_tp, what):
    for k in KEYS:
        assert torch.equal(o_ref[k], o_tp[k]), (what, k)


def _run(cfg, tps, prompt_len=20, steps=3):
    from invariant_deterministic_full_b200 import model as mdl, ops
    from invariant_deterministic_full_b200.tp import TPModel
    assert torch.cuda.is_available()
    m = mdl.Model(cfg, n_slots=2, capacity=64, init="device")
    V = cfg["vocab"]
    prompts = [synth.prompt_tokens(40 + b, prompt_len - 3 * b, V) for b in range(2)]
    # reference: bi_decode_step (tp = 1): both prompts as one prefill batch, then greedy decode of both
    ids = np.concatenate(prompts)
    slots = np.concatenate([[b] * len(p) for b, p in enumerate(prompts)])
    pos = np.concatenate([np.arange(len(p)) for p in prompts])
    ref = [m.step(ids, slots, pos)]
    nxt = [int(ref[0]["argmax"][len(prompts[0]) - 1]), int(ref[0]["argmax"][-1])]
    seq = [(ids, slots, pos)]
    cur = [len(p) for p in prompts]
    for _ in range(steps):
        step = (np.array(nxt), np.array([0, 1]), np.array(cur))
        o = m.step(*step)
        ref.append(o)
        seq.append(step)
        nxt = [int(v) for v in o["argmax"].cpu()]
        cur = [c + 1 for c in cur]
    torch.cuda.synchronize()
    for tp in tps:
        t = TPModel(m, tp)
        for i, (a, b, c) in enumerate(seq):
            _check(ref[i], t.step(a, b, c), (tp, i))
        # the ranks' caches hold the reference cache's kv heads, split in rank order
        hk = cfg["n_kv_heads"] // tp
        for r in range(tp):
            kv = t.w[r]["kv"]
            assert torch.equal(kv.k, m.kv.k[:, :, r * hk:(r + 1) * hk]), (tp, r, "k")
            assert torch.equal(kv.v, m.kv.v[:, :, r * hk:(r + 1) * hk]), (tp, r, "v")
        del t
    torch.cuda.synchronize()
    assert ops.device_error(reset=True) == 0
    m.close()


def test_tp_tiny_bitwise_equals_decode_step():
    _run(configs.TINY, (2, 4))


def test_tp_llama8b_width_two_layers_bitwise_equals_decode_step():
    _run(configs.shrink(configs.LLAMA8B, n_layers=2), (2, 4, 8))
