"""Divergence study through bi_decode_step on the tiny config (GPU): the invariant path gives the same greedy
tokens for every prompt alone and batched; LayerCast keeps the bf16 weights and doubles the KV bytes; the study's
rates are well formed."""
import pytest

from synth import configs

pytestmark = pytest.mark.gpu


def test_divergence_study_tiny():
    import torch
    assert torch.cuda.is_available()
    from invariant_deterministic_full_b200 import divergence as dv, ops
    ops.device_error(reset=True)
    r = dv.study(configs.TINY, n_prompts=6, prompt_len=16, n_steps=24)
    assert r["batch_alone_vs_batched"]["invariant"]["exact_agreement"] == 1.0
    m = r["memory"]
    P = dv.param_count(configs.TINY)
    assert m["allocated_weights_bf16"] == m["allocated_weights_layercast"] == 2 * P
    assert m["allocated_kv_layercast"] == 2 * m["allocated_kv_bf16"]
    v = r["vs_layercast"]
    for k in ("bf16_no_recompute", "bf16_selective_recompute"):
        c = v[k]
        assert 0.0 <= c["exact_agreement"] <= 1.0 and c["exact_agreement"] + c["diverged"] == pytest.approx(1.0)
    assert 0.0 <= v["recompute_rate"] <= 1.0
    assert ops.device_error() == 0
