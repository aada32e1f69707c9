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


def _oracle_greedy(cfg, w, prompt, n_steps, mode):
    """The oracle's own greedy run: the prompt, then one token at a time after the stored keys/values.
    Returns the generated tokens and the oracle's top-2 margin at each choice."""
    import numpy as np
    import oracle
    res, _, (k, v) = oracle.forward_ctx(cfg, w, prompt, mode=mode, want_kv=True)
    toks, margins = [int(res[-1, 2])], [float(res[-1, 3])]
    for _ in range(n_steps):
        res, _, (k1, v1) = oracle.forward_ctx(cfg, w, np.array(toks[-1:], np.int32), k, v, mode=mode, want_kv=True)
        k, v = np.concatenate([k, k1], axis=1), np.concatenate([v, v1], axis=1)
        toks.append(int(res[-1, 2]))
        margins.append(float(res[-1, 3]))
    return toks, margins


def test_divergence_index_matches_the_oracles_greedy_runs():
    """The study's bf16-vs-LayerCast divergence on the tiny config against the oracle's own greedy runs in
    bf16-storage emulation and in exact fp64.  A greedy choice is decided where the oracle's top-2 margin is clear
    of the path's logit error: > 0.05 for bf16 (the parity bound), > 1e-3 for LayerCast (1e-5 relative).  On each
    prompt's decided stretch the GPU's bf16 tokens are the oracle's bf16 tokens and its LayerCast tokens the exact
    oracle's; a bf16/exact divergence sits at a near-tie by nature, so the GPU's divergence index is never before
    the end of the stretch, and prompts whose whole run is decided and agrees give no divergence on the GPU either.
    The LM head is drawn with std 0.25 so that most margins are clear."""
    import torch
    import synth
    from invariant_deterministic_full_b200 import divergence as dv, model as mdl, ops
    from invariant_deterministic_full_b200._lib import MODE_BF16, MODE_LAYERCAST
    import oracle
    assert torch.cuda.is_available()
    cfg = configs.TINY
    V, H = cfg["vocab"], cfg["hidden"]
    w = synth.model_weights(cfg)
    w["lm_head"] = synth.normal_bf16(synth.key(synth.WEIGHT_SEED, synth.S_LMHEAD), V * H, 0.25).reshape(V, H)
    prompts = [synth.prompt_tokens(2000 + r, 16, V) for r in range(24)]
    n_steps = 24

    def gpu_run(mode):
        m = mdl.Model(cfg, mode=mode, n_slots=len(prompts), capacity=64, margin_threshold=0.0, host_weights=w)
        seqs, _ = mdl.greedy_generate(m, prompts, n_steps)
        m.close()
        return [s[16:] for s in seqs]

    g_bf, g_lc = gpu_run(MODE_BF16), gpu_run(MODE_LAYERCAST)
    decided, whole = 0, 0
    for p, gb, gl in zip(prompts, g_bf, g_lc):
        ob, mb = _oracle_greedy(cfg, w, p, n_steps, oracle.OR_BF16)
        oe, me = _oracle_greedy(cfg, w, p, n_steps, oracle.OR_EXACT)
        nb = next((i for i, m in enumerate(mb) if m <= 0.05), len(mb))  # bf16 choices decided before nb
        ne = next((i for i, m in enumerate(me) if m <= 1e-3), len(me))  # exact choices decided before ne
        assert gb[:nb] == ob[:nb] and gl[:ne] == oe[:ne]
        n = min(nb, ne)
        i_or, i_gpu = dv.divergence_index(ob, oe), dv.divergence_index(gb, gl)
        assert (i_or is None or i_or >= n) and (i_gpu is None or i_gpu >= n)
        if n == len(ob) and i_or is None:
            assert i_gpu is None
            whole += 1
        decided += n
    assert decided >= 150 and whole >= 3, (decided, whole)
    assert ops.device_error() == 0
