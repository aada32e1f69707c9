"""Greedy-decoding divergence between numeric configurations, on a synthetic model.

Two of the pages measure how far greedy outputs drift when only the arithmetic
changes; this module takes the same measurements through bi_decode_step, on
random-init weights instead of the pages' benchmarks:

- "Give Me FP32 or Give Me Death? Challenges and Solutions for Reproducible
  Reasoning" (techwalker summary, section 7): the divergence index of two runs
  of one prompt is the first generated position at which they choose
  different tokens; a run pair that never differs agrees exactly.  Its
  LayerCast section (and the jiaxiangli summary, section 4) compares the
  memory of LayerCast with FP32 storage.
- "Greedy Decoding Is Not Precision-Invariant" (abstract): exact agreement with
  and without the selective FP32 LM-head recompute.

The reference run is LayerCast: the same bf16 weights with fp32 arithmetic,
activations and KV cache.  The FP32-storage arm (BI_MODE_FP32: the same weight
values held as f32, fp32 FMA everywhere) is run too, so LayerCast is compared
with what it replaces -- in agreement and in measured memory.  Batch invariance
is measured the same way: one configuration run on every prompt alone and on
all prompts in one batch, for the invariant path and for the non-invariant FAST
variant.
"""
import argparse
import json
import statistics

import numpy as np

import synth
from synth import configs

from ._lib import MODE_BF16, MODE_FP32, MODE_LAYERCAST, VARIANT_FAST, VARIANT_INVARIANT


def divergence_index(a, b):
    """First position at which token sequences a and b differ, or None when they agree exactly.
    A sequence that ends early differs at its end."""
    n = min(len(a), len(b))
    for i in range(n):
        if int(a[i]) != int(b[i]):
            return i
    return None if len(a) == len(b) else n


def compare(ref, runs):
    """Per-prompt divergence indices of runs against ref (lists of generated-token sequences) and their summary:
    exact-agreement rate, divergence rate, and the median and mean index over the prompts that diverge."""
    assert len(ref) == len(runs) and len(ref) > 0
    idx = [divergence_index(r, s) for r, s in zip(ref, runs)]
    div = [i for i in idx if i is not None]
    n = len(idx)
    return {"exact_agreement": (n - len(div)) / n, "diverged": len(div) / n,
            "median_index": statistics.median(div) if div else None,
            "mean_index": sum(div) / len(div) if div else None, "indices": idx}


def param_count(cfg):
    """Parameters of the decoder: embedding, per-layer q/k/v/o, gate/up/down and two norms, final norm, LM head."""
    L, H, Hq, Hkv, d, F, V = (cfg["n_layers"], cfg["hidden"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                              cfg["ffn"], cfg["vocab"])
    layer = (Hq + 2 * Hkv) * d * H + H * Hq * d + 3 * F * H + 2 * H
    return 2 * V * H + L * layer + H


def memory_bytes(cfg, kv_tokens, storage):
    """Weights plus KV cache for kv_tokens cached positions (summed over sequences).
    storage: 'bf16' (bf16 weights and KV), 'layercast' (bf16 weights, fp32 KV) or 'fp32' (fp32 weights and KV)."""
    w_b, kv_b = {"bf16": (2, 2), "layercast": (2, 4), "fp32": (4, 4)}[storage]
    per_pos = cfg["n_layers"] * cfg["n_kv_heads"] * cfg["head_dim"] * 2 * kv_b  # k and v of every layer
    return param_count(cfg) * w_b + kv_tokens * per_pos


def _generated(seqs, prompt_len):
    return [s[prompt_len:] for s in seqs]


def _run(model_mod, cfg, prompts, n_steps, mode, variant, threshold, alone, capacity):
    """Greedy tokens generated for every prompt (prompt excluded) by one configuration; all prompts in one batch,
    or every prompt alone (batch 1, slot 0).  Also the fraction of decode rows the LM head recomputed."""
    import torch
    n = len(prompts)
    m = model_mod.Model(cfg, mode=mode, variant=variant, n_slots=1 if alone else n, capacity=capacity,
                        margin_threshold=threshold, init="auto")
    try:
        if alone:
            gens, recs = [], []
            for p in prompts:
                s, r = model_mod.greedy_generate(m, [p], n_steps)
                gens.append(s[0][len(p):])
                recs.append(r["recomputed"])
            rec = float(np.mean(np.concatenate([x.ravel() for x in recs])))
        else:
            s, r = model_mod.greedy_generate(m, prompts, n_steps)
            gens = _generated(s, len(prompts[0]))
            rec = float(np.mean(r["recomputed"]))
        torch.cuda.synchronize()
        alloc = {k: int(v.numel() * v.element_size()) for k, v in m.w.items()}
        kv = int(sum(t.numel() * t.element_size() for t in (m.kv.k, m.kv.v)))
        return gens, rec, sum(alloc.values()), kv
    finally:
        m.close()
        del m
        torch.cuda.empty_cache()


def study(cfg, n_prompts=16, prompt_len=64, n_steps=64, threshold=0.1, seed0=2000):
    """Every comparison of the module on one config: precision (bf16 with and without the selective recompute
    against LayerCast) and batch composition (alone vs one batch, invariant path and FAST variant)."""
    from . import model as model_mod
    V = cfg["vocab"]
    prompts = [synth.prompt_tokens(seed0 + r, prompt_len, V) for r in range(n_prompts)]
    cap = prompt_len + n_steps + 1
    run = lambda **k: _run(model_mod, cfg, prompts, n_steps, capacity=cap, **k)
    ref, _, w_lc, kv_lc = run(mode=MODE_LAYERCAST, variant=VARIANT_INVARIANT, threshold=0.0, alone=False)
    fp, _, w_fp, kv_fp = run(mode=MODE_FP32, variant=VARIANT_INVARIANT, threshold=0.0, alone=False)
    b0, _, w_bf, kv_bf = run(mode=MODE_BF16, variant=VARIANT_INVARIANT, threshold=0.0, alone=False)
    b1, rate, _, _ = run(mode=MODE_BF16, variant=VARIANT_INVARIANT, threshold=threshold, alone=False)
    inv1, _, _, _ = run(mode=MODE_BF16, variant=VARIANT_INVARIANT, threshold=threshold, alone=True)
    f_n, _, _, _ = run(mode=MODE_BF16, variant=VARIANT_FAST, threshold=threshold, alone=False)
    f_1, _, _, _ = run(mode=MODE_BF16, variant=VARIANT_FAST, threshold=threshold, alone=True)
    strip = lambda c: {k: v for k, v in c.items() if k != "indices"}
    no_rc, rc = compare(ref, b0), compare(ref, b1)
    kv_tokens = n_prompts * cap
    lc, fpb = memory_bytes(cfg, kv_tokens, "layercast"), memory_bytes(cfg, kv_tokens, "fp32")
    return {
        "config": cfg["name"], "n_layers": cfg["n_layers"], "prompts": n_prompts, "prompt_len": prompt_len,
        "steps": n_steps, "threshold": threshold,
        "vs_layercast": {"bf16_no_recompute": strip(no_rc), "bf16_selective_recompute": strip(rc),
                         "recompute_gain_pp": 100.0 * (rc["exact_agreement"] - no_rc["exact_agreement"]),
                         "recompute_rate": rate},
        "vs_fp32": {"layercast": strip(compare(fp, ref)), "bf16_no_recompute": strip(compare(fp, b0)),
                    "bf16_selective_recompute": strip(compare(fp, b1))},
        "batch_alone_vs_batched": {"invariant": strip(compare(inv1, b1)), "fast": strip(compare(f_1, f_n))},
        "memory": {"allocated_weights_bf16": w_bf, "allocated_weights_layercast": w_lc,
                   "allocated_weights_fp32": w_fp, "allocated_kv_bf16": kv_bf, "allocated_kv_layercast": kv_lc,
                   "allocated_kv_fp32": kv_fp,
                   "measured_layercast_saving_vs_fp32": 1.0 - (w_lc + kv_lc) / (w_fp + kv_fp),
                   "layercast_bytes": lc, "fp32_storage_bytes": fpb, "layercast_saving_vs_fp32": 1.0 - lc / fpb,
                   "kv_positions": kv_tokens},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--config", default="tiny", choices=sorted(configs.CONFIGS))
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (0 = the config's)")
    ap.add_argument("--prompts", type=int, default=16)
    ap.add_argument("--prompt-len", type=int, default=64)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--threshold", type=float, default=0.1)
    a = ap.parse_args(argv)
    cfg = dict(configs.CONFIGS[a.config])
    if a.layers:
        cfg["n_layers"] = a.layers
    print(json.dumps(study(cfg, a.prompts, a.prompt_len, a.steps, a.threshold)))


if __name__ == "__main__":
    main()
